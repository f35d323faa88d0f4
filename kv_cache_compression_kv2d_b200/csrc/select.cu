// select.cu -- per-segment strategy generation under a byte budget (sm_100a).
//
// MosaicKV ("MosaicKV: Serving Long-Context LLM with Dynamic Two-D KV Cache
// Compression", Fig. 5: segment partitioning and compression-strategy
// generation) chooses one compression pattern per KV-cache segment.  The
// pages define no criterion; this library reads it as minimising lost
// attention mass under a byte budget:
//   seg_select (one thread per segment for r in {4, 8, 16}, S <= 128;
//   otherwise, and for the Token2Chunk variant, one warp per segment):
//     R_j = top-r tokens by s_t (ties to the lower token), ascending;
//     E_FULL = 0, E_TOK = sum_{t not in R} s_t, E_CH = sum_t s_t g_t,
//     E_BOTH = E_TOK + sum_{t in R} s_t g_t        (fp64, ascending t);
//     lower convex hull of (bytes, E) over the four strategies.
//   budget (one CTA per unit):
//     starts every segment at its cheapest hull point and applies hull steps
//     in (efficiency desc, segment asc, step asc) order while they fit the
//     budget, stopping at the first that does not.  The stopping step is
//     found exactly with a byte-weighted radix select over the 96-bit keys
//     (~bits(eff), 4 * segment + step); then per-segment strategies, payload
//     offsets (block scan) and descriptors are written.
// Every fp64 sum, product and quotient uses the _rn intrinsics so that no
// multiply-add is fused and the results are bit-identical to the same
// operations done one at a time in IEEE double precision.
#include <algorithm>

#include "kernels.h"

namespace kv2d {

namespace {

// Segments per CTA (one warp each, then one lane each).  Small CTAs: the
// sequential phases 2 and 3 keep only three warps (then one) busy, so eight
// CTAs of 8 warps per SM overlap one CTA's sequential phase with the
// others' ranking.
constexpr int kSegWarps = 8;
static_assert(kSegWarps >= 3 && kSegWarps <= 32, "phase 2 needs three warps; phases 2 and 3 give each segment one lane");

struct SegArgs {
    SeqPlan plan;
    int Hkv, S, r, max_nseg;
    int chunk_len, chunk_budget;   // Token2Chunk; chunk_len 0: plain top-r
    int64_t bytes[4];
    int32_t order[4];
    const float* s;
    int64_t s_stride;
    const double* g;
    int64_t g_stride;
    uint8_t* tidx;
    double* E;
    uint8_t* hull;
    double* eff;
    int32_t* dbytes;
    double* dbg_E;
    int32_t dbg_seg_stride;
};

// Shared memory of one CTA: per segment (row) the fp32 s_t, the fp64 s_t g_t
// and the kept flags, rows padded by one element so that lane-per-segment
// reads spread over the banks; then the three sums per segment.
__host__ __device__ constexpr int seg_row(int S) { return S + 1; }
inline int seg_smem_bytes(int S) {
    return kSegWarps * seg_row(S) * (8 + 4 + 1 + 2) + 3 * kSegWarps * 8 + 16;
}

// Token2Chunk on one segment by one lane (Kara, "What carries the
// argument"; the steps follow the library's reading): rk[t] is the rank of
// token t by (s desc, t asc) and inv[k] the token of rank k.  Writes kept[t].
__device__ void chunk_select(const float* srow, const uint8_t* rk, const uint8_t* inv, uint8_t* kept,
                             int S, int r, int alpha, int gamma) {
    const int ncore = r - alpha;
    for (int t = 0; t < S; ++t) kept[t] = rk[t] < ncore ? 1 : 0;
    // candidate gaps between consecutive core tokens (at most ncore - 1)
    double cm[32];
    int ca[32], cg[32];
    int nc = 0, prev = -1;
    for (int t = 0; t < S; ++t) {
        if (!kept[t]) continue;
        if (prev >= 0 && t - prev - 1 >= 1 && t - prev + 1 <= gamma && nc < 32) {
            double m = 0.0;
            for (int x = prev + 1; x < t; ++x) m = __dadd_rn(m, static_cast<double>(srow[x]));
            cm[nc] = m;
            ca[nc] = prev;
            cg[nc] = t - prev - 1;
            ++nc;
        }
        prev = t;
    }
    // by (merit desc, start asc)
    for (int i = 0; i < nc; ++i) {
        int best = i;
        for (int k = i + 1; k < nc; ++k)
            if (cm[k] > cm[best] || (cm[k] == cm[best] && ca[k] < ca[best])) best = k;
        const double tm = cm[i];
        const int ta = ca[i], tg = cg[i];
        cm[i] = cm[best];
        ca[i] = ca[best];
        cg[i] = cg[best];
        cm[best] = tm;
        ca[best] = ta;
        cg[best] = tg;
    }
    int rem = alpha;
    for (int i = 0; i < nc; ++i) {
        if (cg[i] > rem) continue;
        for (int x = ca[i] + 1; x <= ca[i] + cg[i]; ++x) kept[x] = 1;
        rem -= cg[i];
    }
    for (int k = 0; k < S && rem > 0; ++k) {
        const int t = inv[k];
        if (kept[t]) continue;
        kept[t] = 1;
        --rem;
    }
}

// The error proxies of segment js of unit u from its three sums, written
// out, and the lower convex hull of its options over (bytes, E).
__device__ __forceinline__ void finish_segment(const SegArgs& A, int u, int js, double ech, double ekept,
                                               double etok) {
    const int64_t slot = static_cast<int64_t>(u) * A.max_nseg + js;
    double E[4];
    E[KV2D_FULL] = 0.0;
    E[KV2D_TOK] = etok;
    E[KV2D_CH] = ech;
    E[KV2D_BOTH] = __dadd_rn(etok, ekept);
    for (int k = 0; k < 4; ++k) A.E[slot * 4 + k] = E[k];
    if (A.dbg_E)
        for (int k = 0; k < 4; ++k)
            A.dbg_E[(static_cast<int64_t>(u) * A.dbg_seg_stride + js) * 4 + k] = E[k];
    // lower convex hull over (bytes, E), options visited by (bytes, id)
    int hv[4];
    int nh = 0;
    hv[nh++] = A.order[0];
    for (int i = 1; i < 4; ++i) {
        const int o = A.order[i];
        const int last = hv[nh - 1];
        if (E[o] >= E[last]) continue;
        if (A.bytes[o] == A.bytes[last]) {
            hv[nh - 1] = o;
            continue;
        }
        while (nh >= 2) {
            const int pa = hv[nh - 2], pb = hv[nh - 1];
            const double lhs = __dmul_rn(__dsub_rn(E[pa], E[pb]),
                                         static_cast<double>(A.bytes[o] - A.bytes[pb]));
            const double rhs = __dmul_rn(__dsub_rn(E[pb], E[o]),
                                         static_cast<double>(A.bytes[pb] - A.bytes[pa]));
            if (lhs <= rhs) --nh;
            else break;
        }
        hv[nh++] = o;
    }
    uint8_t* H = A.hull + slot * 8;
    H[0] = static_cast<uint8_t>(nh);
    for (int k = 0; k < 4; ++k) H[1 + k] = static_cast<uint8_t>(k < nh ? hv[k] : 0);
    for (int k = 1; k < nh; ++k) {
        const int64_t db = A.bytes[hv[k]] - A.bytes[hv[k - 1]];
        A.dbytes[slot * 3 + k - 1] = static_cast<int32_t>(db);
        A.eff[slot * 3 + k - 1] =
            __ddiv_rn(__dsub_rn(E[hv[k - 1]], E[hv[k]]), static_cast<double>(db));
    }
}


// Phase 1, one warp per segment: R_j by rank counting (two tokens per lane
// and pass), tidx, kept flags, and the products s_t g_t.  Phase 2, one lane
// per segment: E_CH (warp 0), the kept part of E_BOTH (warp 1) and E_TOK
// (warp 2), each summed sequentially in ascending t.  Phase 3, one lane per
// segment: the error proxies and the lower hull.
__global__ void __launch_bounds__(kSegWarps * 32) seg_select_kernel(const __grid_constant__ SegArgs A) {
    pdl_wait();
    extern __shared__ __align__(16) uint8_t seg_smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int u = blockIdx.y;
    const int b = u / A.Hkv;
    const int nseg = A.plan.nseg[b];
    const int jb = blockIdx.x * kSegWarps;
    if (jb >= nseg) return;
    const int S = A.S, r = A.r, RW = seg_row(S);
    double* sgs = reinterpret_cast<double*>(seg_smem);                      // [kSegWarps][RW]
    double* sums = sgs + kSegWarps * RW;                                    // [3][kSegWarps]
    float* ss = reinterpret_cast<float*>(sums + 3 * kSegWarps);             // [kSegWarps][RW]
    uint8_t* kept = reinterpret_cast<uint8_t*>(ss + kSegWarps * RW);        // [kSegWarps][RW]
    uint8_t* rks = kept + kSegWarps * RW;                                   // [kSegWarps][RW] ranks
    uint8_t* invs = rks + kSegWarps * RW;                                   // [kSegWarps][RW] rank -> t
    const bool chunk = A.chunk_len > 0;

    const int j = jb + warp;
    if (j < nseg) {
        const int64_t t0 = static_cast<int64_t>(j) * S;
        float* srow = ss + warp * RW;
        for (int t = lane; t < S; t += 32) {
            const float sv = A.s[static_cast<int64_t>(u) * A.s_stride + t0 + t];
            srow[t] = sv;
            sgs[warp * RW + t] = __dmul_rn(static_cast<double>(sv), A.g[static_cast<int64_t>(u) * A.g_stride + t0 + t]);
        }
        __syncwarp();
        const int64_t slot = static_cast<int64_t>(u) * A.max_nseg + j;
        int before = 0;
        for (int tb = 0; tb < S; tb += 64) {
            // two tokens per lane and pass: t = tb + lane and tb + 32 + lane
            const int ta = tb + lane, tc = tb + 32 + lane;
            const float va = (ta < S) ? srow[ta] : 0.f;
            const float vc = (tc < S) ? srow[tc] : 0.f;
            int ra = 0, rc = 0;
            for (int t2 = 0; t2 < S; ++t2) {
                const float v2 = srow[t2];
                ra += (v2 > va) || (v2 == va && t2 < ta);
                rc += (v2 > vc) || (v2 == vc && t2 < tc);
            }
            if (chunk) {
                if (ta < S) {
                    rks[warp * RW + ta] = static_cast<uint8_t>(ra);
                    invs[warp * RW + ra] = static_cast<uint8_t>(ta);
                }
                if (tc < S) {
                    rks[warp * RW + tc] = static_cast<uint8_t>(rc);
                    invs[warp * RW + rc] = static_cast<uint8_t>(tc);
                }
                continue;
            }
            const bool ka = ta < S && ra < r, kc = tc < S && rc < r;
            if (ta < S) kept[warp * RW + ta] = ka ? 1 : 0;
            if (tc < S) kept[warp * RW + tc] = kc ? 1 : 0;
            const uint32_t lt = (1u << lane) - 1u;
            const uint32_t ba = __ballot_sync(0xffffffffu, ka);
            if (ka) A.tidx[slot * r + before + __popc(ba & lt)] = static_cast<uint8_t>(ta);
            before += __popc(ba);
            const uint32_t bc = __ballot_sync(0xffffffffu, kc);
            if (kc) A.tidx[slot * r + before + __popc(bc & lt)] = static_cast<uint8_t>(tc);
            before += __popc(bc);
        }
        if (chunk) {
            __syncwarp();
            if (lane == 0) {
                chunk_select(srow, rks + warp * RW, invs + warp * RW, kept + warp * RW, S, r,
                             A.chunk_budget, A.chunk_len);
                int w = 0;
                for (int t = 0; t < S; ++t)
                    if (kept[warp * RW + t]) A.tidx[slot * r + w++] = static_cast<uint8_t>(t);
            }
        }
    }
    __syncthreads();
    if (warp < 3 && lane < kSegWarps && jb + lane < nseg) {
        // lane <-> segment jb + lane; the fp64 sums in ascending t
        double acc = 0.0;
        const double* grow = sgs + lane * RW;
        const float* srow = ss + lane * RW;
        const uint8_t* krow = kept + lane * RW;
#pragma unroll 8
        for (int t = 0; t < S; ++t) {
            const bool kp = krow[t] != 0;
            if (warp == 0) acc = __dadd_rn(acc, grow[t]);
            else if (warp == 1) { if (kp) acc = __dadd_rn(acc, grow[t]); }
            else if (!kp) acc = __dadd_rn(acc, static_cast<double>(srow[t]));
        }
        sums[warp * kSegWarps + lane] = acc;
    }
    __syncthreads();
    if (warp != 0 || lane >= kSegWarps || jb + lane >= nseg) return;
    finish_segment(A, u, jb + lane, sums[lane], sums[kSegWarps + lane], sums[2 * kSegWarps + lane]);
}

// One thread per segment, for r a power of two in {4, 8, 16} with S <= 128
// (the default shapes: S = 64, r = 8 and S = 128, r = 16).  A warp stages
// the s_t and g_t of its 32 consecutive segments (contiguous in memory)
// through shared memory with coalesced 16-byte loads; rows are padded so
// that each thread's 16-byte reads of its own row hit distinct bank groups.
// Top-r: each token becomes one 64-bit key, bits(s_t) << 8 | (255 - t),
// which orders by s_t (non-negative, so its bits are monotone) and then by
// the lower t; read as an fp64 number the key is a positive subnormal whose
// order is the key's, so fmax / fmin sort it exactly (min / max return one
// of their operands).  Groups of R keys are sorted by a bitonic network and
// merged into the running R largest (max against the reversed group, then
// a bitonic merge).  Then the three sums in ascending t and the hull, as in
// the general kernel.
constexpr int kSmallSegs = 32;

// 16 / 8 / 4 bytes global -> shared by this thread, asynchronously; both
// addresses aligned to the size.
__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async8(void* dst, const void* src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async4(void* dst, const void* src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}

template <int N>
__device__ __forceinline__ void bitonic_sort_desc(double (&v)[N]) {
#pragma unroll
    for (int k = 2; k <= N; k <<= 1) {
#pragma unroll
        for (int j = k >> 1; j > 0; j >>= 1) {
#pragma unroll
            for (int i = 0; i < N; ++i) {
                const int l = i ^ j;
                if (l > i) {
                    const double hi = fmax(v[i], v[l]), lo = fmin(v[i], v[l]);
                    v[i] = (i & k) == 0 ? hi : lo;
                    v[l] = (i & k) == 0 ? lo : hi;
                }
            }
        }
    }
}

template <int N>
__device__ __forceinline__ void bitonic_merge_desc(double (&v)[N]) {
#pragma unroll
    for (int j = N >> 1; j > 0; j >>= 1) {
#pragma unroll
        for (int i = 0; i < N; ++i) {
            const int l = i ^ j;
            if (l > i) {
                const double hi = fmax(v[i], v[l]), lo = fmin(v[i], v[l]);
                v[i] = hi;
                v[l] = lo;
            }
        }
    }
}

inline int seg_small_smem_bytes(int S) { return kSmallSegs * ((S + 4) * 4 + (S + 2) * 8); }

template <int R>
__global__ void __launch_bounds__(kSmallSegs) seg_select_small_kernel(const __grid_constant__ SegArgs A) {
    pdl_wait();
    extern __shared__ __align__(16) uint8_t seg_smem[];
    const int lane = threadIdx.x;
    const int u = blockIdx.y;
    const int b = u / A.Hkv;
    const int nseg = A.plan.nseg[b];
    const int jb = blockIdx.x * kSmallSegs;
    if (jb >= nseg) return;
    const int S = A.S, SR = S + 4, GR = S + 2;
    float* srows = reinterpret_cast<float*>(seg_smem);                          // [32][S + 4]
    double* grows = reinterpret_cast<double*>(srows + kSmallSegs * SR);         // [32][S + 2]
    const int nv = min(kSmallSegs, nseg - jb);
    {
        // every 16-byte piece is an asynchronous copy issued back to back,
        // then one wait: the warp pays the L2 latency once, not once per
        // load (at small sizes it is alone on its SM)
        const float4* s4 = reinterpret_cast<const float4*>(A.s + static_cast<int64_t>(u) * A.s_stride +
                                                           static_cast<int64_t>(jb) * S);
        const int q4 = S / 4, n4 = nv * q4;
        for (int i = lane; i < n4; i += kSmallSegs)
            cp_async16(srows + (i / q4) * SR + 4 * (i % q4), s4 + i);
        const double2* g2 = reinterpret_cast<const double2*>(A.g + static_cast<int64_t>(u) * A.g_stride +
                                                             static_cast<int64_t>(jb) * S);
        const int q2 = S / 2, n2 = nv * q2;
        for (int i = lane; i < n2; i += kSmallSegs)
            cp_async16(grows + (i / q2) * GR + 2 * (i % q2), g2 + i);
        asm volatile("cp.async.wait_all;" ::: "memory");
    }
    __syncwarp();
    if (lane >= nv) return;
    const int js = jb + lane;
    const float* srow = srows + lane * SR;
    const double* grow = grows + lane * GR;
    auto key_of = [&](float sv, int t) {
        return __longlong_as_double(static_cast<long long>(
            (static_cast<uint64_t>(__float_as_uint(sv)) << 8) | static_cast<uint64_t>(255 - t)));
    };
    double top[R];
    for (int g0 = 0; g0 < S; g0 += R) {
        double cur[R];
#pragma unroll
        for (int i = 0; i < R; i += 4) {
            const float4 v4 = *reinterpret_cast<const float4*>(srow + g0 + i);
            cur[i] = key_of(v4.x, g0 + i);
            cur[i + 1] = key_of(v4.y, g0 + i + 1);
            cur[i + 2] = key_of(v4.z, g0 + i + 2);
            cur[i + 3] = key_of(v4.w, g0 + i + 3);
        }
        bitonic_sort_desc<R>(cur);
        if (g0 == 0) {
#pragma unroll
            for (int i = 0; i < R; ++i) top[i] = cur[i];
        } else {
#pragma unroll
            for (int i = 0; i < R; ++i) top[i] = fmax(top[i], cur[R - 1 - i]);
            bitonic_merge_desc<R>(top);
        }
    }
    // kept tokens as a 128-bit mask, then tidx ascending
    uint64_t k0 = 0, k1 = 0;
#pragma unroll
    for (int i = 0; i < R; ++i) {
        const int t = 255 - static_cast<int>(__double_as_longlong(top[i]) & 255);
        if (t < 64) k0 |= 1ull << t;
        else k1 |= 1ull << (t - 64);
    }
    const int64_t slot = static_cast<int64_t>(u) * A.max_nseg + js;
    {
        uint64_t m0 = k0, m1 = k1;
#pragma unroll
        for (int i = 0; i < R; ++i) {
            int t;
            if (m0) {
                t = __ffsll(static_cast<long long>(m0)) - 1;
                m0 &= m0 - 1;
            } else {
                t = 64 + __ffsll(static_cast<long long>(m1)) - 1;
                m1 &= m1 - 1;
            }
            A.tidx[slot * R + i] = static_cast<uint8_t>(t);
        }
    }
    // the three fp64 sums in ascending t (products and sums rounded once)
    double ech = 0.0, ekept = 0.0, etok = 0.0;
    for (int t0 = 0; t0 < S; t0 += 4) {
        const float4 v4 = *reinterpret_cast<const float4*>(srow + t0);
        const double2 ga = *reinterpret_cast<const double2*>(grow + t0);
        const double2 gb = *reinterpret_cast<const double2*>(grow + t0 + 2);
        const float sv[4] = {v4.x, v4.y, v4.z, v4.w};
        const double gv[4] = {ga.x, ga.y, gb.x, gb.y};
        const uint64_t kw = (t0 < 64) ? (k0 >> t0) : (k1 >> (t0 - 64));
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const double sd = static_cast<double>(sv[e]);
            const double p = __dmul_rn(sd, gv[e]);
            ech = __dadd_rn(ech, p);
            if ((kw >> e) & 1) ekept = __dadd_rn(ekept, p);
            else etok = __dadd_rn(etok, sd);
        }
    }
    finish_segment(A, u, js, ech, ekept, etok);
}

// ---------------------------------------------------------------- budget

constexpr int kBudgetThreads = 1024;

struct BudgetArgs {
    SeqPlan plan;
    int Hkv, S, max_nseg;
    int64_t bytes[4];
    int all_full;
    const uint8_t* hull;
    const double* eff;
    const int32_t* dbytes;
    uint8_t* strat;
    int32_t* unit_ok;
    uint64_t* desc;
    int32_t max_segs;
    const int64_t* used_bytes;     // live: where this call's segments start
    int32_t* out_n_segs;           // where the new bookkeeping goes (live or staged)
    int64_t* out_used_bytes;
    int32_t* out_comp_end;
    int64_t arena_stride;
    uint32_t* status;
};

__device__ __forceinline__ long long block_sum(long long v, long long* red) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    __syncthreads();
    if (lane == 0) red[warp] = v;
    __syncthreads();
    long long t = 0;
    if (warp == 0) {
        t = (lane < (blockDim.x >> 5)) ? red[lane] : 0;
        for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
        if (lane == 0) red[32] = t;
    }
    __syncthreads();
    return red[32];
}

// Exclusive block scan; returns this thread's prefix and writes the block
// total to *total.
__device__ __forceinline__ long long block_exscan(long long v, long long* red, long long* total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    long long inc = v;
    for (int o = 1; o < 32; o <<= 1) {
        const long long n = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += n;
    }
    __syncthreads();
    if (lane == 31) red[warp] = inc;
    __syncthreads();
    if (warp == 0) {
        long long w = (lane < (blockDim.x >> 5)) ? red[lane] : 0;
        long long wi = w;
        for (int o = 1; o < 32; o <<= 1) {
            const long long n = __shfl_up_sync(0xffffffffu, wi, o);
            if (lane >= o) wi += n;
        }
        red[lane] = wi - w;            // exclusive warp offsets
        if (lane == 31) red[32] = wi;  // total
    }
    __syncthreads();
    const long long res = red[warp] + inc - v;
    *total = red[32];
    return res;
}

__device__ __forceinline__ uint64_t upg_hi(double eff) {
    return ~static_cast<uint64_t>(__double_as_longlong(eff));
}

// Per-segment hull data cached in shared memory when it fits.
constexpr int kBudgetCacheSegs = 2048;
constexpr int kBudgetSmem = kBudgetCacheSegs * (8 + 3 * 8 + 3 * 4);

__global__ void __launch_bounds__(kBudgetThreads) budget_kernel(const __grid_constant__ BudgetArgs A) {
    pdl_wait();
    const int u = blockIdx.x;
    const int b = u / A.Hkv, h = u % A.Hkv;
    const int nseg = A.plan.nseg[b];
    const int tid = threadIdx.x;
    if (nseg == 0) {
        if (tid == 0) A.unit_ok[u] = 1;
        return;
    }
    __shared__ unsigned long long hist[256];
    __shared__ unsigned int hcnt[256];
    __shared__ long long red[33];
    __shared__ uint64_t s_phi;
    __shared__ uint32_t s_plo;
    __shared__ long long s_below;
    __shared__ int s_mode;            // 0 all full, 1 all steps, 2 threshold
    __shared__ int s_unique;
    const uint8_t* H = A.hull + static_cast<int64_t>(u) * A.max_nseg * 8;
    const double* EF = A.eff + static_cast<int64_t>(u) * A.max_nseg * 3;
    const int32_t* DB = A.dbytes + static_cast<int64_t>(u) * A.max_nseg * 3;
    extern __shared__ __align__(16) uint8_t budget_smem[];
    if (nseg <= kBudgetCacheSegs) {
        double* efs = reinterpret_cast<double*>(budget_smem);
        int32_t* dbs = reinterpret_cast<int32_t*>(efs + 3 * kBudgetCacheSegs);
        uint8_t* hs = reinterpret_cast<uint8_t*>(dbs + 3 * kBudgetCacheSegs);
        // asynchronous copies issued back to back, one wait: the L2 latency
        // is paid once, not once per iteration
        for (int i = tid; i < nseg * 3; i += kBudgetThreads) {
            cp_async8(efs + i, EF + i);
            cp_async4(dbs + i, DB + i);
        }
        for (int i = tid; i < nseg * 2; i += kBudgetThreads)
            cp_async4(reinterpret_cast<uint32_t*>(hs) + i, reinterpret_cast<const uint32_t*>(H) + i);
        asm volatile("cp.async.wait_all;" ::: "memory");
        __syncthreads();
        H = hs;
        EF = efs;
        DB = dbs;
    }

    long long base_p = 0, wsum_p = 0;
    for (int j = tid; j < nseg; j += kBudgetThreads) {
        const int nv = H[j * 8];
        base_p += A.bytes[H[j * 8 + 1]];
        for (int k = 1; k < nv; ++k) wsum_p += DB[j * 3 + k - 1];
    }
    const long long base = block_sum(base_p, red);
    const long long wsum = block_sum(wsum_p, red);
    const long long rem = A.plan.Bu[b] - base;
    if (tid == 0) {
        s_mode = A.all_full ? 0 : (wsum <= rem ? 1 : 2);
        s_phi = 0;
        s_plo = 0;
        s_below = 0;
        s_unique = 0;
    }
    __syncthreads();
    const int mode = s_mode;
    // Weighted radix select of the stopping step: the smallest 96-bit key
    // (hi = ~bits(eff), lo = 4 * segment + step) whose prefix weight exceeds
    // rem.  8-bit digits from the top; the search ends early once the chosen
    // digit bucket holds a single key (that key is the answer).
    for (int dp = 0; mode == 2 && dp < 12; ++dp) {
        for (int i = tid; i < 256; i += kBudgetThreads) {
            hist[i] = 0;
            hcnt[i] = 0;
        }
        __syncthreads();
        const uint64_t phi = s_phi;
        const uint32_t plo = s_plo;
        // all lanes of a warp step through (segment, step) slots together so
        // that equal digits can be combined into one atomic per warp
        const int lane = tid & 31;
        for (int j0 = tid - lane; j0 < nseg; j0 += kBudgetThreads) {
            const int j = j0 + lane;
            const int nv = (j < nseg) ? H[j * 8] : 0;
            for (int k = 1; k < 4; ++k) {
                int digit = -1;
                uint32_t w = 0;
                if (k < nv) {
                    const uint64_t hi = upg_hi(EF[j * 3 + k - 1]);
                    const uint32_t lo = static_cast<uint32_t>(j * 4 + k);
                    bool match;
                    int dg;
                    if (dp < 8) {
                        const int sh = 64 - 8 * dp;   // bits above the digit
                        match = (dp == 0) || ((hi >> sh) == (phi >> sh));
                        dg = static_cast<int>((hi >> (56 - 8 * dp)) & 255u);
                    } else {
                        const int dl = dp - 8;
                        const int sh = 32 - 8 * dl;
                        match = (hi == phi) && (dl == 0 || (lo >> sh) == (plo >> sh));
                        dg = static_cast<int>((lo >> (24 - 8 * dl)) & 255u);
                    }
                    if (match) {
                        digit = dg;
                        w = static_cast<uint32_t>(DB[j * 3 + k - 1]);
                    }
                }
                const uint32_t peers = __match_any_sync(0xffffffffu, digit);
                const uint32_t wsum = __reduce_add_sync(peers, w);
                if (digit >= 0 && lane == __ffs(peers) - 1) {
                    atomicAdd(&hist[digit], static_cast<unsigned long long>(wsum));
                    atomicAdd(&hcnt[digit], static_cast<unsigned>(__popc(peers)));
                }
            }
        }
        __syncthreads();
        if (tid < 32) {
            // lane l owns buckets 8l .. 8l+7; find the first bucket where the
            // running weight (below + everything before it + it) exceeds rem
            const int lane = tid;
            long long wl = 0;
#pragma unroll
            for (int i = 0; i < 8; ++i) wl += static_cast<long long>(hist[lane * 8 + i]);
            long long incl = wl;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const long long n = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += n;
            }
            long long cum = s_below + (incl - wl);
            int found = -1;
            long long before = 0;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const long long hw = static_cast<long long>(hist[lane * 8 + i]);
                if (found < 0 && cum + hw > rem) {
                    found = lane * 8 + i;
                    before = cum;
                }
                cum += hw;
            }
            const uint32_t bal = __ballot_sync(0xffffffffu, found >= 0);
            const int src = bal ? (__ffs(bal) - 1) : 31;
            const int v = __shfl_sync(0xffffffffu, bal ? found : 255, src);
            const long long bv = __shfl_sync(0xffffffffu, before, src);
            if (lane == 0) {
                s_below = bal ? bv : s_below;
                if (dp < 8) s_phi |= static_cast<uint64_t>(v) << (56 - 8 * dp);
                else s_plo |= static_cast<uint32_t>(v) << (24 - 8 * (dp - 8));
                s_unique = (hcnt[v] == 1u);
            }
        }
        __syncthreads();
        if (s_unique) {
            // the bucket holds one key: complete the prefix with its bits
            const uint64_t phi2 = s_phi;
            const uint32_t plo2 = s_plo;
            for (int j = tid; j < nseg; j += kBudgetThreads) {
                const int nv = H[j * 8];
                for (int k = 1; k < nv; ++k) {
                    const uint64_t hi = upg_hi(EF[j * 3 + k - 1]);
                    const uint32_t lo = static_cast<uint32_t>(j * 4 + k);
                    bool match;
                    if (dp < 8) {
                        const int sh = 56 - 8 * dp;   // bits down to this digit
                        match = (hi >> sh) == (phi2 >> sh);
                    } else {
                        const int sh = 24 - 8 * (dp - 8);
                        match = (hi == phi2) && ((lo >> sh) == (plo2 >> sh));
                    }
                    if (match) {
                        s_phi = hi;
                        s_plo = lo;
                    }
                }
            }
            __syncthreads();
            break;
        }
    }
    const uint64_t phi = s_phi;
    const uint32_t plo = s_plo;

    // strategies and their total bytes
    long long tot_p = 0;
    uint8_t* ST = A.strat + static_cast<int64_t>(u) * A.max_nseg;
    for (int j = tid; j < nseg; j += kBudgetThreads) {
        const int nv = H[j * 8];
        int st;
        if (mode == 0) {
            st = KV2D_FULL;
        } else {
            int level = nv - 1;
            if (mode == 2) {
                level = 0;
                for (int k = 1; k < nv; ++k) {
                    const uint64_t hi = upg_hi(EF[j * 3 + k - 1]);
                    const uint32_t lo = static_cast<uint32_t>(j * 4 + k);
                    if (hi < phi || (hi == phi && lo < plo)) level = k;
                }
            }
            st = H[j * 8 + 1 + level];
        }
        ST[j] = static_cast<uint8_t>(st);
        tot_p += A.bytes[st];
    }
    const long long total = block_sum(tot_p, red);
    const long long used0 = A.used_bytes[u];
    const int segbase = A.plan.r0[b] / A.S;
    if (used0 + total > A.arena_stride || segbase + nseg > A.max_segs) {
        if (tid == 0) {
            set_status(A.status, KV2D_DEV_CAPACITY);
            A.unit_ok[u] = 0;
        }
        return;
    }
    long long carry = used0;
    for (int j0 = 0; j0 < nseg; j0 += kBudgetThreads) {
        const int j = j0 + tid;
        const long long nb = (j < nseg) ? A.bytes[ST[j]] : 0;
        long long chunk_total;
        const long long off = carry + block_exscan(nb, red, &chunk_total);
        if (j < nseg) {
            const uint64_t d = (static_cast<uint64_t>(off >> 4) & 0xffffffffull) |
                               (static_cast<uint64_t>(ST[j]) << 32);
            A.desc[static_cast<int64_t>(u) * A.max_segs + segbase + j] = d;
        }
        carry += chunk_total;
        __syncthreads();
    }
    if (tid == 0) {
        A.out_used_bytes[u] = used0 + total;
        A.out_n_segs[u] = segbase + nseg;
        if (h == 0) A.out_comp_end[b] = A.plan.r0[b] + nseg * A.S;
        A.unit_ok[u] = 1;
    }
}

// Publishes a staged compression: the staged bookkeeping becomes the live
// one (one thread per unit, and per sequence for comp_end).
struct PublishArgs {
    int units, batch;
    const int32_t* st_n_segs;
    const int64_t* st_used_bytes;
    const int32_t* st_comp_end;
    int32_t* n_segs;
    int64_t* used_bytes;
    int32_t* comp_end;
};

__global__ void publish_kernel(const __grid_constant__ PublishArgs A) {
    pdl_wait();
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i < A.units) {
        A.n_segs[i] = A.st_n_segs[i];
        A.used_bytes[i] = A.st_used_bytes[i];
    }
    if (i < A.batch) A.comp_end[i] = A.st_comp_end[i];
}

}  // namespace

cudaError_t launch_publish(int units, int batch, const int32_t* st_n_segs, const int64_t* st_used,
                           const int32_t* st_comp_end, int32_t* n_segs, int64_t* used, int32_t* comp_end,
                           cudaStream_t stream) {
    PublishArgs a{units, batch, st_n_segs, st_used, st_comp_end, n_segs, used, comp_end};
    const int n = std::max(units, batch);
    return launch_k(publish_kernel, dim3((n + 255) / 256), dim3(256), 0, stream, a);
}

cudaError_t launch_selection(const SelectLaunch& L, cudaStream_t stream) {
    const int units = L.batch * L.shp.Hkv;
    if (L.max_nseg > 0) {
        SegArgs sa;
        sa.plan = L.plan;
        sa.Hkv = L.shp.Hkv;
        sa.S = L.shp.S;
        sa.r = L.shp.r;
        sa.max_nseg = L.max_nseg;
        sa.chunk_len = L.shp.chunk_len;
        sa.chunk_budget = L.shp.chunk_budget;
        for (int k = 0; k < 4; ++k) {
            sa.bytes[k] = L.bytes[k];
            sa.order[k] = L.order[k];
        }
        sa.s = L.s;
        sa.s_stride = L.s_stride;
        sa.g = L.g;
        sa.g_stride = L.g_stride;
        sa.tidx = L.tidx;
        sa.E = L.E;
        sa.hull = L.hull;
        sa.eff = L.eff;
        sa.dbytes = L.dbytes;
        sa.dbg_E = L.dbg_E;
        sa.dbg_seg_stride = L.dbg_seg_stride;
        const int r = sa.r;
        const bool small = sa.chunk_len == 0 && sa.S <= 128 && (r == 4 || r == 8 || r == 16) && sa.S % r == 0;
        prof_begin(stream, kProfSegSelect);
        if (small) {
            dim3 grid((L.max_nseg + kSmallSegs - 1) / kSmallSegs, units);
            const int sm_bytes = seg_small_smem_bytes(sa.S);
            auto kern = r == 4 ? seg_select_small_kernel<4> : r == 8 ? seg_select_small_kernel<8>
                                                                      : seg_select_small_kernel<16>;
            cudaError_t e0 = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, sm_bytes);
            if (e0 != cudaSuccess) return e0;
            cudaError_t e1 = launch_k(kern, grid, dim3(kSmallSegs), sm_bytes, stream, sa);
            if (e1 != cudaSuccess) return e1;
        } else {
            dim3 grid((L.max_nseg + kSegWarps - 1) / kSegWarps, units);
            const int sm_bytes = seg_smem_bytes(sa.S);
            cudaError_t e0 = cudaFuncSetAttribute(seg_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, sm_bytes);
            if (e0 != cudaSuccess) return e0;
            cudaError_t e1 = launch_k(seg_select_kernel, grid, dim3(kSegWarps * 32), sm_bytes, stream, sa);
            if (e1 != cudaSuccess) return e1;
        }
        prof_end(stream, kProfSegSelect);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    BudgetArgs ba;
    ba.plan = L.plan;
    ba.Hkv = L.shp.Hkv;
    ba.S = L.shp.S;
    ba.max_nseg = L.max_nseg;
    for (int k = 0; k < 4; ++k) ba.bytes[k] = L.bytes[k];
    ba.all_full = L.all_full;
    ba.hull = L.hull;
    ba.eff = L.eff;
    ba.dbytes = L.dbytes;
    ba.strat = L.strat;
    ba.unit_ok = L.unit_ok;
    ba.desc = L.desc;
    ba.max_segs = L.max_segs;
    ba.used_bytes = L.used_bytes;
    ba.out_n_segs = L.out_n_segs ? L.out_n_segs : L.n_segs;
    ba.out_used_bytes = L.out_used_bytes ? L.out_used_bytes : L.used_bytes;
    ba.out_comp_end = L.out_comp_end ? L.out_comp_end : L.comp_end;
    ba.arena_stride = L.arena_stride;
    ba.status = L.status;
    prof_begin(stream, kProfBudget);
    cudaError_t e = cudaFuncSetAttribute(budget_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         kBudgetSmem);
    if (e != cudaSuccess) return e;
    e = launch_k(budget_kernel, dim3(units), dim3(kBudgetThreads), kBudgetSmem, stream, ba);
    if (e != cudaSuccess) return e;
    prof_end(stream, kProfBudget);
    return cudaGetLastError();
}

}  // namespace kv2d
