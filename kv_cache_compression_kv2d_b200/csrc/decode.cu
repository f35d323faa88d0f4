// decode.cu -- KV append and decode attention over the packed segments
// (sm_100a).
//
// MosaicKV ("MosaicKV: Serving Long-Context LLM with Dynamic Two-D KV Cache
// Compression", Sec. 5.3 PackedAttention and Fig. 6 packed sparse attention)
// runs decode attention directly on the compressed segments.  Here one unit
// (sequence b, KV head h) serves its G query heads from every byte it loads:
//   - the unit's work is its packed arena plus its dense tail
//     [comp_end, seq_len), 512 bytes per dense token; the kernel splits that
//     byte range evenly over nsplit CTAs (a CTA takes the segments whose
//     first byte falls in its range, found by binary search on the
//     descriptors, and the tail tokens likewise);
//   - each warp streams whole segments, 32/G tokens per step, with 8-byte
//     coalesced loads per lane: FULL / TOK / dense rows as d-slices, CH / BOTH
//     keys as (index, value) pairs gathered against q in shared memory;
//   - scores meet an online softmax per head in the log2 domain; warps, then
//     CTAs, merge their (max, sum, output) partials in a fixed order, the
//     last CTA of a unit (atomic ticket) writing the fp16 output.
#include "kernels.h"

namespace kv2d {

namespace {

constexpr int kDecWarps = 8;
constexpr int kDecThreads = kDecWarps * 32;
constexpr float kNegInfF = -__builtin_huge_valf();

// ------------------------------------------------------------------ append

__global__ void append_kernel(const __grid_constant__ AppendLaunch A) {
    const int b = blockIdx.x;
    __shared__ int ok;
    const int t = A.seq_len[b];
    if (threadIdx.x == 0) ok = 1;
    __syncthreads();
    for (int idx = threadIdx.x; idx < A.Hkv * 32; idx += blockDim.x) {
        const int h = idx >> 5, part = idx & 31;
        const int ch = part & 15;
        const bool isv = part >= 16;
        __half* row = dense_row(A.dv, isv ? A.v : A.k, b, h, t, A.status);
        if (!row) {
            ok = 0;
            continue;
        }
        const __half* src = (isv ? A.v_new : A.k_new) + (static_cast<int64_t>(b) * A.Hkv + h) * kHeadDim;
        *reinterpret_cast<uint4*>(row + ch * 8) = *reinterpret_cast<const uint4*>(src + ch * 8);
    }
    __syncthreads();
    if (threadIdx.x == 0 && ok) A.seq_len[b] = t + 1;
}

// ------------------------------------------------------------------ decode

template <int G>
struct WarpState {
    float m[G];        // running max per head (log2 domain), same in all lanes
    float lp;          // partial softmax sum of this lane's (token, head) pairs
    float o[G][4];     // output accumulators: heads x this lane's 4 channels
};

__device__ __forceinline__ void half4_to_float(uint2 v, float (&f)[4]) {
    const __half2 a = *reinterpret_cast<const __half2*>(&v.x);
    const __half2 c = *reinterpret_cast<const __half2*>(&v.y);
    const float2 fa = __half22float2(a), fc = __half22float2(c);
    f[0] = fa.x;
    f[1] = fa.y;
    f[2] = fc.x;
    f[3] = fc.y;
}

// Reduces 32 per-lane values across the warp so that lane l ends with the
// full sum of value index l (value index = token * G + head).
__device__ __forceinline__ float transpose_reduce32(float (&v)[32]) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const bool up = lane & 16;
        const float send = up ? v[i] : v[i + 16];
        const float keep = up ? v[i + 16] : v[i];
        v[i] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const bool up = lane & 8;
        const float send = up ? v[i] : v[i + 8];
        const float keep = up ? v[i + 8] : v[i];
        v[i] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const bool up = lane & 4;
        const float send = up ? v[i] : v[i + 4];
        const float keep = up ? v[i + 4] : v[i];
        v[i] = keep + __shfl_xor_sync(0xffffffffu, send, 4);
    }
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const bool up = lane & 2;
        const float send = up ? v[i] : v[i + 2];
        const float keep = up ? v[i + 2] : v[i];
        v[i] = keep + __shfl_xor_sync(0xffffffffu, send, 2);
    }
    {
        const bool up = lane & 1;
        const float send = up ? v[0] : v[1];
        const float keep = up ? v[1] : v[0];
        v[0] = keep + __shfl_xor_sync(0xffffffffu, send, 1);
    }
    return v[0];
}

// Same within groups of G lanes for G values.
template <int G>
__device__ __forceinline__ float transpose_reduce_group(float (&v)[G]) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int s = G / 2; s >= 1; s >>= 1) {
#pragma unroll
        for (int i = 0; i < s; ++i) {
            const bool up = lane & s;
            const float send = up ? v[i] : v[i + s];
            const float keep = up ? v[i + s] : v[i];
            v[i] = keep + __shfl_xor_sync(0xffffffffu, send, s);
        }
    }
    return v[0];
}

// One softmax step: lane l holds the score x of (token l / G, head l % G)
// (valid == false -> not a token), vs[tt] holds this lane's 4 channels of
// token tt's value row.  p_s is a 32-float per-warp scratch.
template <int G>
__device__ __forceinline__ void softmax_step(WarpState<G>& st, float x, bool valid,
                                             const uint2 (&vs)[32 / G], float* p_s) {
    constexpr int TB = 32 / G;
    const int lane = threadIdx.x & 31;
    const int gl = lane % G;
    x = valid ? x : kNegInfF;
    float mx = x;
#pragma unroll
    for (int s = G; s < 32; s <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, s));
    float alpha[G];
    float mine = kNegInfF;
    bool changed = false;
#pragma unroll
    for (int g = 0; g < G; ++g) {
        const float mh = __shfl_sync(0xffffffffu, mx, g);
        const float mn = fmaxf(st.m[g], mh);
        alpha[g] = (st.m[g] == mn) ? 1.f : fast_exp2(st.m[g] - mn);
        changed |= (st.m[g] != mn);
        st.m[g] = mn;
        if (g == gl) mine = mn;
    }
    float al = 1.f;
#pragma unroll
    for (int g = 0; g < G; ++g)
        if (g == gl) al = alpha[g];
    const float p = valid ? fast_exp2(x - mine) : 0.f;
    st.lp = st.lp * al + p;
    if (__any_sync(0xffffffffu, changed)) {
#pragma unroll
        for (int g = 0; g < G; ++g)
#pragma unroll
            for (int e = 0; e < 4; ++e) st.o[g][e] *= alpha[g];
    }
    p_s[lane] = p;
    __syncwarp();
#pragma unroll
    for (int tt = 0; tt < TB; ++tt) {
        float vf[4];
        half4_to_float(vs[tt], vf);
#pragma unroll
        for (int g = 0; g < G; ++g) {
            const float pg = p_s[tt * G + g];
#pragma unroll
            for (int e = 0; e < 4; ++e) st.o[g][e] = fmaf(pg, vf[e], st.o[g][e]);
        }
    }
    __syncwarp();
}

// Dense key rows: krow(i) / vrow(i) give row i's pointers (nullptr -> skip).
template <int G, typename RowK, typename RowV>
__device__ __forceinline__ void dense_rows(WarpState<G>& st, int ntok, RowK krow, RowV vrow,
                                           const float (&qr)[G][4], float* p_s) {
    constexpr int TB = 32 / G;
    const int lane = threadIdx.x & 31;
    for (int t0 = 0; t0 < ntok; t0 += TB) {
        uint2 ks[TB], vs[TB];
#pragma unroll
        for (int tt = 0; tt < TB; ++tt) {
            ks[tt] = make_uint2(0, 0);
            vs[tt] = make_uint2(0, 0);
            if (t0 + tt < ntok) {
                const __half* kp = krow(t0 + tt);
                const __half* vp = vrow(t0 + tt);
                if (kp) ks[tt] = *reinterpret_cast<const uint2*>(kp + lane * 4);
                if (vp) vs[tt] = *reinterpret_cast<const uint2*>(vp + lane * 4);
            }
        }
        float part[32];
#pragma unroll
        for (int tt = 0; tt < TB; ++tt) {
            float kf[4];
            half4_to_float(ks[tt], kf);
#pragma unroll
            for (int g = 0; g < G; ++g) {
                float a = qr[g][0] * kf[0];
                a = fmaf(qr[g][1], kf[1], a);
                a = fmaf(qr[g][2], kf[2], a);
                a = fmaf(qr[g][3], kf[3], a);
                part[tt * G + g] = a;
            }
        }
        const float x = transpose_reduce32(part);
        const bool valid = (t0 + lane / G) < ntok;
        softmax_step<G>(st, x, valid, vs, p_s);
    }
}

// Channel-sparse keys: ci[t][c] indices, kv[t][c] fp16 values, V rows dense.
template <int G>
__device__ __forceinline__ void sparse_rows(WarpState<G>& st, int ntok, int c, const uint8_t* ci,
                                            const __half* kv, const __half* V, const float* q_s,
                                            float* p_s) {
    constexpr int TB = 32 / G;
    const int lane = threadIdx.x & 31;
    const int tl = lane / G, sg = lane % G;
    for (int t0 = 0; t0 < ntok; t0 += TB) {
        uint2 vs[TB];
#pragma unroll
        for (int tt = 0; tt < TB; ++tt) {
            vs[tt] = make_uint2(0, 0);
            if (t0 + tt < ntok)
                vs[tt] = *reinterpret_cast<const uint2*>(V + static_cast<int64_t>(t0 + tt) * kHeadDim + lane * 4);
        }
        float part[G];
#pragma unroll
        for (int g = 0; g < G; ++g) part[g] = 0.f;
        const int t = t0 + tl;
        if (t < ntok) {
            const uint8_t* cr = ci + static_cast<int64_t>(t) * c;
            const __half* kr = kv + static_cast<int64_t>(t) * c;
            for (int x = sg; x < c; x += G) {
                const int ch = cr[x];
                const float kvf = __half2float(kr[x]);
#pragma unroll
                for (int g = 0; g < G; ++g) part[g] = fmaf(q_s[ch * G + g], kvf, part[g]);
            }
        }
        const float x = transpose_reduce_group<G>(part);
        const bool valid = (t0 + lane / G) < ntok;
        softmax_step<G>(st, x, valid, vs, p_s);
    }
}

struct DecodeArgs {
    int Hkv, Hq, S, r, c;
    float c2;
    DenseView dv;
    const uint8_t* arena;
    int64_t arena_stride;
    const uint64_t* desc;
    int32_t max_segs;
    const int32_t* n_segs;
    const int64_t* used_bytes;
    const int32_t* comp_end;
    const int32_t* seq_len;
    const __half* q;
    __half* out;
    int nsplit;
    float* part;
    uint32_t* ticket;
    uint32_t* status;
};

constexpr int64_t kTailBytes = 2 * kHeadDim * 2;   // K + V row of one dense token

template <int G>
__global__ void __launch_bounds__(kDecThreads) decode_kernel(const __grid_constant__ DecodeArgs A) {
    constexpr int TB = 32 / G;                     // tokens per warp step
    const int sp = blockIdx.x, u = blockIdx.y;
    const int b = u / A.Hkv, h = u % A.Hkv;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    __shared__ __align__(16) float q_s[kHeadDim * G];
    __shared__ float p_s[kDecWarps][32];
    __shared__ float wm[kDecWarps][G], wl[kDecWarps][G];
    __shared__ __align__(16) float wo[kDecWarps][G][kHeadDim];
    __shared__ long long hdr[4];       // lo, hi, U, ce | ntail
    __shared__ int cnt[2];
    __shared__ int is_last;
    __shared__ float sc[64][G];

    // ---- this CTA's share [lo, hi) of the unit's bytes: packed arena, then
    // the dense tail at 512 bytes per token
    if (tid == 0) {
        int T = A.seq_len[b];
        int ce = A.comp_end[b];
        const int64_t U = A.used_bytes[u];
        const int cap = A.dv.block_table ? A.dv.max_blocks * A.dv.block_size : A.dv.capacity;
        if (T < 0 || T > cap || ce < 0 || ce > T) {
            set_status(A.status, KV2D_DEV_SEQ_RANGE);
            T = max(0, min(T, cap));
            ce = max(0, min(ce, T));
        }
        const int64_t Wt = U + static_cast<int64_t>(T - ce) * kTailBytes;
        hdr[0] = Wt * sp / A.nsplit;
        hdr[1] = Wt * (sp + 1) / A.nsplit;
        hdr[2] = U;
        hdr[3] = (static_cast<long long>(ce) << 32) | static_cast<unsigned>(T - ce);
        cnt[0] = 0;
        cnt[1] = 0;
    }
    for (int i = tid; i < G * kHeadDim; i += kDecThreads) {
        const int g = i / kHeadDim, x = i % kHeadDim;
        q_s[x * G + g] =
            __half2float(A.q[(static_cast<int64_t>(b) * A.Hq + h * G + g) * kHeadDim + x]) * A.c2;
    }
    __syncthreads();
    const int64_t lo = hdr[0], hi = hdr[1], U = hdr[2];
    const int ce = static_cast<int>(hdr[3] >> 32), ntail = static_cast<int>(hdr[3] & 0xffffffff);
    const int nsg = A.n_segs[u];
    const uint64_t* D = A.desc + static_cast<int64_t>(u) * A.max_segs;
    {
        // segments whose first byte lies below lo / below hi (offsets ascend)
        int c_lo = 0, c_hi = 0;
        for (int j = tid; j < nsg; j += kDecThreads) {
            const int64_t off = static_cast<int64_t>(D[j] & 0xffffffffull) * 16;
            c_lo += off < lo;
            c_hi += off < hi;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            c_lo += __shfl_xor_sync(0xffffffffu, c_lo, o);
            c_hi += __shfl_xor_sync(0xffffffffu, c_hi, o);
        }
        if (lane == 0) {
            atomicAdd(&cnt[0], c_lo);
            atomicAdd(&cnt[1], c_hi);
        }
    }
    __syncthreads();
    const int j_lo = cnt[0], j_hi = cnt[1];
    auto tail_at_or_after = [&](int64_t x) -> int {
        if (x <= U) return 0;
        const int64_t i = (x - U + kTailBytes - 1) / kTailBytes;
        return static_cast<int>(i < ntail ? i : static_cast<int64_t>(ntail));
    };
    const int t_lo = ce + tail_at_or_after(lo), t_hi = ce + tail_at_or_after(hi);

    WarpState<G> st;
#pragma unroll
    for (int g = 0; g < G; ++g) {
        st.m[g] = kNegInfF;
#pragma unroll
        for (int e = 0; e < 4; ++e) st.o[g][e] = 0.f;
    }
    st.lp = 0.f;
    float qr[G][4];
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
        for (int e = 0; e < 4; ++e) qr[g][e] = q_s[(lane * 4 + e) * G + g];

    // ---- work items: (segment, block of TB tokens) in order, then tail blocks;
    // item i goes to warp i % 8.  A segment has ceil(ntok / TB) blocks.
    const uint8_t* ubase = A.arena + static_cast<int64_t>(u) * A.arena_stride;
    float* ps = p_s[warp];
    const int nb_full = (A.S + TB - 1) / TB, nb_tok = (A.r + TB - 1) / TB;
    int seg = j_lo, blk = 0, item = 0;
    // walk segments; each warp takes its own items
    while (seg < j_hi) {
        const uint64_t d = D[seg];
        const int sty = static_cast<int>((d >> 32) & 255u);
        const bool tok = (sty == KV2D_TOK || sty == KV2D_BOTH);
        const int nblk = tok ? nb_tok : nb_full;
        // first block of this segment owned by this warp
        int first = (warp - item) % kDecWarps;
        if (first < 0) first += kDecWarps;
        if (first < nblk) {
            const int ntok = tok ? A.r : A.S;
            const uint8_t* p0 = ubase + static_cast<int64_t>(d & 0xffffffffull) * 16 + (tok ? pad16(A.r) : 0);
            for (blk = first; blk < nblk; blk += kDecWarps) {
                const int t0 = blk * TB;
                const int n = min(TB, ntok - t0);
                if (sty == KV2D_FULL || sty == KV2D_TOK) {
                    const __half* K = reinterpret_cast<const __half*>(p0) + static_cast<int64_t>(t0) * kHeadDim;
                    const __half* V = reinterpret_cast<const __half*>(p0) + static_cast<int64_t>(ntok + t0) * kHeadDim;
                    dense_rows<G>(
                        st, n, [&](int i) { return K + static_cast<int64_t>(i) * kHeadDim; },
                        [&](int i) { return V + static_cast<int64_t>(i) * kHeadDim; }, qr, ps);
                } else {
                    const uint8_t* ci = p0;
                    const __half* kv = reinterpret_cast<const __half*>(p0 + pad16(static_cast<int64_t>(ntok) * A.c));
                    const __half* V = reinterpret_cast<const __half*>(
                        reinterpret_cast<const uint8_t*>(kv) + pad16(static_cast<int64_t>(ntok) * A.c * 2));
                    sparse_rows<G>(st, n, A.c, ci + static_cast<int64_t>(t0) * A.c,
                                   kv + static_cast<int64_t>(t0) * A.c,
                                   V + static_cast<int64_t>(t0) * kHeadDim, q_s, ps);
                }
            }
        }
        item += nblk;
        ++seg;
    }
    {
        const int ntb = (t_hi - t_lo + TB - 1) / TB;
        int first = (warp - item) % kDecWarps;
        if (first < 0) first += kDecWarps;
        uint32_t* status = A.status;
        const DenseView& dv = A.dv;
        for (int tb = first; tb < ntb; tb += kDecWarps) {
            const int t0 = t_lo + tb * TB;
            const int n = min(TB, t_hi - t0);
            dense_rows<G>(
                st, n, [&](int i) { return dense_row(dv, dv.k, b, h, t0 + i, status); },
                [&](int i) { return dense_row(dv, dv.v, b, h, t0 + i, status); }, qr, ps);
        }
    }

    // ---- warp partials -> shared memory
    float l = st.lp;
#pragma unroll
    for (int s = G; s < 32; s <<= 1) l += __shfl_xor_sync(0xffffffffu, l, s);
    if (lane < G) {
        float mg = kNegInfF;
#pragma unroll
        for (int g = 0; g < G; ++g)
            if (g == lane) mg = st.m[g];
        wm[warp][lane] = mg;
        wl[warp][lane] = l;
    }
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
        for (int e = 0; e < 4; ++e) wo[warp][g][lane * 4 + e] = st.o[g][e];
    __syncthreads();

    // ---- CTA partial: part[u][sp][g] = {M, L, O[d]}
    constexpr int kRec = kHeadDim + 2;
    float* myp = A.part + (static_cast<int64_t>(u) * A.nsplit + sp) * G * kRec;
    for (int i = tid; i < G * kHeadDim; i += kDecThreads) {
        const int g = i / kHeadDim, x = i % kHeadDim;
        float M = kNegInfF;
#pragma unroll
        for (int w = 0; w < kDecWarps; ++w) M = fmaxf(M, wm[w][g]);
        float O = 0.f, L = 0.f;
        if (M != kNegInfF) {
#pragma unroll
            for (int w = 0; w < kDecWarps; ++w) {
                if (wm[w][g] == kNegInfF) continue;
                const float scl = fast_exp2(wm[w][g] - M);
                O = fmaf(wo[w][g][x], scl, O);
                L = fmaf(wl[w][g], scl, L);
            }
        }
        myp[g * kRec + 2 + x] = O;
        if (x == 0) {
            myp[g * kRec] = M;
            myp[g * kRec + 1] = L;
        }
    }
    __threadfence();
    __syncthreads();
    if (tid == 0) is_last = (atomicAdd(&A.ticket[u], 1u) == static_cast<uint32_t>(A.nsplit - 1));
    __syncthreads();
    if (!is_last) return;
    __threadfence();

    // ---- last CTA of the unit: merge the splits in order
    const float* up = A.part + static_cast<int64_t>(u) * A.nsplit * G * kRec;
    for (int i = tid; i < A.nsplit * G; i += kDecThreads) sc[i / G][i % G] = __ldcg(up + i * kRec);
    __syncthreads();
    if (tid < G) {
        float M = kNegInfF;
        for (int s2 = 0; s2 < A.nsplit; ++s2) M = fmaxf(M, sc[s2][tid]);
        float L = 0.f;
        for (int s2 = 0; s2 < A.nsplit; ++s2) {
            const float ms = sc[s2][tid];
            const float scl = (ms == kNegInfF) ? 0.f : fast_exp2(ms - M);
            sc[s2][tid] = scl;
            L = fmaf(__ldcg(up + (s2 * G + tid) * kRec + 1), scl, L);
        }
        wl[0][tid] = L;
    }
    __syncthreads();
    for (int i = tid; i < G * kHeadDim; i += kDecThreads) {
        const int g = i / kHeadDim, x = i % kHeadDim;
        float O = 0.f;
        for (int s2 = 0; s2 < A.nsplit; ++s2) {
            const float scl = sc[s2][g];
            if (scl != 0.f) O = fmaf(__ldcg(up + (s2 * G + g) * kRec + 2 + x), scl, O);
        }
        const float L = wl[0][g];
        const float res = (L > 0.f) ? O / L : 0.f;
        A.out[(static_cast<int64_t>(b) * A.Hq + h * G + g) * kHeadDim + x] = __float2half_rn(res);
    }
    if (tid == 0) A.ticket[u] = 0;
}

}  // namespace

int decode_split_count(int units, int64_t max_seq_len, int num_sms) {
    // two CTAs per SM, one wave
    int ns = (2 * num_sms) / units;
    const int by_len = static_cast<int>((max_seq_len + 255) / 256);
    ns = min(ns, max(1, by_len));
    return max(1, min(ns, 64));
}

cudaError_t launch_append(const AppendLaunch& L, cudaStream_t stream) {
    prof_begin(stream, kProfAppend);
    append_kernel<<<L.batch, 256, 0, stream>>>(L);
    prof_end(stream, kProfAppend);
    return cudaGetLastError();
}

cudaError_t launch_decode(const DecodeLaunch& L, cudaStream_t stream) {
    DecodeArgs a;
    a.Hkv = L.shp.Hkv;
    a.Hq = L.shp.Hq;
    a.S = L.shp.S;
    a.r = L.shp.r;
    a.c = L.shp.c;
    a.c2 = L.scale_log2;
    a.dv = L.dv;
    a.arena = L.arena;
    a.arena_stride = L.arena_stride;
    a.desc = L.desc;
    a.max_segs = L.max_segs;
    a.n_segs = L.n_segs;
    a.used_bytes = L.used_bytes;
    a.comp_end = L.comp_end;
    a.seq_len = L.seq_len;
    a.q = L.q;
    a.out = L.out;
    a.nsplit = L.nsplit;
    a.part = L.part;
    a.ticket = L.ticket;
    a.status = L.status;
    const int units = L.batch * L.shp.Hkv;
    cudaError_t e = cudaMemsetAsync(L.ticket, 0, sizeof(uint32_t) * units, stream);
    if (e != cudaSuccess) return e;
    dim3 grid(L.nsplit, units);
    prof_begin(stream, kProfDecode);
    switch (L.shp.G) {
    case 2: decode_kernel<2><<<grid, kDecThreads, 0, stream>>>(a); break;
    case 4: decode_kernel<4><<<grid, kDecThreads, 0, stream>>>(a); break;
    case 8: decode_kernel<8><<<grid, kDecThreads, 0, stream>>>(a); break;
    default: return cudaErrorInvalidValue;
    }
    prof_end(stream, kProfDecode);
    return cudaGetLastError();
}

}  // namespace kv2d
