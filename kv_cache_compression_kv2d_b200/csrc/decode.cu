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
//   - each warp takes 16-token blocks and runs q.k and p.v on the tensor
//     cores (mma.sync m16n8k16, fp16 in, fp32 accumulate; the G heads are
//     the rows of the 16-row tile); key and value fragments come straight
//     from global memory with 16-byte loads; CH / BOTH keys are first
//     scattered into a dense 16 x 128 tile in shared memory;
//   - scores meet an online softmax per head in the log2 domain; warps, then
//     CTAs, merge their (max, sum, output) partials in a fixed order, the
//     last CTA of a unit (atomic ticket) writing the fp16 output.
#include "kernels.h"

namespace kv2d {

namespace {

constexpr int kDecWarps = 4;
constexpr int kDecThreads = kDecWarps * 32;
constexpr float kNegInfF = -__builtin_huge_valf();

// ------------------------------------------------------------------ append

__global__ void append_kernel(const __grid_constant__ AppendLaunch A) {
    pdl_wait();
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
constexpr int kDescCache = 1024;                   // descriptors staged per CTA

// ------------------------------------------------------ tensor-core decode
//
// Per warp, blocks of 16 tokens go through two m16n8k16 products (fp16 in,
// fp32 accumulate):
//   S[16 x 16] = Q[16 x 128] K^T   (rows = the G query heads, zero-padded)
//   O[16 x 128] += P[16 x 16] V    (P = softmax numerators in fp16)
// Lane (g = lane / 4, t = lane % 4).  The q.k contraction runs over d in a
// fixed permuted order: mma k-index 2t+e of step ks <-> d = 32t + 4ks + e
// and 2t+8+e <-> d = 32t + 4ks + 2 + e, so a lane's key data for all eight
// steps is the contiguous window [32t, 32t + 32) of a row.  In p.v the
// output column n of n-tile j stands for d = 16n + j, so a lane's value data
// is the window [16g, 16g + 16) of rows 2t, 2t+1, 2t+8, 2t+9.

__device__ __forceinline__ void mma16816(float& d0, float& d1, uint32_t a0, uint32_t a2, uint32_t b0,
                                         uint32_t b1) {
    float x2, x3;   // rows 8..15 of the tile: never used
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
        "{%8, %9}, {%10, %11, %12, %13};"
        : "=f"(d0), "=f"(d1), "=f"(x2), "=f"(x3)
        : "r"(a0), "r"(0u), "r"(a2), "r"(0u), "r"(b0), "r"(b1), "f"(d0), "f"(d1), "f"(0.f),
          "f"(0.f));
    (void)x2;
    (void)x3;
}

struct MmaState {
    float m;          // running max of this lane's head row (log2 domain)
    float lp;         // this lane's share of the row's softmax sum
    float o[16][2];   // O[g][d = 32t + 16e + j] at o[j][e]
};

__device__ __forceinline__ uint4 ld_nc16(const void* p) {
    return *reinterpret_cast<const uint4*>(p);
}

// One 16-token block.  kw[nt][i]: this lane's key window of row nt*8 + g
// (chunk i of [32t, 32t+32)); vw[k][i]: value window of row {2t, 2t+1,
// 2t+8, 2t+9}[k], chunk i of [16g, 16g+16).  ntok valid tokens.
__device__ __forceinline__ void mma_block(MmaState& st, const uint32_t (&qa)[8][2], const uint4 (&kw)[2][4],
                                          const uint4 (&vw)[4][2], int ntok, float c2) {
    const int lane = threadIdx.x & 31;
    const int t = lane & 3;
    float sacc[2][2];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
        sacc[nt][0] = 0.f;
        sacc[nt][1] = 0.f;
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
            const uint4& w = kw[nt][ks >> 1];
            const uint32_t b0 = (ks & 1) ? w.z : w.x;
            const uint32_t b1 = (ks & 1) ? w.w : w.y;
            mma16816(sacc[nt][0], sacc[nt][1], qa[ks][0], qa[ks][1], b0, b1);
        }
    }
    // scores of tokens nt*8 + 2t + e, online softmax over the head row
    float x[4];
    bool ok[4];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int tok = nt * 8 + 2 * t + e;
            ok[nt * 2 + e] = tok < ntok;
            x[nt * 2 + e] = ok[nt * 2 + e] ? sacc[nt][e] * c2 : kNegInfF;
        }
    float bm = fmaxf(fmaxf(x[0], x[1]), fmaxf(x[2], x[3]));
    bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 1));
    bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 2));
    const float mn = fmaxf(st.m, bm);
    const float alpha = (st.m == mn) ? 1.f : fast_exp2(st.m - mn);   // st.m = -inf -> 0
    st.m = mn;
    float p[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) p[i] = ok[i] ? fast_exp2(x[i] - mn) : 0.f;
    st.lp = st.lp * alpha + ((p[0] + p[1]) + (p[2] + p[3]));
    if (__any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            st.o[j][0] *= alpha;
            st.o[j][1] *= alpha;
        }
    }
    const __half2 pa = __floats2half2_rn(p[0], p[1]);
    const __half2 pb = __floats2half2_rn(p[2], p[3]);
    const uint32_t a0 = *reinterpret_cast<const uint32_t*>(&pa);
    const uint32_t a2 = *reinterpret_cast<const uint32_t*>(&pb);
#pragma unroll
    for (int j = 0; j < 16; ++j) {
        // element j of the windows: chunk j / 8, 32-bit word (j % 8) / 2
        const int ci = j >> 3, wi = (j & 7) >> 1;
        const uint32_t sel = (j & 1) ? 0x7632u : 0x5410u;
        auto word = [&](const uint4& q4) {
            return wi == 0 ? q4.x : wi == 1 ? q4.y : wi == 2 ? q4.z : q4.w;
        };
        const uint32_t b0 = __byte_perm(word(vw[0][ci]), word(vw[1][ci]), sel);
        const uint32_t b1 = __byte_perm(word(vw[2][ci]), word(vw[3][ci]), sel);
        mma16816(st.o[j][0], st.o[j][1], a0, a2, b0, b1);
    }
}

// Position of channel chunk c (16 bytes) of row r in a warp's 16 x 128 key
// tile, XOR-swizzled so that the fragment loads of 8 lanes hit 8 different
// bank groups.
__device__ __forceinline__ int tile_chunk(int r, int c) {
    return c ^ (((c >> 3) & 1) << 1) ^ (r & 1);
}

template <int G>
__global__ void __launch_bounds__(kDecThreads) decode_kernel(const __grid_constant__ DecodeArgs A) {
    const int sp = blockIdx.x, u = blockIdx.y;
    const int b = u / A.Hkv, h = u % A.Hkv;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, t = lane & 3;
    __shared__ float wm[kDecWarps][G], wl[kDecWarps][G];
    // per-warp 16 x 128 key tiles; reused for the warp partials at the end
    __shared__ __align__(16) uint8_t ktile[kDecWarps][16 * 256];
    static_assert(sizeof(float) * kDecWarps * G * kHeadDim <= sizeof(ktile), "partials fit");
    float (*wo)[G][kHeadDim] = reinterpret_cast<float (*)[G][kHeadDim]>(&ktile[0][0]);
    __shared__ long long hdr[4];
    __shared__ int cnt[2];
    __shared__ int is_last;
    __shared__ float sc[64][G];
    __shared__ uint64_t dsm[kDescCache];

    pdl_wait();
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
    // q fragments (rows g < G): halves [32t, 32t + 32) of head g, step ks at 4ks
    uint32_t qa[8][2];
    {
        uint4 qw[4] = {make_uint4(0, 0, 0, 0), make_uint4(0, 0, 0, 0), make_uint4(0, 0, 0, 0),
                       make_uint4(0, 0, 0, 0)};
        if (g < G) {
            const __half* qrow = A.q + (static_cast<int64_t>(b) * A.Hq + h * G + g) * kHeadDim + 32 * t;
#pragma unroll
            for (int i = 0; i < 4; ++i) qw[i] = ld_nc16(qrow + 8 * i);
        }
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
            const uint4& w = qw[ks >> 1];
            qa[ks][0] = (ks & 1) ? w.z : w.x;
            qa[ks][1] = (ks & 1) ? w.w : w.y;
        }
    }
    __syncthreads();
    const int64_t lo = hdr[0], hi = hdr[1], U = hdr[2];
    const int ce = static_cast<int>(hdr[3] >> 32), ntail = static_cast<int>(hdr[3] & 0xffffffff);
    const int nsg = A.n_segs[u];
    const uint64_t* D = A.desc + static_cast<int64_t>(u) * A.max_segs;
    {
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
    const bool cached = (j_hi - j_lo) <= kDescCache;
    if (cached)
        for (int j = j_lo + tid; j < j_hi; j += kDecThreads) dsm[j - j_lo] = D[j];
    __syncthreads();
    auto tail_at_or_after = [&](int64_t x) -> int {
        if (x <= U) return 0;
        const int64_t i = (x - U + kTailBytes - 1) / kTailBytes;
        return static_cast<int>(i < ntail ? i : static_cast<int64_t>(ntail));
    };
    const int t_lo = ce + tail_at_or_after(lo), t_hi = ce + tail_at_or_after(hi);

    MmaState st;
    st.m = kNegInfF;
    st.lp = 0.f;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
        st.o[j][0] = 0.f;
        st.o[j][1] = 0.f;
    }
    const float c2 = A.c2;
    const uint8_t* ubase = A.arena + static_cast<int64_t>(u) * A.arena_stride;
    uint8_t* tile = ktile[warp];
    const uint4 zero4 = make_uint4(0, 0, 0, 0);

    // dense rows: Kr(i) / Vr(i) point at row i of the block (nullptr -> zeros)
    auto dense_block = [&](auto Kr, auto Vr, int n) {
        uint4 kw[2][4], vw[4][2];
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            const int r = nt * 8 + g;
            const __half* kp = (r < n) ? Kr(r) : nullptr;
#pragma unroll
            for (int i = 0; i < 4; ++i) kw[nt][i] = kp ? ld_nc16(kp + 32 * t + 8 * i) : zero4;
        }
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const int r = 2 * t + (k & 1) + 8 * (k >> 1);
            const __half* vp = (r < n) ? Vr(r) : nullptr;
#pragma unroll
            for (int i = 0; i < 2; ++i) vw[k][i] = vp ? ld_nc16(vp + 16 * g + 8 * i) : zero4;
        }
        mma_block(st, qa, kw, vw, n, c2);
    };

    // ---- work items: (segment, block of 16 tokens), then tail blocks;
    // item i goes to warp i % kDecWarps
    int seg = j_lo, item = 0;
    while (seg < j_hi) {
        const uint64_t d = cached ? dsm[seg - j_lo] : D[seg];
        const int sty = static_cast<int>((d >> 32) & 255u);
        const bool tok = (sty == KV2D_TOK || sty == KV2D_BOTH);
        const int ntok = tok ? A.r : A.S;
        const int nblk = (ntok + 15) >> 4;
        int first = (warp - item) % kDecWarps;
        if (first < 0) first += kDecWarps;
        if (first < nblk) {
            const uint8_t* p0 = ubase + static_cast<int64_t>(d & 0xffffffffull) * 16 + (tok ? pad16(A.r) : 0);
            for (int blk = first; blk < nblk; blk += kDecWarps) {
                const int t0 = blk * 16;
                const int n = min(16, ntok - t0);
                if (sty == KV2D_FULL || sty == KV2D_TOK) {
                    const __half* K = reinterpret_cast<const __half*>(p0) + static_cast<int64_t>(t0) * kHeadDim;
                    const __half* V = reinterpret_cast<const __half*>(p0) + static_cast<int64_t>(ntok + t0) * kHeadDim;
                    dense_block([&](int i) { return K + static_cast<int64_t>(i) * kHeadDim; },
                                [&](int i) { return V + static_cast<int64_t>(i) * kHeadDim; }, n);
                } else {
                    const int c = A.c;
                    const uint8_t* ci = p0 + static_cast<int64_t>(t0) * c;
                    const __half* kv = reinterpret_cast<const __half*>(p0 + pad16(static_cast<int64_t>(ntok) * c)) +
                                       static_cast<int64_t>(t0) * c;
                    const __half* V = reinterpret_cast<const __half*>(
                                          p0 + pad16(static_cast<int64_t>(ntok) * c) +
                                          pad16(static_cast<int64_t>(ntok) * c * 2)) +
                                      static_cast<int64_t>(t0) * kHeadDim;
                    // dense 16 x 128 key tile in shared memory: zero, scatter
#pragma unroll
                    for (int i = 0; i < 8; ++i)
                        reinterpret_cast<uint4*>(tile)[lane + 32 * i] = zero4;
                    __syncwarp();
                    // 16 (index, value) pairs per lane from three 16-byte loads
                    // (the pair arrays start 16-byte aligned; a read past the
                    // last pair stays inside the segment's later sections)
                    const int np = n * c;
                    for (int e0 = lane * 16; e0 < np; e0 += 32 * 16) {
                        const uint4 iw = ld_nc16(ci + e0);
                        const uint4 va = ld_nc16(kv + e0), vb = ld_nc16(kv + e0 + 8);
                        const uint32_t iws[4] = {iw.x, iw.y, iw.z, iw.w};
                        const uint32_t vws[8] = {va.x, va.y, va.z, va.w, vb.x, vb.y, vb.z, vb.w};
                        int r = e0 / c, col = e0 - r * c;
#pragma unroll
                        for (int k = 0; k < 16; ++k) {
                            if (e0 + k < np) {
                                const int ch = (iws[k >> 2] >> (8 * (k & 3))) & 0xff;
                                const uint16_t hv = static_cast<uint16_t>(vws[k >> 1] >> (16 * (k & 1)));
                                *reinterpret_cast<uint16_t*>(tile + r * 256 + tile_chunk(r, ch >> 3) * 16 + (ch & 7) * 2) = hv;
                            }
                            if (++col == c) {
                                col = 0;
                                ++r;
                            }
                        }
                    }
                    __syncwarp();
                    uint4 kw[2][4], vw[4][2];
#pragma unroll
                    for (int nt = 0; nt < 2; ++nt) {
                        const int r = nt * 8 + g;
#pragma unroll
                        for (int i = 0; i < 4; ++i)
                            kw[nt][i] = *reinterpret_cast<const uint4*>(tile + r * 256 + tile_chunk(r, 4 * t + i) * 16);
                    }
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const int r = 2 * t + (k & 1) + 8 * (k >> 1);
#pragma unroll
                        for (int i = 0; i < 2; ++i)
                            vw[k][i] = (r < n) ? ld_nc16(V + static_cast<int64_t>(r) * kHeadDim + 16 * g + 8 * i) : zero4;
                    }
                    __syncwarp();
                    mma_block(st, qa, kw, vw, n, c2);
                }
            }
        }
        item += nblk;
        ++seg;
    }
    {
        const int ntb = (t_hi - t_lo + 15) >> 4;
        int first = (warp - item) % kDecWarps;
        if (first < 0) first += kDecWarps;
        uint32_t* status = A.status;
        const DenseView& dv = A.dv;
        for (int tb = first; tb < ntb; tb += kDecWarps) {
            const int t0 = t_lo + tb * 16;
            const int n = min(16, t_hi - t0);
            dense_block([&](int i) -> const __half* { return dense_row(dv, dv.k, b, h, t0 + i, status); },
                        [&](int i) -> const __half* { return dense_row(dv, dv.v, b, h, t0 + i, status); }, n);
        }
    }

    // ---- warp partials -> shared memory (lanes with g < G hold real rows)
    __syncthreads();   // every warp is done with its key tile
    float l = st.lp;
    l += __shfl_xor_sync(0xffffffffu, l, 1);
    l += __shfl_xor_sync(0xffffffffu, l, 2);
    if (g < G) {
        if (t == 0) {
            wm[warp][g] = st.m;
            wl[warp][g] = l;
        }
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            wo[warp][g][32 * t + j] = st.o[j][0];
            wo[warp][g][32 * t + 16 + j] = st.o[j][1];
        }
    }
    __syncthreads();

    // ---- CTA partial: part[u][sp][g] = {M, L, 0, 0, O[d]} (16-byte aligned O)
    constexpr int kRec = kHeadDim + 4;
    float* myp = A.part + (static_cast<int64_t>(u) * A.nsplit + sp) * G * kRec;
    for (int i = tid; i < G * kHeadDim; i += kDecThreads) {
        const int gg = i / kHeadDim, x = i % kHeadDim;
        float M = kNegInfF;
#pragma unroll
        for (int w = 0; w < kDecWarps; ++w) M = fmaxf(M, wm[w][gg]);
        float O = 0.f, L = 0.f;
        if (M != kNegInfF) {
#pragma unroll
            for (int w = 0; w < kDecWarps; ++w) {
                if (wm[w][gg] == kNegInfF) continue;
                const float scl = fast_exp2(wm[w][gg] - M);
                O = fmaf(wo[w][gg][x], scl, O);
                L = fmaf(wl[w][gg], scl, L);
            }
        }
        myp[gg * kRec + 4 + x] = O;
        if (x == 0) {
            myp[gg * kRec] = M;
            myp[gg * kRec + 1] = L;
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
        for (int s2 = 0; s2 < A.nsplit; ++s2) {
            const float ms = sc[s2][tid];
            sc[s2][tid] = (ms == kNegInfF) ? 0.f : fast_exp2(ms - M);
        }
    }
    __syncthreads();
    if (tid < G) {
        float L = 0.f;
        for (int s2 = 0; s2 < A.nsplit; ++s2)
            L = fmaf(__ldcg(up + (s2 * G + tid) * kRec + 1), sc[s2][tid], L);
        wl[0][tid] = L;
    }
    // a thread merges 4 consecutive channels of one head; up to 16 splits'
    // 16-byte records are loaded before they are summed in split order
    for (int i = tid; i < G * (kHeadDim / 4); i += kDecThreads) {
        const int gg = i / (kHeadDim / 4), x4 = (i % (kHeadDim / 4)) * 4;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int s0 = 0; s0 < A.nsplit; s0 += 16) {
            float4 v16[16];
#pragma unroll
            for (int k = 0; k < 16; ++k)
                v16[k] = (s0 + k < A.nsplit)
                             ? __ldcg(reinterpret_cast<const float4*>(up + ((s0 + k) * G + gg) * kRec + 4 + x4))
                             : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int k = 0; k < 16; ++k) {
                if (s0 + k >= A.nsplit) break;
                const float scl = sc[s0 + k][gg];
                acc.x = fmaf(v16[k].x, scl, acc.x);
                acc.y = fmaf(v16[k].y, scl, acc.y);
                acc.z = fmaf(v16[k].z, scl, acc.z);
                acc.w = fmaf(v16[k].w, scl, acc.w);
            }
        }
        reinterpret_cast<float4*>(ktile)[(gg * kHeadDim + x4) / 4] = acc;
    }
    __syncthreads();
    for (int i = tid; i < G * kHeadDim; i += kDecThreads) {
        const int gg = i / kHeadDim, x = i % kHeadDim;
        const float L = wl[0][gg];
        const float O = reinterpret_cast<const float*>(ktile)[gg * kHeadDim + x];
        const float res = (L > 0.f) ? O / L : 0.f;
        A.out[(static_cast<int64_t>(b) * A.Hq + h * G + gg) * kHeadDim + x] = __float2half_rn(res);
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
    cudaError_t e = launch_k(append_kernel, dim3(L.batch), dim3(256), 0, stream, L);
    if (e != cudaSuccess) return e;
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
    cudaError_t e = cudaSuccess;
    dim3 grid(L.nsplit, units);
    prof_begin(stream, kProfDecode);
    switch (L.shp.G) {
    case 2: e = launch_k(decode_kernel<2>, grid, dim3(kDecThreads), 0, stream, a); break;
    case 4: e = launch_k(decode_kernel<4>, grid, dim3(kDecThreads), 0, stream, a); break;
    case 8: e = launch_k(decode_kernel<8>, grid, dim3(kDecThreads), 0, stream, a); break;
    default: return cudaErrorInvalidValue;
    }
    if (e != cudaSuccess) return e;
    prof_end(stream, kProfDecode);
    return cudaGetLastError();
}

}  // namespace kv2d
