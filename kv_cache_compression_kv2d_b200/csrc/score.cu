// score.cu -- per-unit scoring of the KV cache (sm_100a).
//
// MosaicKV ("MosaicKV: Serving Long-Context LLM with Dynamic Two-D KV Cache
// Compression", Core claim and Fig. 6 Stage-1) identifies important elements
// of every KV vector; Kara ("KARA: Efficient Reasoning LLM Serving via
// Sliding-Window KV Cache Compression", "What carries the argument") scores
// keys by the attention that all queries of a recent window give them.
// The kernels here compute, per unit (sequence b, KV head h):
//   pass 1    : lse of every window row over the causal region, from a
//               tcgen05 product Q_w K^T (M = 128 window rows, N = 128 keys),
//               split over key ranges -> per-split (max, sum) partials; the
//               first split of each row tile also sums |q_d| over its rows
//   pass 2    : merges the lse partials in split order, then
//               s_t = sum_rows exp(l - lse) from the transposed product
//               K Q_w^T (M = 128 keys, N = window rows) so that each TMEM lane
//               owns one key and sums over queries in-thread; the two
//               epilogue warpgroups take alternate tiles, each accumulator
//               split in two column halves with their own barriers
//   chan      : a_d = (sum of the |q_d| tile sums) / (G*W); per key: top-c
//               channels of |k_d| a_d and g_t in fp64 (a
//               packed 16-bit SIMD selection network for c <= 32, a full
//               32-bit register sort otherwise)
// Both products take their operands from shared memory written by TMA with
// the 128-byte swizzle; the fp32 accumulators live in tensor memory.
#include "kernels.h"

namespace kv2d {

namespace {

constexpr int kPassThreads = 320;    // 8 epilogue warps, 1 TMA warp, 1 MMA warp
constexpr int kStage = 128 * 256;    // one K tile: 128 keys x 128 fp16
constexpr int kP1Stages = 2;   // ~99 KB of shared memory: two CTAs per SM
// Part of the exponentials of a fully visible tile run on the FMA pipe
// (exp2_fma) instead of MUFU.  Pass 1: every n-th (0: none).  Pass 2, which
// sums 2^x of G*W columns per key and leans on MUFU harder than pass 1 (that
// also tracks row maxima): this many pairs of each 8 columns (exp2_fma2).
#ifndef KV2D_P1_FMA_EVERY
#define KV2D_P1_FMA_EVERY 8
#endif
#ifndef KV2D_P2_POLY_PAIRS
#define KV2D_P2_POLY_PAIRS 1
#endif
constexpr int kP1FmaEvery = KV2D_P1_FMA_EVERY;
constexpr int kP2PolyPairs = KV2D_P2_POLY_PAIRS;

template <int EVERY>
__device__ __forceinline__ float exp2_mixed(float x, int j) {
    if constexpr (EVERY > 0) {
        if (j % EVERY == EVERY - 1) return exp2_fma(x);
    }
    return fast_exp2(x);
}
constexpr uint32_t kNegInf = 0xff800000u;

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
    return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// Issues the TMA loads of one 128-key tile starting at token t0 into dst
// (two 16 KB halves of 64 channels; rows in token order).
__device__ __forceinline__ void load_key_tile(uint8_t* dst, const CUtensorMap* kmap,
                                              uint64_t* bar, const DenseView& dv, int paged,
                                              int b, int h, int t0, int T, uint32_t* status) {
    if (!paged) {
        tma_load_4d(dst, kmap, bar, 0, t0, h, b);
        tma_load_4d(dst + 16384, kmap, bar, 64, t0, h, b);
        return;
    }
    for (int j = 0; j < 8; ++j) {
        int t = t0 + 16 * j;
        int lb = t / dv.block_size;
        int phys = -1;
        if (lb < dv.max_blocks) phys = dv.block_table[static_cast<int64_t>(b) * dv.max_blocks + lb];
        if (phys < 0 || phys >= dv.num_blocks) {
            if (t < T) set_status(status, KV2D_DEV_BLOCK_TABLE);
            phys = 0;
        }
        int row = t % dv.block_size;
        tma_load_4d(dst + j * 2048, kmap, bar, 0, row, h, phys);
        tma_load_4d(dst + 16384 + j * 2048, kmap, bar, 64, row, h, phys);
    }
}

// --------------------------------------------------------------- pass 1

struct Pass1Args {
    SeqPlan plan;
    UnitShape shp;
    DenseView dv;
    int paged;
    int kps, nsplit;
    float2* part;
    float* apart;          // [units][mtiles][d]: sum of |q| over the tile's rows
    uint32_t* status;
};

__global__ void __launch_bounds__(kPassThreads, 1)
    score_pass1_kernel(const __grid_constant__ CUtensorMap qmap,
                       const __grid_constant__ CUtensorMap kmap, const __grid_constant__ Pass1Args A) {
    const int sp = blockIdx.x, mt = blockIdx.y, u = blockIdx.z;
    const int Hkv = A.shp.Hkv, W = A.shp.W, GW = A.shp.GW, GWpad = A.shp.GWpad;
    const int b = u / Hkv, h = u % Hkv;
    const int T = A.plan.T[b], r0 = A.plan.r0[b];
    const int k_lo = r0 + sp * A.kps;
    const int k_hi = min(T, k_lo + A.kps);
    const int nt = k_hi > k_lo ? (k_hi - k_lo + kKeyTile - 1) / kKeyTile : 0;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    if (nt == 0) {
        pdl_wait();
        if (tid < 128) {
            int rho = mt * 128 + tid;
            if (rho < GW)
                A.part[(static_cast<int64_t>(u) * GWpad + rho) * A.nsplit + sp] =
                    make_float2(__uint_as_float(kNegInf), 0.f);
        }
        return;
    }

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    uint8_t* q_s = smem;                                   // 32 KB
    uint8_t* k_s = smem + 32768;                           // stages
    uint64_t* full = reinterpret_cast<uint64_t*>(k_s + kP1Stages * kStage);
    uint64_t* empty = full + kP1Stages;
    uint64_t* tfull = empty + kP1Stages;
    uint64_t* tempty = tfull + 4;
    uint64_t* qbar = tempty + 4;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(qbar + 1);
    float* xm = reinterpret_cast<float*>(tmem_slot + 4);   // [256]
    float* xl = xm + 256;

    if (tid == 0) {
        for (int i = 0; i < kP1Stages; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], 1);
        }
        for (int i = 0; i < 4; ++i) {
            mbar_init(&tfull[i], 1);
            mbar_init(&tempty[i], 128);
        }
        mbar_init(qbar, 1);
        mbar_fence_init();
    }
    if (warp == 9) {
        tmem_alloc(tmem_slot, 256);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    pdl_wait();

    if (warp == 8) {
        if (lane == 0) {
            tma_prefetch_desc(&qmap);
            tma_prefetch_desc(&kmap);
            const int qrow0 = (b * A.shp.Hq + h * A.shp.G) * W + mt * 128;
            mbar_expect_tx(qbar, 32768);
            for (int hf = 0; hf < 2; ++hf)
                for (int rb = 0; rb < 2; ++rb)
                    tma_load_2d(q_s + hf * 16384 + rb * 8192, &qmap, qbar, hf * 64, qrow0 + rb * 64);
            for (int i = 0; i < nt; ++i) {
                const int s = i % kP1Stages;
                if (i >= kP1Stages && !mbar_wait(&empty[s], ((i / kP1Stages) - 1) & 1, A.status))
                    break;
                mbar_expect_tx(&full[s], kStage);
                load_key_tile(k_s + s * kStage, &kmap, &full[s], A.dv, A.paged, b, h,
                              k_lo + i * kKeyTile, T, A.status);
            }
        }
    } else if (warp == 9) {
        if (lane == 0) {
            // each warpgroup's accumulator is two 64-key halves with their
            // own barriers, so the MMA refills the first half while the
            // epilogue still reads the second
            constexpr uint32_t idesc = idesc_f16_f32(128, 64);
            const uint32_t qa = smem_u32(q_s);
            bool ok = mbar_wait(qbar, 0, A.status);
            for (int i = 0; ok && i < nt; ++i) {
                const int s = i % kP1Stages, buf = i & 1;
                if (!mbar_wait(&full[s], (i / kP1Stages) & 1, A.status)) break;
                const uint32_t ka = smem_u32(k_s + s * kStage);
                for (int hh = 0; hh < 2; ++hh) {
                    const int hb = 2 * buf + hh;
                    if (i >= 2 && !mbar_wait(&tempty[hb], ((i >> 1) - 1) & 1, A.status)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk) {
                        const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
                        umma_f16(tmem + hb * 64, sw128_kmajor_desc(qa + off),
                                 sw128_kmajor_desc(ka + hh * 8192 + off), idesc, kk > 0 ? 1u : 0u);
                    }
                    umma_commit(&tfull[hb]);
                }
                if (!ok) break;
                umma_commit(&empty[s]);
            }
        }
    } else {
        // epilogue: warps 0-3 take even tiles (TMEM columns 0..127), warps
        // 4-7 odd tiles (columns 128..255), each as two 64-column halves;
        // thread <-> window row.
        const int wg = warp >> 2, lg = warp & 3;
        const int row = lg * 32 + lane;
        const int rho = mt * 128 + row;
        const int pw = (rho < GW) ? (T - W + (rho % W)) : -1;   // last key the row sees
        const int lim = min(pw, k_hi - 1);
        const float c2 = A.shp.c2;
        float m = __uint_as_float(kNegInf), l = 0.f;
        for (int i = wg; i < nt; i += 2) {
            if (!mbar_wait(&tfull[2 * wg], (i >> 1) & 1, A.status)) break;
            tc_fence_after();
            const int t_base = k_lo + i * kKeyTile;
            const uint32_t taddr = tmem + (static_cast<uint32_t>(lg * 32) << 16) + wg * 128;
            const bool whole = (t_base + kKeyTile - 1 <= lim);
            // four 32-column chunks; chunk c+1's TMEM load is in flight while
            // chunk c is processed (online max / sum in the log2 domain)
            auto proc = [&](const uint32_t (&r)[32], int cc) {
                float mraw = __uint_as_float(kNegInf);
                if (whole) {
#pragma unroll
                    for (int j = 0; j < 32; ++j) mraw = fmaxf(mraw, __uint_as_float(r[j]));
                } else {
                    const int t0 = t_base + cc * 32;
#pragma unroll
                    for (int j = 0; j < 32; ++j)
                        if (t0 + j <= lim) mraw = fmaxf(mraw, __uint_as_float(r[j]));
                }
                if (mraw == __uint_as_float(kNegInf)) return;     // nothing visible here
                const float mx = mraw * c2;                       // c2 > 0: order kept
                if (mx > m) {
                    l = (l == 0.f) ? 0.f : l * fast_exp2(m - mx);
                    m = mx;
                }
                const float nm = -m;
                float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
                if (whole) {
                    // packed pairs: (a0, a1) and (a2, a3) accumulate columns
                    // 4q + {0, 1} and 4q + {2, 3}, each lane as the scalar
                    // multiply-add / add would
                    const float2 c2v = make_float2(c2, c2), nmv = make_float2(nm, nm);
                    float2 a01 = make_float2(0.f, 0.f), a23 = make_float2(0.f, 0.f);
#pragma unroll
                    for (int j = 0; j < 32; j += 4) {
                        const float2 x01 = f2_fma(make_float2(__uint_as_float(r[j]), __uint_as_float(r[j + 1])), c2v, nmv);
                        const float2 x23 =
                            f2_fma(make_float2(__uint_as_float(r[j + 2]), __uint_as_float(r[j + 3])), c2v, nmv);
                        a01 = f2_add(a01, make_float2(exp2_mixed<kP1FmaEvery>(x01.x, j),
                                                      exp2_mixed<kP1FmaEvery>(x01.y, j + 1)));
                        a23 = f2_add(a23, make_float2(exp2_mixed<kP1FmaEvery>(x23.x, j + 2),
                                                      exp2_mixed<kP1FmaEvery>(x23.y, j + 3)));
                    }
                    a0 = a01.x;
                    a1 = a01.y;
                    a2 = a23.x;
                    a3 = a23.y;
                } else {
                    const int t0 = t_base + cc * 32;
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        const float e = fast_exp2(fmaf(__uint_as_float(r[j]), c2, nm));
                        a0 += (t0 + j <= lim) ? e : 0.f;
                    }
                }
                l += (a0 + a1) + (a2 + a3);
            };
            // half buffer 2 wg holds chunks 0, 1 (columns wg * 128 + 0..63),
            // half buffer 2 wg + 1 chunks 2, 3
            uint32_t ra[32], rb[32];
            tmem_ld32(taddr, ra);
            tmem_ld_wait(ra);
            tmem_ld32(taddr + 32, rb);
            proc(ra, 0);
            tmem_ld_wait(rb);
            if (!mbar_wait(&tfull[2 * wg + 1], (i >> 1) & 1, A.status)) break;
            tc_fence_after();
            tmem_ld32(taddr + 64, ra);
            proc(rb, 1);
            tc_fence_before();
            mbar_arrive(&tempty[2 * wg]);
            tmem_ld_wait(ra);
            tmem_ld32(taddr + 96, rb);
            proc(ra, 2);
            tmem_ld_wait(rb);
            proc(rb, 3);
            tc_fence_before();
            mbar_arrive(&tempty[2 * wg + 1]);
        }
        if (wg == 1) {
            xm[row] = m;
            xl[row] = l;
        }
        if (sp == 0) {
            // sum of |q| over this tile's window rows, two threads per
            // channel (64 rows each), read from the swizzled Q tile once its
            // TMA load has landed (a warpgroup with no tiles gets here first)
            mbar_wait(qbar, 0, A.status);
            const int x = (wg * 128 + row) & 127, half = (wg * 128 + row) >> 7;
            const int hf = x >> 6, cw = ((x & 63) * 2) >> 4, wb = ((x & 63) * 2) & 15;
            float acc = 0.f;
            for (int rr = half * 64; rr < half * 64 + 64; ++rr) {
                if (mt * 128 + rr >= GW) break;
                const uint8_t* p = q_s + hf * 16384 + rr * 128 + ((cw ^ (rr & 7)) << 4) + wb;
                acc += fabsf(__half2float(*reinterpret_cast<const __half*>(p)));
            }
            named_bar_sync(3, 256);
            if (half == 1) xm[128 + x] = acc;     // xm[128..255] is free space
            named_bar_sync(3, 256);
            if (half == 0)
                A.apart[(static_cast<int64_t>(u) * (GWpad / 128) + mt) * kHeadDim + x] = acc + xm[128 + x];
        }
        named_bar_sync(1, 256);
        if (wg == 0 && rho < GW) {
            const float m1 = xm[row], l1 = xl[row];
            const float M = fmaxf(m, m1);
            float L = 0.f;
            if (M != __uint_as_float(kNegInf)) {
                if (l > 0.f) L += l * fast_exp2(m - M);
                if (l1 > 0.f) L += l1 * fast_exp2(m1 - M);
            }
            A.part[(static_cast<int64_t>(u) * GWpad + rho) * A.nsplit + sp] = make_float2(M, L);
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 9) tmem_dealloc(tmem, 256);
}

// --------------------------------------------------------------- pass 2

struct Pass2Args {
    SeqPlan plan;
    UnitShape shp;
    DenseView dv;
    int paged;
    int kps, nstages, nqc, Nc;
    const float2* part;    // pass-1 partials [units][GWpad][nsplit1]
    int nsplit1;
    float* dbg_lse;
    float* s;
    int64_t s_stride;
    float* dbg_s;
    int64_t dbg_stride;
    uint32_t* status;
};

__global__ void __launch_bounds__(kPassThreads, 1)
    score_pass2_kernel(const __grid_constant__ CUtensorMap qmap,
                       const __grid_constant__ CUtensorMap kmap, const __grid_constant__ Pass2Args A) {
    const int sp = blockIdx.x, u = blockIdx.y;
    const int Hkv = A.shp.Hkv, W = A.shp.W, GWpad = A.shp.GWpad;
    const int b = u / Hkv, h = u % Hkv;
    const int T = A.plan.T[b], r0 = A.plan.r0[b];
    const int r_end = r0 + A.plan.nseg[b] * A.shp.S;
    const int k_lo = r0 + sp * A.kps;
    const int k_hi = min(r_end, k_lo + A.kps);
    const int nt = k_hi > k_lo ? (k_hi - k_lo + kKeyTile - 1) / kKeyTile : 0;
    if (nt == 0) return;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int NS = A.nstages, nqc = A.nqc, Nc = A.Nc;
    const bool split_cols = (nqc == 2);          // both WGs on every tile
    const uint32_t ncols = split_cols ? 512u : (Nc == 256 ? 512u : 256u);

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    uint8_t* q_s = smem;                                  // GWpad x 256 B
    uint8_t* k_s = smem + GWpad * 256;
    float* nlse_s = reinterpret_cast<float*>(k_s + NS * kStage);   // -lse per column
    int* wpos_s = reinterpret_cast<int*>(nlse_s + GWpad);
    float* sb = reinterpret_cast<float*>(wpos_s + GWpad);
    uint64_t* full = reinterpret_cast<uint64_t*>(sb + 128);
    uint64_t* empty = full + 4;
    uint64_t* tfull = empty + 4;
    uint64_t* tempty = tfull + 4;
    uint64_t* qbar = tempty + 4;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(qbar + 1);

    if (tid == 0) {
        for (int i = 0; i < NS; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], 1);
        }
        for (int i = 0; i < 4; ++i) {
            mbar_init(&tfull[i], 1);
            mbar_init(&tempty[i], split_cols ? 256 : 128);
        }
        mbar_init(qbar, 1);
        mbar_fence_init();
    }
    if (warp == 9) {
        tmem_alloc(tmem_slot, ncols);
        tmem_relinquish();
    }
    pdl_wait();
    // lse of every window row: merge the pass-1 split partials in split order
    // (padded rows get +inf so that they weigh nothing)
    for (int i = tid; i < GWpad; i += kPassThreads) {
        float out = __int_as_float(0x7f800000);
        if (i < A.shp.GW) {
            const float2* p = A.part + (static_cast<int64_t>(u) * GWpad + i) * A.nsplit1;
            float M = __uint_as_float(kNegInf), L = 0.f;
            for (int s0 = 0; s0 < A.nsplit1; s0 += 8) {
                float2 v[8];
#pragma unroll
                for (int k2 = 0; k2 < 8; ++k2)
                    v[k2] = (s0 + k2 < A.nsplit1) ? p[s0 + k2] : make_float2(__uint_as_float(kNegInf), 0.f);
#pragma unroll
                for (int k2 = 0; k2 < 8; ++k2) {
                    if (!(v[k2].y > 0.f)) continue;
                    const float M2 = fmaxf(M, v[k2].x);
                    L = L * exp2f(M - M2) + v[k2].y * exp2f(v[k2].x - M2);
                    M = M2;
                }
            }
            out = M + log2f(L);
            if (A.dbg_lse && sp == 0) {
                const int g = i / W, wi = i % W;
                A.dbg_lse[(static_cast<int64_t>(b) * A.shp.Hq + h * A.shp.G + g) * W + wi] =
                    out * 0.69314718055994531f;
            }
        }
        nlse_s[i] = -out;
        wpos_s[i] = i % W;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 8) {
        if (lane == 0) {
            tma_prefetch_desc(&qmap);
            tma_prefetch_desc(&kmap);
            const int qrow0 = (b * A.shp.Hq + h * A.shp.G) * W;
            mbar_expect_tx(qbar, GWpad * 256);
            for (int qc = 0; qc < nqc; ++qc)
                for (int hf = 0; hf < 2; ++hf)
                    for (int rb = 0; rb < Nc / 64; ++rb)
                        tma_load_2d(q_s + qc * Nc * 256 + hf * Nc * 128 + rb * 8192, &qmap, qbar,
                                    hf * 64, qrow0 + qc * Nc + rb * 64);
            for (int i = 0; i < nt; ++i) {
                const int s = i % NS;
                if (i >= NS && !mbar_wait(&empty[s], ((i / NS) - 1) & 1, A.status)) break;
                mbar_expect_tx(&full[s], kStage);
                load_key_tile(k_s + s * kStage, &kmap, &full[s], A.dv, A.paged, b, h,
                              k_lo + i * kKeyTile, T, A.status);
            }
        }
    } else if (warp == 9) {
        if (lane == 0) {
            const uint32_t idesc = idesc_f16_f32(128, Nc);
            const uint32_t qa = smem_u32(q_s);
            bool ok = mbar_wait(qbar, 0, A.status);
            // G*W <= 256: each warpgroup's accumulator is two half-width
            // buffers with their own barriers, so the MMA refills the first
            // half while the epilogue still reads the second
            const bool halves = !split_cols;
            const uint32_t idesc_h = idesc_f16_f32(128, Nc / 2);
            for (int i = 0; ok && halves && i < nt; ++i) {
                // tile i into the half buffers 2 (i & 1) + h, Nc / 2 columns each
                const int s = i % NS;
                if (!mbar_wait(&full[s], (i / NS) & 1, A.status)) break;
                const uint32_t ka = smem_u32(k_s + s * kStage);
                for (int hh = 0; hh < 2; ++hh) {
                    const int hb = 2 * (i & 1) + hh;
                    if (i >= 2 && !mbar_wait(&tempty[hb], ((i >> 1) - 1) & 1, A.status)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t qb = qa + hh * (Nc / 2) * 128;
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk) {
                        const uint32_t aoff = (kk >> 2) * 16384 + (kk & 3) * 32;
                        const uint32_t boff = (kk >> 2) * (Nc * 128) + (kk & 3) * 32;
                        umma_f16(tmem + hb * (Nc / 2), sw128_kmajor_desc(ka + aoff),
                                 sw128_kmajor_desc(qb + boff), idesc_h, kk > 0 ? 1u : 0u);
                    }
                    umma_commit(&tfull[hb]);
                }
                if (!ok) break;
                umma_commit(&empty[s]);
            }
            // split-column mode: both column halves of every tile into one
            // buffer pair
            for (int i = 0; ok && split_cols && i < nt; ++i) {
                const int s = i % NS;
                if (!mbar_wait(&full[s], (i / NS) & 1, A.status)) break;
                if (i >= 1 && !mbar_wait(&tempty[0], (i - 1) & 1, A.status)) break;
                tc_fence_after();
                const uint32_t ka = smem_u32(k_s + s * kStage);
                for (int qc = 0; qc < nqc; ++qc) {
                    const uint32_t dcol = qc * Nc;
                    const uint32_t qb = qa + qc * Nc * 256;
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk) {
                        const uint32_t aoff = (kk >> 2) * 16384 + (kk & 3) * 32;
                        const uint32_t boff = (kk >> 2) * (Nc * 128) + (kk & 3) * 32;
                        umma_f16(tmem + dcol, sw128_kmajor_desc(ka + aoff),
                                 sw128_kmajor_desc(qb + boff), idesc, kk > 0 ? 1u : 0u);
                    }
                }
                umma_commit(&empty[s]);
                umma_commit(&tfull[0]);
            }
        }
    } else {
        // epilogue: thread <-> key (TMEM lane), loop over query columns.
        const int wg = warp >> 2, lg = warp & 3;
        const int row = lg * 32 + lane;
        const float c2 = A.shp.c2;
        const int tw = T - W;                 // keys <= tw are seen by every row
        const int step = split_cols ? 1 : 2;
        const bool halves = !split_cols;
        const int nparts = halves ? 2 : 1;
        const int ncol = halves ? Nc / 2 : Nc;    // columns per TMEM buffer
        for (int i = split_cols ? 0 : wg; i < nt; i += step) {
            const int k = split_cols ? i : (i >> 1);
            const int t = k_lo + i * kKeyTile + row;
            const int need = t - tw;          // row visible iff wpos >= need
            float sacc = 0.f;
            bool ok = true;
            for (int part = 0; part < nparts; ++part) {
                const int buf = split_cols ? 0 : 2 * wg + part;
                if (!mbar_wait(&tfull[buf], k & 1, A.status)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const int qc = split_cols ? wg : 0;
                const uint32_t taddr = tmem + (static_cast<uint32_t>(lg * 32) << 16) +
                                       (split_cols ? qc * Nc : buf * ncol);
                const int col0 = split_cols ? qc * Nc : part * ncol;
                // 32-column chunks, double-buffered: chunk c+1's TMEM load is
                // in flight while chunk c is summed
                auto proc = [&](const uint32_t (&r)[32], int cc) {
                    const float4* l4 = reinterpret_cast<const float4*>(nlse_s + col0 + cc);
                    if (need <= 0) {
                        // packed pairs: (a0, a1) and (a2, a3) accumulate
                        // columns 4q + {0, 1} and 4q + {2, 3}; of each 8
                        // columns the last kP2PolyPairs pairs take exp2 on
                        // the FMA pipe, the rest on MUFU
                        const float2 c2v = make_float2(c2, c2);
                        float2 a01 = make_float2(0.f, 0.f), a23 = make_float2(0.f, 0.f);
#pragma unroll
                        for (int j = 0; j < 32; j += 8) {
                            const float4 n0 = l4[j >> 2], n1 = l4[(j >> 2) + 1];
                            float2 x[4];
                            x[0] = f2_fma(make_float2(__uint_as_float(r[j]), __uint_as_float(r[j + 1])), c2v,
                                          make_float2(n0.x, n0.y));
                            x[1] = f2_fma(make_float2(__uint_as_float(r[j + 2]), __uint_as_float(r[j + 3])), c2v,
                                          make_float2(n0.z, n0.w));
                            x[2] = f2_fma(make_float2(__uint_as_float(r[j + 4]), __uint_as_float(r[j + 5])), c2v,
                                          make_float2(n1.x, n1.y));
                            x[3] = f2_fma(make_float2(__uint_as_float(r[j + 6]), __uint_as_float(r[j + 7])), c2v,
                                          make_float2(n1.z, n1.w));
                            float2 e[4];
#pragma unroll
                            for (int q = 0; q < 4; ++q)
                                e[q] = (q >= 4 - kP2PolyPairs) ? exp2_fma2(x[q])
                                                               : make_float2(fast_exp2(x[q].x), fast_exp2(x[q].y));
                            a01 = f2_add(a01, e[0]);
                            a23 = f2_add(a23, e[1]);
                            a01 = f2_add(a01, e[2]);
                            a23 = f2_add(a23, e[3]);
                        }
                        sacc += (a01.x + a01.y) + (a23.x + a23.y);
                    } else {
                        const int* wp = wpos_s + col0 + cc;
                        float a0 = 0.f;
#pragma unroll
                        for (int j = 0; j < 32; ++j) {
                            const float e = fast_exp2(fmaf(__uint_as_float(r[j]), c2, nlse_s[col0 + cc + j]));
                            a0 += (wp[j] >= need) ? e : 0.f;
                        }
                        sacc += a0;
                    }
                };
                uint32_t ra[32], rb[32];
                const int nch = ncol / 32;        // 2 .. 8 chunks
                tmem_ld32(taddr, ra);
                tmem_ld_wait(ra);
#pragma unroll 1
                for (int ch = 0; ch < nch; ch += 2) {
                    if (ch + 1 < nch) tmem_ld32(taddr + (ch + 1) * 32, rb);
                    proc(ra, ch * 32);
                    if (ch + 1 < nch) {
                        tmem_ld_wait(rb);
                        if (ch + 2 < nch) tmem_ld32(taddr + (ch + 2) * 32, ra);
                        proc(rb, (ch + 1) * 32);
                        if (ch + 2 < nch) tmem_ld_wait(ra);
                    }
                }
                tc_fence_before();
                if (!split_cols) mbar_arrive(&tempty[buf]);
            }
            if (!ok) break;
            if (split_cols) {
                if (wg == 1) sb[row] = sacc;
                named_bar_sync(1, 256);
                if (wg == 0) sacc = sacc + sb[row];
                named_bar_sync(2, 256);
                mbar_arrive(&tempty[0]);
            }
            if ((!split_cols || wg == 0) && t < k_hi) {
                const int64_t rel = t - r0;
                A.s[static_cast<int64_t>(u) * A.s_stride + rel] = sacc;
                if (A.dbg_s) A.dbg_s[static_cast<int64_t>(u) * A.dbg_stride + rel] = sacc;
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 9) tmem_dealloc(tmem, ncols);
}

// ------------------------------------------------- channel top-c and g_t

// Bitonic sort of 128 keys into descending order, fully unrolled so that
// every index is a compile-time constant and the array stays in registers.
__device__ __forceinline__ void sort128_desc(uint32_t (&v)[128]) {
#pragma unroll
    for (int k = 2; k <= 128; k <<= 1) {
#pragma unroll
        for (int j = k >> 1; j > 0; j >>= 1) {
#pragma unroll
            for (int i = 0; i < 128; ++i) {
                const int l = i ^ j;
                if (l > i) {
                    const uint32_t a = v[i], c = v[l];
                    const uint32_t hi = max(a, c), lo = min(a, c);
                    if ((i & k) == 0) {
                        v[i] = hi;
                        v[l] = lo;
                    } else {
                        v[i] = lo;
                        v[l] = hi;
                    }
                }
            }
        }
    }
}

struct ChanArgs {
    SeqPlan plan;
    int Hkv, S, c, GW, mtiles;
    DenseView dv;
    int paged;
    const float* apart;    // [units][mtiles][d] partial sums of |q|
    float* dbg_a;
    double* g;
    uint4* cmask;          // [units][g_stride]: bit x set iff channel x is kept
    int64_t g_stride;
    double* dbg_g;
    int64_t dbg_stride;
    uint32_t* status;
};

// a_x = (sum of the row-tile partial sums, in tile order) / (G * W).
__device__ __forceinline__ float chan_weight(const ChanArgs& A, int u, int x) {
    float s = 0.f;
    for (int mt = 0; mt < A.mtiles; ++mt) s += A.apart[(static_cast<int64_t>(u) * A.mtiles + mt) * kHeadDim + x];
    return s / static_cast<float>(A.GW);
}

// One thread per key.  The block's 128 key rows sit in shared memory with
// their 16-byte chunks XOR-swizzled by (row & 7), so that 8 consecutive
// threads reading the same logical chunk hit 8 different bank groups.
//
// Selection: f_x = fp32(|k_x| * a_x) is the correctly rounded value of the
// exact product e_x = |k_x| * a_x, so it is monotone in e_x.  Sorting the
// 32-bit keys (f_x with its low 7 bits replaced by 127 - x) gives the order
// (trunc(f) desc, x asc).  Let v be the truncated value of the c-th key:
// channels above v are in, channels below are out, and channels equal to v
// are ranked exactly by (e desc, x asc) in fp64 when they straddle the cut.
__global__ void __launch_bounds__(128) chan_kernel_generic(const __grid_constant__ ChanArgs A) {
    pdl_wait();
    const int u = blockIdx.y;
    const int b = u / A.Hkv, h = u % A.Hkv;
    const int r0 = A.plan.r0[b];
    const int ntok = A.plan.nseg[b] * A.S;
    const int base = blockIdx.x * 128;
    if (base >= ntok) return;
    __shared__ __align__(16) uint8_t rows[128 * 256];
    __shared__ float as[128];
    const int tid = threadIdx.x;
    as[tid] = chan_weight(A, u, tid);
    if (A.dbg_a && blockIdx.x == 0) A.dbg_a[static_cast<int64_t>(u) * kHeadDim + tid] = as[tid];
    for (int idx = tid; idx < 128 * 16; idx += 128) {
        const int rr = idx >> 4, ch = idx & 15;
        uint4 val = make_uint4(0, 0, 0, 0);
        if (base + rr < ntok) {
            const __half* src = dense_row(A.dv, A.dv.k, b, h, r0 + base + rr, A.status);
            if (src) val = *reinterpret_cast<const uint4*>(src + ch * 8);
        }
        *reinterpret_cast<uint4*>(rows + rr * 256 + ((ch ^ (rr & 7)) << 4)) = val;
    }
    __syncthreads();
    const int t = base + tid;
    if (t >= ntok) return;
    const uint8_t* myrow = rows + tid * 256;
    const int sw = tid & 7;
    const int c = A.c;

    uint32_t key[128];
#pragma unroll
    for (int ch = 0; ch < 16; ++ch) {
        const uint4 q = *reinterpret_cast<const uint4*>(myrow + ((ch ^ sw) << 4));
        const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const int x = ch * 8 + e * 2 + hh;
                const uint16_t hb = static_cast<uint16_t>(hh ? (w[e] >> 16) : (w[e] & 0xffff));
                const float mag = fabsf(__half2float(__ushort_as_half(hb)));
                const float f = __fmul_rn(mag, as[x]);
                key[x] = (__float_as_uint(f) & 0xFFFFFF80u) | static_cast<uint32_t>(127 - x);
            }
        }
    }
    sort128_desc(key);
    uint32_t kc = 0;
#pragma unroll
    for (int i = 0; i < 128; ++i)
        if (i == c - 1) kc = key[i];
    const uint32_t v = kc >> 7;
    int n_gt = 0, n_eq = 0;
    uint32_t m0 = 0, m1 = 0, m2 = 0, m3 = 0;
#pragma unroll
    for (int i = 0; i < 128; ++i) {
        const uint32_t tv = key[i] >> 7;
        n_gt += (tv > v);
        n_eq += (tv == v);
        if (i < c) {
            const int x = 127 - static_cast<int>(key[i] & 127u);
            const uint32_t bit = 1u << (x & 31);
            m0 |= (x >> 5) == 0 ? bit : 0u;
            m1 |= (x >> 5) == 1 ? bit : 0u;
            m2 |= (x >> 5) == 2 ? bit : 0u;
            m3 |= (x >> 5) == 3 ? bit : 0u;
        }
    }
    auto elem = [&](int x) -> float {
        const int ch = x >> 3, within = x & 7;
        const uint16_t hb = *reinterpret_cast<const uint16_t*>(myrow + ((ch ^ sw) << 4) + within * 2);
        return fabsf(__half2float(__ushort_as_half(hb)));
    };
    if (n_gt + n_eq > c) {
        // exact ranking of the channels whose truncated key equals v
        const int need = c - n_gt;
        for (int x = 0; x < 128; ++x) {
            const float f = __fmul_rn(elem(x), as[x]);
            if ((__float_as_uint(f) >> 7) != v) continue;
            const double ex = __dmul_rn(static_cast<double>(elem(x)), static_cast<double>(as[x]));
            int rank = 0;
            for (int y = 0; y < 128; ++y) {
                if (y == x) continue;
                const float fy = __fmul_rn(elem(y), as[y]);
                if ((__float_as_uint(fy) >> 7) != v) continue;
                const double ey =
                    __dmul_rn(static_cast<double>(elem(y)), static_cast<double>(as[y]));
                rank += (ey > ex) || (ey == ex && y < x);
            }
            const uint32_t bit = 1u << (x & 31);
            const uint32_t set = rank < need ? bit : 0u;
            const int w = x >> 5;
            if (w == 0) m0 = (m0 & ~bit) | set;
            else if (w == 1) m1 = (m1 & ~bit) | set;
            else if (w == 2) m2 = (m2 & ~bit) | set;
            else m3 = (m3 & ~bit) | set;
        }
    }
    const int64_t slot = static_cast<int64_t>(u) * A.g_stride + t;
    double tot = 0.0, drop = 0.0;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
        const uint32_t mw = (w == 0) ? m0 : (w == 1) ? m1 : (w == 2) ? m2 : m3;
#pragma unroll 4
        for (int bit = 0; bit < 32; ++bit) {
            const int x = w * 32 + bit;
            const double e = __dmul_rn(static_cast<double>(elem(x)), static_cast<double>(as[x]));
            tot = __dadd_rn(tot, e);
            if (!((mw >> bit) & 1u)) drop = __dadd_rn(drop, e);
        }
    }
    A.cmask[slot] = make_uint4(m0, m1, m2, m3);
    const double gv = tot > 0.0 ? __ddiv_rn(drop, tot) : 0.0;
    A.g[slot] = gv;
    if (A.dbg_g) A.dbg_g[static_cast<int64_t>(u) * A.dbg_stride + t] = gv;
}


// ---- fast path for c <= 32
//
// Keys are fp16 roundings of the fp32 products |k_x| * a_x.  Both roundings
// are correct roundings (fp16 conversion, min / max and compare keep
// subnormals), so a key is a monotone function of the exact product and
// key_x > key_y implies e_x > e_y.  Register j holds channels 2j (low half)
// and 2j + 1 (high half), so each __hmax2 / __hmin2 pair is two
// compare-exchanges and registers 0..31 / 32..63 hold four lists of 32 keys
// (even and odd channels of 0..63 and of 64..127).  Each list is sorted by
// Batcher's odd-even merge network (191 compare-exchanges for 32 inputs);
// max(X_i, Y_{31-i}) of two descending lists is the set of their 32
// largest, which a bitonic merge sorts again; one more such split gives the
// 32 largest keys of all 128 and v, the c-th largest.  Channels with key > v
// are in and those below are out.  When more than c keys are >= v, the keys
// equal to v straddle the cut and are ranked exactly by (e desc, x asc): by
// their fp32 products, and by the exact fp64 products only where those tie
// (one pass over them when a single one is kept or dropped).  The membership
// pass forms the keys again from the K tile instead of keeping them, so
// only the sort holds them in registers.

__device__ __forceinline__ void ce2(__half2& a, __half2& b) {
    const __half2 hi = __hmax2(a, b), lo = __hmin2(a, b);
    a = hi;
    b = lo;
}

// One (p, k) stage of Batcher's odd-even merge sort of 32 registers into
// descending order, then the next stage; every register index is a
// compile-time constant after unrolling.
template <int P, int K>
__device__ __forceinline__ void oem32_pass(__half2 (&v)[32]) {
#pragma unroll
    for (int j = K % P; j + K < 32; j += 2 * K) {
#pragma unroll
        for (int i = 0; i < K; ++i) {
            if (i < 32 - j - K && (i + j) / (2 * P) == (i + j + K) / (2 * P))
                ce2(v[i + j], v[i + j + K]);
        }
    }
    if constexpr (K > 1) oem32_pass<P, K / 2>(v);
    else if constexpr (P < 16) oem32_pass<P * 2, P * 2>(v);
}

__device__ __forceinline__ void sort32_desc2(__half2 (&v)[32]) {
    oem32_pass<1, 1>(v);
}

// Sorts a bitonic sequence of 32 registers into descending order.
template <int J>
__device__ __forceinline__ void merge32_desc2(__half2 (&v)[32]) {
    if constexpr (J > 0) {
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            const int l = i ^ J;
            if (l > i) ce2(v[i], v[l]);
        }
        merge32_desc2<J / 2>(v);
    }
}

template <int J>
__device__ __forceinline__ void merge32_desc_f(float (&w)[32]) {
    if constexpr (J > 0) {
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            const int l = i ^ J;
            if (l > i) {
                const float hi = fmaxf(w[i], w[l]), lo = fminf(w[i], w[l]);
                w[i] = hi;
                w[l] = lo;
            }
        }
        merge32_desc_f<J / 2>(w);
    }
}

// The key of channels 2e + {0, 1} of a 16-byte K chunk word: fp16 roundings
// of the fp32 products |k_x| * a_x (a monotone function of the exact
// product; see above).
__device__ __forceinline__ __half2 key_pair(uint32_t w, float al, float ah) {
    const float2 m = __half22float2(*reinterpret_cast<const __half2*>(&w));
    return __floats2half2_rn(__fmul_rn(fabsf(m.x), al), __fmul_rn(fabsf(m.y), ah));
}

// Membership masks of one thread's 128 keys against v: bit x of M[x / 32]
// is set iff key_x >= v, of Gt iff key_x > v.  The keys are formed again
// from the K row (the same operations as for the sort, so the same values)
// rather than kept in shared memory, which leaves room for more resident
// CTAs.  A compare yields 0xffff per half; one AND-OR per register moves
// both flags to spare bit positions, and a final shuffle puts each channel
// at its own bit.
template <typename ChunkFn>
__device__ __forceinline__ void key_masks(ChunkFn chunk, const float* af, __half2 vv, uint32_t (&M)[4],
                                          uint32_t (&Gt)[4]) {
    // one copy of the loop body: the unrolled networks and masks of this
    // kernel overflow the instruction cache (instruction-fetch stalls were
    // its largest); the words move through M[0..3] / Gt[0..3] as a queue
#pragma unroll 1
    for (int wd = 0; wd < 4; ++wd) {
        uint32_t lo = 0, hi = 0, glo = 0, ghi = 0;
#pragma unroll
        for (int g4 = 0; g4 < 4; ++g4) {
            const int gi = wd * 4 + g4;
            const uint4 q = chunk(gi);
            const float4 a0 = *reinterpret_cast<const float4*>(af + 8 * gi);
            const float4 a1 = *reinterpret_cast<const float4*>(af + 8 * gi + 4);
            const uint32_t w[4] = {q.x, q.y, q.z, q.w};
            const float al[4] = {a0.x, a0.z, a1.x, a1.z};
            const float ah[4] = {a0.y, a0.w, a1.y, a1.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int s = g4 * 4 + e;        // channels 2s, 2s + 1 of this word
                const __half2 kk = key_pair(w[e], al[e], ah[e]);
                const uint32_t mk = __hge2_mask(kk, vv), gk = __hgt2_mask(kk, vv);
                if (s < 8) {
                    const uint32_t bits = (1u << (2 * s)) | (1u << (2 * s + 17));
                    lo |= mk & bits;
                    glo |= gk & bits;
                } else {
                    const uint32_t bits = (1u << (2 * s - 16)) | (1u << (2 * s + 1));
                    hi |= mk & bits;
                    ghi |= gk & bits;
                }
            }
        }
        const uint32_t mw = (lo & 0x5555u) | ((lo >> 16) & 0xAAAAu) | ((hi << 16) & 0x55550000u) | (hi & 0xAAAA0000u);
        const uint32_t gw = (glo & 0x5555u) | ((glo >> 16) & 0xAAAAu) | ((ghi << 16) & 0x55550000u) | (ghi & 0xAAAA0000u);
        M[0] = M[1];
        M[1] = M[2];
        M[2] = M[3];
        M[3] = mw;
        Gt[0] = Gt[1];
        Gt[1] = Gt[2];
        Gt[2] = Gt[3];
        Gt[3] = gw;
    }
}

// fp64 acc + x * y unless (m & bit) != 0, as one fused multiply-add: the
// callers' products are exact in fp64 (an fp16 magnitude times an fp32
// weight: 11 x 24 significant bits), so rounding x * y + acc once equals
// adding the exact product with one rounding.  One compare into a predicate
// and one guarded instruction, so the skipped add costs no 64-bit select.
__device__ __forceinline__ double dfma_unless(double acc, double x, double y, uint32_t m, uint32_t bit) {
    asm("{\n\t.reg .pred p;\n\t.reg .b32 t;\n\t"
        "and.b32 t, %3, %4;\n\t"
        "setp.eq.u32 p, t, 0;\n\t"
        "@p fma.rn.f64 %0, %1, %2, %0;\n\t}"
        : "+d"(acc)
        : "d"(x), "d"(y), "r"(m), "r"(bit));
    return acc;
}

// An fp16 value (bits) widened to fp64 in one conversion (exact).
__device__ __forceinline__ double h2d(uint16_t bits) {
    double d;
    asm("cvt.f64.f16 %0, %1;" : "=d"(d) : "h"(bits));
    return d;
}

// Rows of a 128-row K tile in the 128-byte-swizzled layout of the scoring
// passes: row r, 16-byte chunk j of a 64-channel half at
// half * 16384 + r * 128 + ((j ^ (r & 7)) << 4), so the 8 threads of each
// quarter-warp (consecutive rows) read 8 different bank groups.
struct ChanRow {
    const uint8_t* row;   // tile + r * 128
    int sw;               // r & 7
    __device__ __forceinline__ uint4 chunk(int j) const {     // channels 8j .. 8j + 7
        return *reinterpret_cast<const uint4*>(row + (j >> 3) * 16384 + (((j & 7) ^ sw) << 4));
    }
    __device__ __forceinline__ uint16_t kbits(int x) const {  // |k_x| as fp16 bits
        const uint16_t* p = reinterpret_cast<const uint16_t*>(row + (x >> 6) * 16384 + ((((x >> 3) & 7) ^ sw) << 4));
        return static_cast<uint16_t>(p[x & 7] & 0x7fffu);
    }
};

// Keep mask of one key row (bit x set iff channel x is kept), c <= 32;
// af / ad hold the weights a_x in fp32 and fp64.
__device__ __forceinline__ uint4 chan_row_mask(const ChanRow R, const float* af, const double* ad, int c) {
    auto chunk = [&](int j) { return R.chunk(j); };
    // the 32 largest keys of the even channels (low halves, L) and of the odd
    // channels (high halves, H), as bitonic sequences in srt[0..31]
    __half2 srt[32];
    {
        __half2 hi[32];
#pragma unroll
        for (int gi = 0; gi < 16; ++gi) {
            const uint4 q = chunk(gi);
            const float4 a0 = *reinterpret_cast<const float4*>(af + 8 * gi);
            const float4 a1 = *reinterpret_cast<const float4*>(af + 8 * gi + 4);
            __half2* d = gi < 8 ? srt + 4 * gi : hi + 4 * (gi - 8);
            d[0] = key_pair(q.x, a0.x, a0.y);
            d[1] = key_pair(q.y, a0.z, a0.w);
            d[2] = key_pair(q.z, a1.x, a1.y);
            d[3] = key_pair(q.w, a1.z, a1.w);
        }
        // one copy of the 32-key network, run on each half in turn (the
        // halves swap places between the runs and are back in place after
        // the second): half the code of two unrolled copies
#pragma unroll 1
        for (int rep = 0; rep < 2; ++rep) {
            sort32_desc2(srt);
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                const __half2 tmp = srt[i];
                srt[i] = hi[i];
                hi[i] = tmp;
            }
        }
#pragma unroll
        for (int i = 0; i < 32; ++i) srt[i] = __hmax2(srt[i], hi[31 - i]);
    }
    merge32_desc2<16>(srt);          // low halves: L, high halves: H, descending
    float vf;
    if (c == 32) {
        // the 32 largest of all are max(L_i, H_{31-i}); with the halves of
        // register 31-i swapped, one __hmax2 forms the pairs for i and 31-i
        __half2 mn = __half2half2(__ushort_as_half(0x7c00));   // +inf
#pragma unroll
        for (int i = 0; i < 16; ++i) mn = __hmin2(mn, __hmax2(srt[i], __lowhigh2highlow(srt[31 - i])));
        vf = fminf(__low2float(mn), __high2float(mn));
    } else {
        float w[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) w[i] = fmaxf(__low2float(srt[i]), __high2float(srt[31 - i]));
        merge32_desc_f<16>(w);       // 32 largest of all 128, descending
        vf = w[0];
#pragma unroll
        for (int i = 1; i < 32; ++i) vf = (i < c) ? w[i] : vf;
    }
    const __half2 vv = __float2half2_rn(vf);   // vf is a key value: exact in fp16

    // the K tile is read again below; without this fence the compiler
    // hoists those loads above the sort and keeps both live (160 registers
    // instead of 96)
    uint32_t M[4], G[4];
    asm volatile("" ::: "memory");
    key_masks(chunk, af, vv, M, G);
    const int n_ge = __popc(M[0]) + __popc(M[1]) + __popc(M[2]) + __popc(M[3]);
    if (n_ge > c) {
        // the keys equal to v straddle the cut: keep the c - n_gt best of
        // them by (e desc, x asc).  The fp32 products f = fp32(|k| a) are
        // correctly rounded, so f_y > f_x implies e_y > e_x; only equal f
        // need the exact fp64 products.
        const int n_gt = __popc(G[0]) + __popc(G[1]) + __popc(G[2]) + __popc(G[3]);
        const int need = c - n_gt;
        const uint32_t qm[4] = {M[0] & ~G[0], M[1] & ~G[1], M[2] & ~G[2], M[3] & ~G[3]};
        uint32_t keep[4] = {0, 0, 0, 0};
        // y ranks above x: f_y > f_x, or equal f and (e_y > e_x, or equal e and y < x)
        auto above = [&](int y, double ky, float fy, int x, double kx, float fx) {
            if (fy != fx) return fy > fx;
            const double ex = __dmul_rn(kx, ad[x]), ey = __dmul_rn(ky, ad[y]);
            return (ey > ex) || (ey == ex && y < x);
        };
        if (need == 1 || need == n_ge - n_gt - 1) {
            // one pass over the tied channels: keep the single best one, or
            // keep all but the single worst one
            const bool best = need == 1;
            int bx = -1;
            double bk = 0.0;
            float bf = 0.f;
            for (int wi = 0; wi < 4; ++wi) {
                for (uint32_t m = qm[wi]; m; m &= m - 1) {
                    const int x = wi * 32 + __ffs(m) - 1;
                    const double kx = h2d(R.kbits(x));
                    const float fx = __fmul_rn(static_cast<float>(kx), af[x]);
                    if (bx < 0 || above(x, kx, fx, bx, bk, bf) == best) {
                        bx = x;
                        bk = kx;
                        bf = fx;
                    }
                }
            }
#pragma unroll
            for (int wi = 0; wi < 4; ++wi) {
                const uint32_t bit = (bx >> 5) == wi ? 1u << (bx & 31) : 0u;
                keep[wi] = best ? bit : (qm[wi] & ~bit);
            }
        } else {
            for (int wi = 0; wi < 4; ++wi) {
                for (uint32_t m = qm[wi]; m; m &= m - 1) {
                    const int x = wi * 32 + __ffs(m) - 1;
                    const double kx = h2d(R.kbits(x));
                    const float fx = __fmul_rn(static_cast<float>(kx), af[x]);
                    int rank = 0;
                    for (int wj = 0; wj < 4; ++wj) {
                        for (uint32_t m2 = qm[wj]; m2; m2 &= m2 - 1) {
                            const int y = wj * 32 + __ffs(m2) - 1;
                            if (y == x) continue;
                            const double ky = h2d(R.kbits(y));
                            rank += above(y, ky, __fmul_rn(static_cast<float>(ky), af[y]), x, kx, fx);
                        }
                    }
                    if (rank < need) keep[wi] |= 1u << (x & 31);
                }
            }
        }
#pragma unroll
        for (int wi = 0; wi < 4; ++wi) M[wi] = G[wi] | keep[wi];
    }
    return make_uint4(M[0], M[1], M[2], M[3]);
}

// g_t of one key row under keep mask m: both fp64 sums ascending in x; |k|
// widened exactly, and e = |k| a_x is exact in fp64, so each fused
// multiply-add rounds exactly as adding e does.
__device__ __forceinline__ double chan_row_g(const ChanRow R, const double* ad, uint4 m) {
    const uint32_t M[4] = {m.x, m.y, m.z, m.w};
    double tot = 0.0, drop = 0.0;
#pragma unroll 1
    for (int j = 0; j < 16; ++j) {
        const uint4 q = R.chunk(j);
        const uint32_t mw = ((j < 4) ? M[0] : (j < 8) ? M[1] : (j < 12) ? M[2] : M[3]) >> ((j & 3) * 8);
        const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const double2 a2 = *reinterpret_cast<const double2*>(ad + 8 * j + 2 * e);
            // fp16 -> fp32 on the FMA pipe, then |.| and fp32 -> fp64: all exact
            const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w[e]));
            const double k0 = static_cast<double>(fabsf(f.x));
            const double k1 = static_cast<double>(fabsf(f.y));
            tot = __fma_rn(k0, a2.x, tot);
            drop = dfma_unless(drop, k0, a2.x, mw, 1u << (2 * e));
            tot = __fma_rn(k1, a2.y, tot);
            drop = dfma_unless(drop, k1, a2.y, mw, 2u << (2 * e));
        }
    }
    return tot > 0.0 ? __ddiv_rn(drop, tot) : 0.0;
}

constexpr int kChanTile = 0;                  // 128 K rows, two 64-channel halves (SW128)
constexpr int kChanAf = kStage;               // float [128]
constexpr int kChanAd = kChanAf + 512;        // double [128]
constexpr int kChanBar = kChanAd + 1024;      // one mbarrier
constexpr int kChanSmem = 1024 + kChanBar + 16;

// One CTA per 128 tokens of a unit, one thread per token, for short
// regions.  K is never written by the kernels this one follows, so the
// tile's copy is issued before the wait on them and overlaps their tail.
// The tile is the only large shared buffer (about 35 KB per CTA), and the
// kernel is held to 96 registers, so five CTAs of 128 threads share an SM.
__global__ void __launch_bounds__(128, 5) chan_kernel_c32(const __grid_constant__ CUtensorMap kmap,
                                                          const __grid_constant__ ChanArgs A) {
    extern __shared__ uint8_t chan_smem_raw[];
    uint8_t* sm = align1024(chan_smem_raw);
    uint8_t* tile = sm + kChanTile;
    float* af = reinterpret_cast<float*>(sm + kChanAf);
    double* ad = reinterpret_cast<double*>(sm + kChanAd);
    uint64_t* bar = reinterpret_cast<uint64_t*>(sm + kChanBar);

    const int u = blockIdx.y;
    const int b = u / A.Hkv, h = u % A.Hkv;
    const int r0 = A.plan.r0[b];
    const int ntok = A.plan.nseg[b] * A.S;
    const int base = blockIdx.x * 128;
    if (base >= ntok) return;
    const int tid = threadIdx.x;
    if (tid == 0) {
        mbar_init(bar, 1);
        mbar_fence_init();
        tma_prefetch_desc(&kmap);
        mbar_expect_tx(bar, kStage);
        load_key_tile(tile, &kmap, bar, A.dv, A.paged, b, h, r0 + base, r0 + ntok, A.status);
    }
    pdl_wait();
    {
        const float av = chan_weight(A, u, tid);
        if (A.dbg_a && blockIdx.x == 0) A.dbg_a[static_cast<int64_t>(u) * kHeadDim + tid] = av;
        af[tid] = av;
        ad[tid] = static_cast<double>(av);
    }
    __syncthreads();
    if (!mbar_wait(bar, 0, A.status)) return;
    const int t = base + tid;
    if (t >= ntok) return;
    const ChanRow R{tile + tid * 128, tid & 7};
    const uint4 m = chan_row_mask(R, af, ad, A.c);
    const double gv = chan_row_g(R, ad, m);
    const int64_t slot = static_cast<int64_t>(u) * A.g_stride + t;
    A.cmask[slot] = m;
    A.g[slot] = gv;
    if (A.dbg_g) A.dbg_g[static_cast<int64_t>(u) * A.dbg_stride + t] = gv;
}

}  // namespace

// ------------------------------------------------------------------ host

int score_pass1_smem_bytes() {
    return 1024 + 32768 + kP1Stages * kStage + 256 + 1536;
}

int score_pass2_smem_bytes(int gwpad) {
    const int ns = gwpad <= 256 ? 4 : 2;
    return 1024 + gwpad * 256 + ns * kStage + gwpad * 8 + 512 + 256;
}

cudaError_t launch_scoring(const ScoreLaunch& L, cudaStream_t stream) {
    const int units = L.batch * L.shp.Hkv;
    cudaError_t e = cudaSuccess;

    Pass1Args p1;
    p1.plan = L.plan;
    p1.shp = L.shp;
    p1.dv = L.dv;
    p1.paged = L.paged;
    p1.kps = L.kps1;
    p1.nsplit = L.nsplit1;
    p1.part = L.part;
    p1.apart = L.apart;
    p1.status = L.status;
    const int smem1 = score_pass1_smem_bytes();
    e = cudaFuncSetAttribute(score_pass1_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem1);
    if (e != cudaSuccess) return e;
    dim3 g1(L.nsplit1, L.shp.GWpad / 128, units);
    prof_begin(stream, kProfPass1);
    e = launch_k(score_pass1_kernel, g1, dim3(kPassThreads), smem1, stream, L.qmap, L.kmap, p1);
    if (e != cudaSuccess) return e;
    prof_end(stream, kProfPass1);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;

    Pass2Args p2;
    p2.plan = L.plan;
    p2.shp = L.shp;
    p2.dv = L.dv;
    p2.paged = L.paged;
    p2.kps = L.kps2;
    p2.nstages = L.shp.GWpad <= 256 ? 4 : 2;
    p2.nqc = L.shp.GWpad <= 256 ? 1 : 2;
    p2.Nc = L.shp.GWpad / p2.nqc;
    p2.part = L.part;
    p2.nsplit1 = L.nsplit1;
    p2.dbg_lse = L.dbg_lse;
    p2.s = L.s;
    p2.s_stride = L.s_stride;
    p2.dbg_s = L.dbg_s;
    p2.dbg_stride = L.dbg_stride;
    p2.status = L.status;
    const int smem2 = score_pass2_smem_bytes(L.shp.GWpad);
    e = cudaFuncSetAttribute(score_pass2_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem2);
    if (e != cudaSuccess) return e;
    dim3 g2(L.nsplit2, units);
    prof_begin(stream, kProfPass2);
    e = launch_k(score_pass2_kernel, g2, dim3(kPassThreads), smem2, stream, L.qmap, L.kmap, p2);
    if (e != cudaSuccess) return e;
    prof_end(stream, kProfPass2);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;

    ChanArgs ca;
    ca.plan = L.plan;
    ca.Hkv = L.shp.Hkv;
    ca.S = L.shp.S;
    ca.c = L.shp.c;
    ca.dv = L.dv;
    ca.paged = L.paged;
    ca.GW = L.shp.GW;
    ca.mtiles = L.shp.GWpad / 128;
    ca.apart = L.apart;
    ca.dbg_a = L.dbg_a;
    ca.g = L.g;
    ca.cmask = L.cmask;
    ca.g_stride = L.g_stride;
    ca.dbg_g = L.dbg_g;
    ca.dbg_stride = L.dbg_stride;
    ca.status = L.status;
    dim3 gc((L.max_nseg * L.shp.S + 127) / 128, units);
    if (gc.x > 0) {
        prof_begin(stream, kProfChan);
        if (L.shp.c <= 32) {
            e = cudaFuncSetAttribute(chan_kernel_c32, cudaFuncAttributeMaxDynamicSharedMemorySize, kChanSmem);
            if (e == cudaSuccess) e = launch_k(chan_kernel_c32, gc, dim3(128), kChanSmem, stream, L.kmap, ca);
        } else {
            e = launch_k(chan_kernel_generic, gc, dim3(128), 0, stream, ca);
        }
        if (e != cudaSuccess) return e;
        prof_end(stream, kProfChan);
    }
    return cudaGetLastError();
}

}  // namespace kv2d
