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
//               owns one key and sums over queries in-thread
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
    uint64_t* tempty = tfull + 2;
    uint64_t* qbar = tempty + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(qbar + 1);
    float* xm = reinterpret_cast<float*>(tmem_slot + 4);   // [256]
    float* xl = xm + 256;

    if (tid == 0) {
        for (int i = 0; i < kP1Stages; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
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
            constexpr uint32_t idesc = idesc_f16_f32(128, 128);
            const uint32_t qa = smem_u32(q_s);
            bool ok = mbar_wait(qbar, 0, A.status);
            for (int i = 0; ok && i < nt; ++i) {
                const int s = i % kP1Stages, buf = i & 1;
                if (!mbar_wait(&full[s], (i / kP1Stages) & 1, A.status)) break;
                if (i >= 2 && !mbar_wait(&tempty[buf], ((i >> 1) - 1) & 1, A.status)) break;
                tc_fence_after();
                const uint32_t ka = smem_u32(k_s + s * kStage);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
                    umma_f16(tmem + buf * 128, sw128_kmajor_desc(qa + off),
                             sw128_kmajor_desc(ka + off), idesc, kk > 0 ? 1u : 0u);
                }
                umma_commit(&empty[s]);
                umma_commit(&tfull[buf]);
            }
        }
    } else {
        // epilogue: warps 0-3 take even tiles (TMEM columns 0..127), warps
        // 4-7 odd tiles (columns 128..255); thread <-> window row.
        const int wg = warp >> 2, lg = warp & 3;
        const int row = lg * 32 + lane;
        const int rho = mt * 128 + row;
        const int pw = (rho < GW) ? (T - W + (rho % W)) : -1;   // last key the row sees
        const int lim = min(pw, k_hi - 1);
        const float c2 = A.shp.c2;
        float m = __uint_as_float(kNegInf), l = 0.f;
        for (int i = wg; i < nt; i += 2) {
            if (!mbar_wait(&tfull[wg], (i >> 1) & 1, A.status)) break;
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
#pragma unroll
                    for (int j = 0; j < 32; j += 4) {
                        a0 += fast_exp2(fmaf(__uint_as_float(r[j]), c2, nm));
                        a1 += fast_exp2(fmaf(__uint_as_float(r[j + 1]), c2, nm));
                        a2 += fast_exp2(fmaf(__uint_as_float(r[j + 2]), c2, nm));
                        a3 += fast_exp2(fmaf(__uint_as_float(r[j + 3]), c2, nm));
                    }
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
            uint32_t ra[32], rb[32];
            tmem_ld32(taddr, ra);
            tmem_ld_wait(ra);
            tmem_ld32(taddr + 32, rb);
            proc(ra, 0);
            tmem_ld_wait(rb);
            tmem_ld32(taddr + 64, ra);
            proc(rb, 1);
            tmem_ld_wait(ra);
            tmem_ld32(taddr + 96, rb);
            proc(ra, 2);
            tmem_ld_wait(rb);
            proc(rb, 3);
            tc_fence_before();
            mbar_arrive(&tempty[wg]);
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
    float* lse_s = reinterpret_cast<float*>(k_s + NS * kStage);
    int* wpos_s = reinterpret_cast<int*>(lse_s + GWpad);
    float* sb = reinterpret_cast<float*>(wpos_s + GWpad);
    uint64_t* full = reinterpret_cast<uint64_t*>(sb + 128);
    uint64_t* empty = full + 4;
    uint64_t* tfull = empty + 4;
    uint64_t* tempty = tfull + 2;
    uint64_t* qbar = tempty + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(qbar + 1);

    if (tid == 0) {
        for (int i = 0; i < NS; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
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
        lse_s[i] = out;
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
            for (int i = 0; ok && i < nt; ++i) {
                const int s = i % NS;
                const int buf = split_cols ? 0 : (i & 1);
                if (!mbar_wait(&full[s], (i / NS) & 1, A.status)) break;
                if (split_cols) {
                    if (i >= 1 && !mbar_wait(&tempty[0], (i - 1) & 1, A.status)) break;
                } else if (i >= 2 && !mbar_wait(&tempty[buf], ((i >> 1) - 1) & 1, A.status)) {
                    break;
                }
                tc_fence_after();
                const uint32_t ka = smem_u32(k_s + s * kStage);
                for (int qc = 0; qc < nqc; ++qc) {
                    const uint32_t dcol = split_cols ? qc * Nc : buf * Nc;
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
                umma_commit(&tfull[buf]);
            }
        }
    } else {
        // epilogue: thread <-> key (TMEM lane), loop over query columns.
        const int wg = warp >> 2, lg = warp & 3;
        const int row = lg * 32 + lane;
        const float c2 = A.shp.c2;
        const int tw = T - W;                 // keys <= tw are seen by every row
        const int step = split_cols ? 1 : 2;
        for (int i = split_cols ? 0 : wg; i < nt; i += step) {
            const int buf = split_cols ? 0 : wg;
            const int k = split_cols ? i : (i >> 1);
            if (!mbar_wait(&tfull[buf], k & 1, A.status)) break;
            tc_fence_after();
            const int t = k_lo + i * kKeyTile + row;
            const int qc = split_cols ? wg : 0;
            const uint32_t taddr = tmem + (static_cast<uint32_t>(lg * 32) << 16) +
                                   (split_cols ? qc * Nc : buf * Nc);
            const int col0 = qc * Nc;
            const int need = t - tw;          // row visible iff wpos >= need
            float sacc = 0.f;
            // 32-column chunks, double-buffered: chunk c+1's TMEM load is in
            // flight while chunk c is summed
            auto proc = [&](const uint32_t (&r)[32], int cc) {
                const float4* l4 = reinterpret_cast<const float4*>(lse_s + col0 + cc);
                float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
                if (need <= 0) {
#pragma unroll
                    for (int j = 0; j < 32; j += 4) {
                        const float4 lz = l4[j >> 2];
                        a0 += fast_exp2(fmaf(__uint_as_float(r[j]), c2, -lz.x));
                        a1 += fast_exp2(fmaf(__uint_as_float(r[j + 1]), c2, -lz.y));
                        a2 += fast_exp2(fmaf(__uint_as_float(r[j + 2]), c2, -lz.z));
                        a3 += fast_exp2(fmaf(__uint_as_float(r[j + 3]), c2, -lz.w));
                    }
                } else {
                    const int* wp = wpos_s + col0 + cc;
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        const float e = fast_exp2(fmaf(__uint_as_float(r[j]), c2, -lse_s[col0 + cc + j]));
                        a0 += (wp[j] >= need) ? e : 0.f;
                    }
                }
                sacc += (a0 + a1) + (a2 + a3);
            };
            uint32_t ra[32], rb[32];
            const int nch = Nc / 32;          // 4, 6 or 8 chunks (Nc 128..256)
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
            if (split_cols) {
                if (wg == 1) sb[row] = sacc;
                named_bar_sync(1, 256);
                if (wg == 0) sacc = sacc + sb[row];
                named_bar_sync(2, 256);
            }
            mbar_arrive(&tempty[buf]);
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
    const float* apart;    // [units][mtiles][d] partial sums of |q|
    float* dbg_a;
    double* g;
    uint8_t* cidx;
    int64_t g_stride;
    double* dbg_g;
    int64_t dbg_stride;
    uint32_t* status;
};

// a_x = (sum of the row-tile partial sums, in tile order) / (G * W); the
// first CTA of a unit also writes it to the debug output.
__device__ __forceinline__ float chan_weight(const ChanArgs& A, int u, int x) {
    float s = 0.f;
    for (int mt = 0; mt < A.mtiles; ++mt) s += A.apart[(static_cast<int64_t>(u) * A.mtiles + mt) * kHeadDim + x];
    const float v = s / static_cast<float>(A.GW);
    if (A.dbg_a && blockIdx.x == 0) A.dbg_a[static_cast<int64_t>(u) * kHeadDim + x] = v;
    return v;
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
    uint8_t* out = A.cidx + slot * c;
    int k = 0;
    double tot = 0.0, drop = 0.0;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
        const uint32_t mw = (w == 0) ? m0 : (w == 1) ? m1 : (w == 2) ? m2 : m3;
#pragma unroll 4
        for (int bit = 0; bit < 32; ++bit) {
            const int x = w * 32 + bit;
            const double e = __dmul_rn(static_cast<double>(elem(x)), static_cast<double>(as[x]));
            tot = __dadd_rn(tot, e);
            if ((mw >> bit) & 1u) out[k++] = static_cast<uint8_t>(x);
            else drop = __dadd_rn(drop, e);
        }
    }
    const double gv = tot > 0.0 ? __ddiv_rn(drop, tot) : 0.0;
    A.g[slot] = gv;
    if (A.dbg_g) A.dbg_g[static_cast<int64_t>(u) * A.dbg_stride + t] = gv;
}


// ---- fast path for c <= 32
//
// Keys are fp16 roundings of the fp32 products |k_x| * a_x (correctly
// rounded twice, so monotone in the exact product; values below 2^-14 are
// set to 0), two channels per register: register i holds channel i in its
// low half and channel 64 + i in its high half, so every __hmax2 / __hmin2
// pair is two compare-exchanges.  Sorting registers 0..31 and 32..63 gives
// four descending 32-lists; max(X_i, Y_{31-i}) and a bitonic merge give the
// top 32 of channels 0..63 (low halves) and of 64..127 (high halves); one
// more merge gives the top 32 of all 128, whose (c-1)-th entry v is the c-th
// largest key.  Channels above v are in, below are out; channels equal to v
// are all in unless they straddle the cut, in which case they are ranked
// exactly by (e desc, x asc) with the fp64 products.

__device__ __forceinline__ void ce2(__half2& a, __half2& b) {
    const __half2 hi = __hmax2(a, b), lo = __hmin2(a, b);
    a = hi;
    b = lo;
}

// One bitonic stage (block size K, distance J) on registers O..O+31, then
// the next; template recursion keeps every register index a compile-time
// constant.
template <int O, int K, int J>
__device__ __forceinline__ void sort32_stage2(__half2 (&v)[64]) {
    if constexpr (J > 0) {
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            const int l = i ^ J;
            if (l > i) {
                if ((i & K) == 0) ce2(v[O + i], v[O + l]);
                else ce2(v[O + l], v[O + i]);
            }
        }
        sort32_stage2<O, K, J / 2>(v);
    } else if constexpr (K < 32) {
        sort32_stage2<O, K * 2, K>(v);
    }
}

template <int O>
__device__ __forceinline__ void sort32_desc2(__half2 (&v)[64]) {
    sort32_stage2<O, 2, 1>(v);
}

template <int J>
__device__ __forceinline__ void merge32_desc2(__half2 (&v)[64]) {
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

// fp16 key of an fp32 product: 0 below the fp16 normal range, inf above it.
__device__ __forceinline__ float key_value(float f) {
    return f < 6.103515625e-05f ? 0.f : f;
}

__global__ void __launch_bounds__(128) chan_kernel_c32(const __grid_constant__ ChanArgs A) {
    pdl_wait();
    const int u = blockIdx.y;
    const int b = u / A.Hkv, h = u % A.Hkv;
    const int r0 = A.plan.r0[b];
    const int ntok = A.plan.nseg[b] * A.S;
    const int base = blockIdx.x * 128;
    if (base >= ntok) return;
    __shared__ __align__(16) float af[128];
    __shared__ double ad[128];
    const int tid = threadIdx.x;
    {
        const float av = chan_weight(A, u, tid);
        af[tid] = av;
        ad[tid] = static_cast<double>(av);
    }
    __syncthreads();
    const int t = base + tid;
    if (t >= ntok) return;
    const int c = A.c;
    const __half* src = dense_row(A.dv, A.dv.k, b, h, r0 + t, A.status);
    auto chunk = [&](int ch) {
        uint4 q = make_uint4(0, 0, 0, 0);
        if (src) q = *reinterpret_cast<const uint4*>(src + ch * 8);
        return q;
    };

    // packed keys: key[i] = (k(i), k(64 + i)) as half2
    __half2 key[64], srt[64];
#pragma unroll
    for (int ch = 0; ch < 8; ++ch) {
        const uint4 lo4 = chunk(ch), hi4 = chunk(ch + 8);
        const uint32_t lw[4] = {lo4.x, lo4.y, lo4.z, lo4.w};
        const uint32_t hw[4] = {hi4.x, hi4.y, hi4.z, hi4.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int x = ch * 8 + 2 * e;               // channels x, x+1 and 64+x, 65+x
            const float2 ml = __half22float2(__habs2(*reinterpret_cast<const __half2*>(&lw[e])));
            const float2 mh = __half22float2(__habs2(*reinterpret_cast<const __half2*>(&hw[e])));
            const float2 al = *reinterpret_cast<const float2*>(af + x);
            const float2 ah = *reinterpret_cast<const float2*>(af + 64 + x);
            key[x] = __floats2half2_rn(key_value(__fmul_rn(ml.x, al.x)), key_value(__fmul_rn(mh.x, ah.x)));
            key[x + 1] = __floats2half2_rn(key_value(__fmul_rn(ml.y, al.y)), key_value(__fmul_rn(mh.y, ah.y)));
            srt[x] = key[x];
            srt[x + 1] = key[x + 1];
        }
    }
    sort32_desc2<0>(srt);
    sort32_desc2<32>(srt);
#pragma unroll
    for (int i = 0; i < 32; ++i) srt[i] = __hmax2(srt[i], srt[63 - i]);
    merge32_desc2<16>(srt);          // low halves: top 32 of channels 0..63 (L),
                                     // high halves: top 32 of 64..127 (H), descending
    float w[32];
#pragma unroll
    for (int i = 0; i < 32; ++i)
        w[i] = fmaxf(__low2float(srt[i]), __high2float(srt[31 - i]));
    merge32_desc_f<16>(w);           // top 32 of all 128, descending
    float vf = __int_as_float(0x7f800000);
#pragma unroll
    for (int i = 0; i < 32; ++i) vf = fminf(vf, (i < c) ? w[i] : __int_as_float(0x7f800000));
    const __half2 vv = __float2half2_rn(vf);   // vf is a key value: exact in fp16

    // membership masks over channels: gt (key > v) and eq (key == v)
    uint32_t g0 = 0, g1 = 0, g2 = 0, g3 = 0, q0 = 0, q1 = 0, q2 = 0, q3 = 0;
#pragma unroll
    for (int i = 0; i < 64; ++i) {
        const uint32_t gt = __hgt2_mask(key[i], vv), eq = __heq2_mask(key[i], vv);
        const uint32_t bit = 1u << (i & 31);
        // low half: channel i; high half: channel 64 + i
        if (i < 32) {
            g0 |= (gt & 1u) ? bit : 0u;
            q0 |= (eq & 1u) ? bit : 0u;
            g2 |= (gt >> 31) ? bit : 0u;
            q2 |= (eq >> 31) ? bit : 0u;
        } else {
            g1 |= (gt & 1u) ? bit : 0u;
            q1 |= (eq & 1u) ? bit : 0u;
            g3 |= (gt >> 31) ? bit : 0u;
            q3 |= (eq >> 31) ? bit : 0u;
        }
    }
    const int n_gt = __popc(g0) + __popc(g1) + __popc(g2) + __popc(g3);
    const int n_eq = __popc(q0) + __popc(q1) + __popc(q2) + __popc(q3);
    if (n_gt + n_eq > c) {
        // the channels equal to v straddle the cut: keep the c - n_gt best of
        // them by the exact product (e desc, x asc)
        const int need = c - n_gt;
        uint32_t qm[4] = {q0, q1, q2, q3};
        uint32_t keep[4] = {0, 0, 0, 0};
        for (int wi = 0; wi < 4; ++wi) {
            for (uint32_t m = qm[wi]; m; m &= m - 1) {
                const int x = wi * 32 + __ffs(m) - 1;
                const uint4 cx = chunk(x >> 3);
                const uint32_t wx = (x & 7) < 2 ? cx.x : (x & 7) < 4 ? cx.y : (x & 7) < 6 ? cx.z : cx.w;
                const float mx = fabsf(__half2float(__ushort_as_half(static_cast<uint16_t>((x & 1) ? (wx >> 16) : (wx & 0xffffu)))));
                const double ex = __dmul_rn(static_cast<double>(mx), ad[x]);
                int rank = 0;
                for (int wj = 0; wj < 4; ++wj) {
                    for (uint32_t m2 = qm[wj]; m2; m2 &= m2 - 1) {
                        const int y = wj * 32 + __ffs(m2) - 1;
                        if (y == x) continue;
                        const uint4 cy = chunk(y >> 3);
                        const uint32_t wy = (y & 7) < 2 ? cy.x : (y & 7) < 4 ? cy.y : (y & 7) < 6 ? cy.z : cy.w;
                        const float my = fabsf(__half2float(__ushort_as_half(static_cast<uint16_t>((y & 1) ? (wy >> 16) : (wy & 0xffffu)))));
                        const double ey = __dmul_rn(static_cast<double>(my), ad[y]);
                        rank += (ey > ex) || (ey == ex && y < x);
                    }
                }
                if (rank < need) keep[wi] |= 1u << (x & 31);
            }
        }
        q0 = keep[0];
        q1 = keep[1];
        q2 = keep[2];
        q3 = keep[3];
    }
    const uint32_t m0 = g0 | q0, m1 = g1 | q1, m2 = g2 | q2, m3 = g3 | q3;

    // g_t: both fp64 sums ascending in x; selected channels written ascending
    const int64_t slot = static_cast<int64_t>(u) * A.g_stride + t;
    uint8_t* out = A.cidx + slot * c;
    int k = 0;
    double tot = 0.0, drop = 0.0;
#pragma unroll 1
    for (int ch = 0; ch < 16; ++ch) {
        const uint4 q = chunk(ch);
        const uint32_t mw = (ch < 4) ? m0 : (ch < 8) ? m1 : (ch < 12) ? m2 : m3;
        const uint32_t qw[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const int x = ch * 8 + e;
            const uint16_t hb = static_cast<uint16_t>((e & 1) ? (qw[e >> 1] >> 16) : (qw[e >> 1] & 0xffffu));
            const double ex = __dmul_rn(static_cast<double>(fabsf(__half2float(__ushort_as_half(hb)))), ad[x]);
            tot = __dadd_rn(tot, ex);
            if ((mw >> (x & 31)) & 1u) out[k++] = static_cast<uint8_t>(x);
            else drop = __dadd_rn(drop, ex);
        }
    }
    const double gv = tot > 0.0 ? __ddiv_rn(drop, tot) : 0.0;
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
    ca.GW = L.shp.GW;
    ca.mtiles = L.shp.GWpad / 128;
    ca.apart = L.apart;
    ca.dbg_a = L.dbg_a;
    ca.g = L.g;
    ca.cidx = L.cidx;
    ca.g_stride = L.g_stride;
    ca.dbg_g = L.dbg_g;
    ca.dbg_stride = L.dbg_stride;
    ca.status = L.status;
    dim3 gc((L.max_nseg * L.shp.S + 127) / 128, units);
    if (gc.x > 0) {
        prof_begin(stream, kProfChan);
        if (L.shp.c <= 32) e = launch_k(chan_kernel_c32, gc, dim3(128), 0, stream, ca);
        else e = launch_k(chan_kernel_generic, gc, dim3(128), 0, stream, ca);
        if (e != cudaSuccess) return e;
        prof_end(stream, kProfChan);
    }
    return cudaGetLastError();
}

}  // namespace kv2d
