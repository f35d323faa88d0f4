// stage2.cu -- decode attention with decode-time token selection over the
// packed segments (sm_100a).
//
// MosaicKV ("MosaicKV: Serving Long-Context LLM with Dynamic Two-D KV Cache
// Compression", Fig. 6: stage 2 runs during the decode stage before each
// attention layer; Sec. 5.3: PackedAttention performs sequence compression
// and attention in every decode layer; Fig. 8: token selection rates of
// 6.25 % and 12.5 %) selects tokens per step with the current query.  The
// pages give no rule; this library reads it as:
//   - candidates: the tokens the unit's packed segments keep, slot j*S + i
//     for token i of segment j; the dense tail [comp_end, seq_len) is always
//     attended;
//   - score of a candidate: the largest over the unit's G query heads of the
//     logit scale * q_g . k (the stored key; kept channels only for CH /
//     BOTH), so one selection serves the heads that share the KV head;
//   - count: n_sel = min(candidates, ceil(rate * n_segs * S));
//   - the n_sel largest scores are kept, ties to the lower slot;
//   - attention over the kept candidates and the dense tail.
// Three kernels:
//   sel_score : one thread per candidate (a CTA scans its segments'
//               kept-token counts), G fp32 dot products with q from shared
//               memory, the maximum written per slot (-inf for empty slots);
//   sel_topn  : one CTA per unit, an exact radix select of the n_sel-th
//               largest score key (8-bit digits), the tied keys taken in
//               slot order by a block scan, the kept slots written ascending;
//   sel_attn  : the unit's items (kept slots, then tail tokens) cut into
//               equal chunks, one CTA per chunk; groups of 8 (G <= 4) or 16
//               lanes per item with lanes over d (16-byte key / value reads),
//               online softmax per head, fixed-order group, warp and chunk
//               merges (the last CTA of a unit, by atomic ticket, writes the
//               fp16 output).
#include <algorithm>

#include "kernels.h"

namespace kv2d {

namespace {

constexpr int kScoreThreads = 256;
constexpr int kTopThreads = 1024;
constexpr int kAttnWarps = 8;
constexpr float kNegInf2 = -__builtin_huge_valf();

struct Sel2Args {
    int Hkv, Hq, G, S, r, c;
    float scale, c2;
    double rate;
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
    int64_t slot_stride;   // slots per unit: (max_seq_len / S) * S, multiple of 4
    float* cscore;         // [units][slot_stride]: scores, compacted per region
    int32_t* cslot;        // [units][slot_stride]: the slot of each compacted score
    int32_t* ccount;       // [units][nreg_max]: candidates of each region
    int nreg_max;
    uint2* gather;         // [units][slot_stride]: kept items {desc low word, strategy | i << 8}
    int32_t* nsel;         // [units]
    float* part;           // [units][nchunk][G][4 + d]
    uint32_t* ticket;      // [units]
    int nchunk;
    float* dbg_score;      // optional [units][slot_stride]
    uint8_t* dbg_sel;      // optional [units][slot_stride]
    uint32_t* status;
};

__host__ __device__ inline int64_t seg_payload(int st, int S, int r, int c) {
    switch (st) {
    case KV2D_FULL: return 4ll * S * kHeadDim;
    case KV2D_TOK: return pad16(r) + 4ll * r * kHeadDim;
    case KV2D_CH: return pad16(static_cast<int64_t>(S) * c) + pad16(2ll * S * c) + 2ll * S * kHeadDim;
    default: return pad16(r) + pad16(static_cast<int64_t>(r) * c) + pad16(2ll * r * c) + 2ll * r * kHeadDim;
    }
}

// Segments a unit holds, clamped to the slot range; a value out of range
// sets KV2D_DEV_SEQ_RANGE (when report is set).
__device__ __forceinline__ int unit_segs(const Sel2Args& A, int u, bool report) {
    int n = A.n_segs[u];
    const int lim = static_cast<int>(min(static_cast<int64_t>(A.max_segs), A.slot_stride / A.S));
    if (n < 0 || n > lim) {
        if (report) set_status(A.status, KV2D_DEV_SEQ_RANGE);
        n = max(0, min(n, lim));
    }
    return n;
}

// Where candidate i of segment j of unit u lives.  kind 0: none (slot past
// the segment's kept tokens, or the segment's bytes outside the arena);
// 1: dense key row; 2: c (index, value) pairs.
struct Cand {
    int kind;
    const uint8_t* key;    // key row, or the index bytes
    const __half* kval;    // sparse key values
    const __half* vrow;    // value row
};

// The unit's packed bytes, clamped into its arena.
__device__ __forceinline__ int64_t unit_used(const Sel2Args& A, int u) {
    const int64_t U = A.used_bytes[u];
    return max(static_cast<int64_t>(0), min(U, A.arena_stride));
}

// Candidate i of the segment with descriptor d; U = the unit's used bytes.
__device__ __forceinline__ Cand candidate_of(const Sel2Args& A, int u, int64_t U, uint64_t d, int i, bool report) {
    Cand cd{0, nullptr, nullptr, nullptr};
    const int st = static_cast<int>((d >> 32) & 255u);
    const int64_t off = static_cast<int64_t>(d & 0xffffffffull) * 16;
    const int S = A.S, r = A.r, c = A.c;
    const bool tok = (st == KV2D_TOK || st == KV2D_BOTH);
    const int ntok = tok ? r : S;
    if (i >= ntok) return cd;
    if (st > KV2D_BOTH || off < 0 || off + seg_payload(st, S, r, c) > U) {
        if (report) set_status(A.status, KV2D_DEV_CAPACITY);
        return cd;
    }
    const uint8_t* sec = A.arena + static_cast<int64_t>(u) * A.arena_stride + off + (tok ? pad16(r) : 0);
    if (st == KV2D_FULL || st == KV2D_TOK) {
        cd.kind = 1;
        cd.key = sec + static_cast<int64_t>(i) * kHeadDim * 2;
        cd.vrow = reinterpret_cast<const __half*>(sec + static_cast<int64_t>(ntok + i) * kHeadDim * 2);
    } else {
        cd.kind = 2;
        cd.key = sec + static_cast<int64_t>(i) * c;
        cd.kval = reinterpret_cast<const __half*>(sec + pad16(static_cast<int64_t>(ntok) * c)) +
                  static_cast<int64_t>(i) * c;
        cd.vrow = reinterpret_cast<const __half*>(sec + pad16(static_cast<int64_t>(ntok) * c) +
                                                  pad16(2ll * ntok * c)) +
                  static_cast<int64_t>(i) * kHeadDim;
    }
    return cd;
}

__device__ __forceinline__ uint64_t seg_desc(const Sel2Args& A, int u, int j) {
    return A.desc[static_cast<int64_t>(u) * A.max_segs + j];
}

// ------------------------------------------------------------- scores

constexpr int kScoreSegs = 64;    // segments per region (one CTA of the score kernel)
constexpr int kQRow = kHeadDim + kHeadDim / 4;

// q rows padded by 4 floats per 16 dims, so that the 8 lanes of a group
// (16 dims each) read distinct bank groups.
__device__ __forceinline__ int qix(int x) { return x + 4 * (x >> 4); }

// One CTA per region of kScoreSegs segments of a unit.  The segments'
// kept-token counts are scanned in shared memory and the region's
// candidates numbered 0..n-1 in slot order; a group of 8 lanes takes one
// candidate (lane k: dims 16k .. 16k + 15, coalesced 32-byte reads of the
// key row, or every 8th (index, value) pair of a sparse key), the group's G
// dot products are summed by a butterfly, and the largest logit is written
// at the candidate's number in the region, with its slot beside it.
template <int G>
__global__ void __launch_bounds__(kScoreThreads) sel_score_kernel(const __grid_constant__ Sel2Args A) {
    pdl_wait();
    __shared__ __align__(16) float qs[G][kQRow];
    __shared__ int pre[kScoreSegs + 1];
    __shared__ uint64_t dsc[kScoreSegs];
    const int u = blockIdx.y;
    const int b = u / A.Hkv, h = u % A.Hkv;
    const int S = A.S;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int grp = lane >> 3, lg = lane & 7;
    const int nsg = unit_segs(A, u, blockIdx.x == 0 && tid == 0);
    const int j0 = blockIdx.x * kScoreSegs;
    if (j0 >= nsg) return;
    const int nj = min(kScoreSegs, nsg - j0);
    for (int x = tid; x < G * kHeadDim; x += kScoreThreads)
        qs[x / kHeadDim][qix(x % kHeadDim)] =
            __half2float(A.q[(static_cast<int64_t>(b) * A.Hq + h * G + x / kHeadDim) * kHeadDim + x % kHeadDim]);
    if (tid < 32) {
        // inclusive scan of the kept-token counts of the region's segments
        int carry = 0;
        for (int k0 = 0; k0 < kScoreSegs; k0 += 32) {
            const int j = j0 + k0 + lane;
            int n = 0;
            uint64_t d = 0;
            if (k0 + lane < nj) {
                d = seg_desc(A, u, j);
                const int st = static_cast<int>((d >> 32) & 255u);
                n = (st == KV2D_TOK || st == KV2D_BOTH) ? A.r : S;
            }
            int x = n;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, x, o);
                if (lane >= o) x += y;
            }
            if (k0 + lane < kScoreSegs) {
                dsc[k0 + lane] = d;
                pre[k0 + lane + 1] = carry + x;
            }
            carry += __shfl_sync(0xffffffffu, x, 31);
        }
        if (lane == 0) pre[0] = 0;
    }
    __syncthreads();
    const int ncand = pre[nj];
    const int64_t rbase = static_cast<int64_t>(u) * A.slot_stride + static_cast<int64_t>(j0) * S;
    if (tid == 0) A.ccount[static_cast<int64_t>(u) * A.nreg_max + blockIdx.x] = ncand;
    if (A.dbg_score) {
        // empty slots of the debug copy (indexed by slot)
        for (int x = tid; x < nj * S; x += kScoreThreads) {
            const int k = x / S, i = x % S;
            if (i >= pre[k + 1] - pre[k]) A.dbg_score[rbase + x] = kNegInf2;
        }
    }
    const int64_t U = unit_used(A, u);
    for (int cb = warp * 4; cb < ncand; cb += kScoreThreads / 8) {
        const int c = cb + grp;
        const bool on = c < ncand;
        int k = 0;
        if (on) {
            int lo = 0, hi = nj;             // the segment k with pre[k] <= c < pre[k + 1]
            while (hi - lo > 1) {
                const int mid = (lo + hi) >> 1;
                if (pre[mid] <= c) lo = mid;
                else hi = mid;
            }
            k = lo;
        }
        const int i = c - pre[k];
        const Cand cd = on ? candidate_of(A, u, U, dsc[k], i, lg == 0) : Cand{0, nullptr, nullptr, nullptr};
        float dot[G];
#pragma unroll
        for (int g = 0; g < G; ++g) dot[g] = 0.f;
        if (cd.kind == 1) {
            const uint4* kp = reinterpret_cast<const uint4*>(cd.key + lg * 32);
            const uint4 w0 = kp[0], w1 = kp[1];
            const uint32_t ws[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
            float kf[16];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&ws[e]));
                kf[2 * e] = f.x;
                kf[2 * e + 1] = f.y;
            }
#pragma unroll
            for (int g = 0; g < G; ++g) {
#pragma unroll
                for (int k4 = 0; k4 < 16; k4 += 4) {
                    const float4 q4 = *reinterpret_cast<const float4*>(&qs[g][qix(lg * 16 + k4)]);
                    dot[g] = fmaf(q4.w, kf[k4 + 3], fmaf(q4.z, kf[k4 + 2], fmaf(q4.y, kf[k4 + 1], fmaf(q4.x, kf[k4], dot[g]))));
                }
            }
        } else if (cd.kind == 2) {
            for (int x = lg; x < A.c; x += 8) {
                const int ci = cd.key[x] & 0x7f;      // indices are < 128; the mask keeps a bad byte in range
                const float kv = __half2float(cd.kval[x]);
#pragma unroll
                for (int g = 0; g < G; ++g) dot[g] = fmaf(qs[g][qix(ci)], kv, dot[g]);
            }
        }
#pragma unroll
        for (int g = 0; g < G; ++g)
#pragma unroll
            for (int off = 4; off > 0; off >>= 1) dot[g] += __shfl_xor_sync(0xffffffffu, dot[g], off);
        if (on && lg == 0) {
            float best = kNegInf2;
            if (cd.kind != 0) {
#pragma unroll
                for (int g = 0; g < G; ++g) best = fmaxf(best, A.scale * dot[g]);
            }
            const int slot = (j0 + k) * S + i;
            A.cscore[rbase + c] = best;
            A.cslot[rbase + c] = slot;
            if (A.dbg_score) A.dbg_score[static_cast<int64_t>(u) * A.slot_stride + slot] = best;
        }
    }
}

// ---------------------------------------------------------- selection

// Order-preserving key of a score: larger score, larger key; -inf (no
// candidate) is 0, every finite score is above it.
__device__ __forceinline__ uint32_t score_key(float s) {
    if (s == kNegInf2) return 0u;
    const uint32_t b = __float_as_uint(s);
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

__device__ __forceinline__ long long block_exscan_ll(long long v, long long* red, long long* total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    long long inc = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const long long n = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += n;
    }
    __syncthreads();
    if (lane == 31) red[warp] = inc;
    __syncthreads();
    if (warp == 0) {
        const long long w = (lane < (blockDim.x >> 5)) ? red[lane] : 0;
        long long wi = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const long long n = __shfl_up_sync(0xffffffffu, wi, o);
            if (lane >= o) wi += n;
        }
        red[lane] = wi - w;
        if (lane == 31) red[32] = wi;
    }
    __syncthreads();
    const long long res = red[warp] + inc - v;
    *total = red[32];
    __syncthreads();
    return res;
}

__global__ void __launch_bounds__(kTopThreads) sel_topn_kernel(const __grid_constant__ Sel2Args A) {
    pdl_wait();
    __shared__ unsigned int hist[256];
    __shared__ long long red[33];
    __shared__ uint32_t s_prefix;
    __shared__ long long s_need;
    extern __shared__ int rp[];            // [nreg + 1]: region prefix of candidate counts
    const int u = blockIdx.x;
    const int tid = threadIdx.x, lane = tid & 31;
    const int S = A.S;
    const int nsg = unit_segs(A, u, false);
    const int nreg = (nsg + kScoreSegs - 1) / kScoreSegs;
    const int64_t RS = static_cast<int64_t>(kScoreSegs) * S;
    const int64_t ubase = static_cast<int64_t>(u) * A.slot_stride;
    const float* sc = A.cscore + ubase;
    // region counts -> prefix (one block scan per 1024 regions)
    long long carry = 0;
    for (int k0 = 0; k0 < nreg; k0 += kTopThreads) {
        const int k = k0 + tid;
        const long long n = (k < nreg) ? A.ccount[static_cast<int64_t>(u) * A.nreg_max + k] : 0;
        long long tot;
        const long long ex = block_exscan_ll(n, red, &tot);
        if (k < nreg) rp[k] = static_cast<int>(carry + ex);
        carry += tot;
    }
    if (tid == 0) rp[nreg] = static_cast<int>(carry);
    __syncthreads();
    const long long ncand = carry;
    const double want = ceil(A.rate * static_cast<double>(static_cast<int64_t>(nsg) * S));
    const long long n_sel = (want >= static_cast<double>(ncand)) ? ncand : static_cast<long long>(want);
    // the n_sel-th largest key, 8 bits at a time from the top
    if (tid == 0) {
        s_prefix = 0u;
        s_need = n_sel;
    }
    __syncthreads();
    for (int pass = 0; pass < 4 && n_sel > 0; ++pass) {
        const int shift = 24 - 8 * pass;
        for (int i = tid; i < 256; i += kTopThreads) hist[i] = 0u;
        __syncthreads();
        const uint32_t pre = s_prefix;
        const uint32_t hmask = pass == 0 ? 0u : (0xffffffffu << (shift + 8));
        // region by region; lanes with the same digit add once (scores
        // cluster in few digits, so plain shared atomics would serialise)
        for (int k = 0; k < nreg; ++k) {
            const int cnt = rp[k + 1] - rp[k];
            const float* rs = sc + k * RS;
            for (int i0 = tid - lane; i0 < cnt; i0 += kTopThreads) {
                const int i = i0 + lane;
                const uint32_t key = (i < cnt) ? score_key(rs[i]) : 0u;
                const int dg = (key != 0u && (key & hmask) == (pre & hmask)) ? static_cast<int>((key >> shift) & 255u) : -1;
                const uint32_t peers = __match_any_sync(0xffffffffu, dg);
                if (dg >= 0 && lane == __ffs(peers) - 1) atomicAdd(&hist[dg], static_cast<unsigned>(__popc(peers)));
            }
        }
        __syncthreads();
        if (tid < 32) {
            // lane l owns digits 255 - 8l .. 248 - 8l (largest first)
            long long cnt = 0;
#pragma unroll
            for (int k = 0; k < 8; ++k) cnt += hist[255 - (8 * tid + k)];
            long long inc = cnt;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const long long n = __shfl_up_sync(0xffffffffu, inc, o);
                if (tid >= o) inc += n;
            }
            const long long need = s_need;
            long long above = inc - cnt;            // keys with larger digits
            int found = -1;
            long long above_found = 0;
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const int dg = 255 - (8 * tid + k);
                const long long hk = hist[dg];
                if (found < 0 && above + hk >= need) {
                    found = dg;
                    above_found = above;
                }
                above += hk;
            }
            const uint32_t bal = __ballot_sync(0xffffffffu, found >= 0);
            const int src = bal ? (__ffs(bal) - 1) : 0;
            const int dg = __shfl_sync(0xffffffffu, found, src);
            const long long ab = __shfl_sync(0xffffffffu, above_found, src);
            if (tid == 0 && bal) {
                s_prefix = pre | (static_cast<uint32_t>(dg) << shift);
                s_need = need - ab;
            }
        }
        __syncthreads();
    }
    const uint32_t v = s_prefix;            // the n_sel-th largest key (0: nothing kept)
    const long long eq_take = s_need;       // keys equal to v to keep, lowest slots first
    if (A.dbg_sel) {
        for (int64_t s = tid; s < static_cast<int64_t>(nsg) * S; s += kTopThreads) A.dbg_sel[ubase + s] = 0;
        __syncthreads();
    }
    // thread tid scans its own contiguous range of candidate numbers (flat
    // over the regions), so block scans give slot order
    const int64_t per = (ncand + kTopThreads - 1) / kTopThreads;
    const int64_t f0 = min(static_cast<int64_t>(ncand), per * tid), f1 = min(static_cast<int64_t>(ncand), f0 + per);
    auto region_of = [&](int64_t f) {
        int lo = 0, hi = nreg;
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (rp[mid] <= f) lo = mid;
            else hi = mid;
        }
        return lo;
    };
    long long n_gt = 0, n_eq = 0;
    {
        int k = (f0 < f1) ? region_of(f0) : 0;
        for (int64_t f = f0; f < f1; ++f) {
            while (f >= rp[k + 1]) ++k;
            const uint32_t key = score_key(sc[k * RS + (f - rp[k])]);
            n_gt += (n_sel > 0 && key > v);
            n_eq += (n_sel > 0 && key == v && key != 0u);
        }
    }
    long long tot_eq;
    const long long eq_before = block_exscan_ll(n_eq, red, &tot_eq);
    const long long mine = n_gt + max(0ll, min(n_eq, eq_take - eq_before));
    long long tot_sel;
    long long pos = block_exscan_ll(mine, red, &tot_sel);
    uint2* out = A.gather + ubase;
    long long eq_seen = eq_before;
    {
        int k = (f0 < f1) ? region_of(f0) : 0;
        for (int64_t f = f0; f < f1; ++f) {
            while (f >= rp[k + 1]) ++k;
            const int64_t at = k * RS + (f - rp[k]);
            const uint32_t key = score_key(sc[at]);
            bool keep = false;
            if (n_sel > 0 && key != 0u) {
                if (key > v) keep = true;
                else if (key == v) keep = (eq_seen++ < eq_take);
            }
            if (keep) {
                const int slot = A.cslot[ubase + at];
                const uint64_t d = seg_desc(A, u, slot / S);
                out[pos++] = make_uint2(static_cast<uint32_t>(d),
                                        static_cast<uint32_t>((d >> 32) & 255u) | (static_cast<uint32_t>(slot % S) << 8));
                if (A.dbg_sel) A.dbg_sel[ubase + slot] = 1;
            }
        }
    }
    if (tid == 0) {
        A.nsel[u] = static_cast<int32_t>(tot_sel);
        if (tot_sel != n_sel) set_status(A.status, KV2D_DEV_BAD_MASK);
    }
}

// ---------------------------------------------------------- attention

// A group of LPI lanes takes one item at a time (LPI = 8 for G <= 4, 16 for
// G = 8), so a warp has 32 / LPI items in flight; lane k of a group owns
// dimensions [k * 128 / LPI, (k + 1) * 128 / LPI).  The group's G logits are
// summed with a butterfly inside the group (fixed order), then each head's
// online softmax (log2 domain) updates the group's running max, sum and
// output slice.  Groups, then warps, then chunks merge in a fixed order.
template <int G>
__global__ void __launch_bounds__(kAttnWarps * 32, 2) sel_attn_kernel(const __grid_constant__ Sel2Args A) {
    pdl_wait();
    constexpr int LPI = (G <= 4) ? 8 : 16;       // lanes per item
    constexpr int DPL = kHeadDim / LPI;          // dims per lane (16 or 8)
    constexpr int IPW = 32 / LPI;                // items per warp in flight
    constexpr int kRec = kHeadDim + 4;
    __shared__ __align__(16) float qs[G][kQRow];
    __shared__ float wm[kAttnWarps][G], wl[kAttnWarps][G];
    __shared__ __align__(16) float wo[kAttnWarps][G][kHeadDim];
    __shared__ int is_last;
    const int c_id = blockIdx.x, u = blockIdx.y;
    const int b = u / A.Hkv, h = u % A.Hkv;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int grp = lane / LPI, lg = lane % LPI;
    for (int x = tid; x < G * kHeadDim; x += kAttnWarps * 32)
        qs[x / kHeadDim][qix(x % kHeadDim)] =
            __half2float(A.q[(static_cast<int64_t>(b) * A.Hq + h * G + x / kHeadDim) * kHeadDim + x % kHeadDim]);
    __syncthreads();
    // the unit's items: kept candidates, then its dense tail tokens
    const int cap = A.dv.block_table ? A.dv.max_blocks * A.dv.block_size : A.dv.capacity;
    int T = A.seq_len[b], ce = A.comp_end[b];
    if (T < 0 || T > cap || ce < 0 || ce > T) {
        if (tid == 0 && c_id == 0) set_status(A.status, KV2D_DEV_SEQ_RANGE);
        T = max(0, min(T, cap));
        ce = max(0, min(ce, T));
    }
    const int64_t nsel = A.nsel[u];
    const int64_t items = nsel + (T - ce);
    const int64_t i_lo = items * c_id / A.nchunk, i_hi = items * (c_id + 1) / A.nchunk;
    const uint2* gl = A.gather + static_cast<int64_t>(u) * A.slot_stride;
    const unsigned gmask = (LPI == 32) ? 0xffffffffu : (((1u << LPI) - 1u) << (grp * LPI));
    float m[G], l[G], o[G][DPL];
#pragma unroll
    for (int g = 0; g < G; ++g) {
        m[g] = kNegInf2;
        l[g] = 0.f;
#pragma unroll
        for (int e = 0; e < DPL; ++e) o[g][e] = 0.f;
    }
    const int d0 = lg * DPL;
    const int64_t U = unit_used(A, u);
    constexpr int64_t kStep = kAttnWarps * IPW;
    // the next item's gather entry is loaded while this one is computed
    int64_t it = i_lo + warp * IPW + grp;
    uint2 ge_n = (it < i_hi && it < nsel) ? gl[it] : make_uint2(0u, 0u);
    for (; it < i_hi; it += kStep) {
        const uint2 ge = ge_n;
        const int64_t it2 = it + kStep;
        if (it2 < i_hi && it2 < nsel) ge_n = gl[it2];
        float dot[G];
#pragma unroll
        for (int g = 0; g < G; ++g) dot[g] = 0.f;
        const __half* vrow = nullptr;
        const __half* krow = nullptr;
        bool skip = false;
        if (it < nsel) {
            const uint64_t dsc = static_cast<uint64_t>(ge.x) | (static_cast<uint64_t>(ge.y & 255u) << 32);
            const Cand cd = candidate_of(A, u, U, dsc, static_cast<int>(ge.y >> 8), lg == 0);
            if (cd.kind == 0) {
                skip = true;                 // (status already set; uniform in the group)
            } else {
                vrow = cd.vrow;
                if (cd.kind == 1) {
                    krow = reinterpret_cast<const __half*>(cd.key);
                } else {
                    for (int x = lg; x < A.c; x += LPI) {
                        const int ci = cd.key[x] & 0x7f;
                        const float kv = __half2float(cd.kval[x]);
#pragma unroll
                        for (int g = 0; g < G; ++g) dot[g] = fmaf(qs[g][qix(ci)], kv, dot[g]);
                    }
                }
            }
        } else {
            const int t = ce + static_cast<int>(it - nsel);
            krow = dense_row(A.dv, A.dv.k, b, h, t, lg == 0 ? A.status : nullptr);
            vrow = dense_row(A.dv, A.dv.v, b, h, t, nullptr);
            skip = !krow || !vrow;           // uniform in the group
        }
        if (skip) continue;
        uint4 vw[DPL / 8];
#pragma unroll
        for (int k = 0; k < DPL / 8; ++k) vw[k] = *reinterpret_cast<const uint4*>(vrow + d0 + 8 * k);
        if (krow) {
            float kf[DPL];
#pragma unroll
            for (int k = 0; k < DPL / 8; ++k) {
                const uint4 kw = *reinterpret_cast<const uint4*>(krow + d0 + 8 * k);
                const uint32_t ws[4] = {kw.x, kw.y, kw.z, kw.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&ws[e]));
                    kf[8 * k + 2 * e] = f.x;
                    kf[8 * k + 2 * e + 1] = f.y;
                }
            }
#pragma unroll
            for (int g = 0; g < G; ++g) {
#pragma unroll
                for (int k4 = 0; k4 < DPL; k4 += 4) {
                    const float4 q4 = *reinterpret_cast<const float4*>(&qs[g][qix(d0 + k4)]);
                    dot[g] = fmaf(q4.w, kf[k4 + 3], fmaf(q4.z, kf[k4 + 2], fmaf(q4.y, kf[k4 + 1], fmaf(q4.x, kf[k4], dot[g]))));
                }
            }
        }
        // the group's G logits (butterfly inside the group, fixed order)
#pragma unroll
        for (int g = 0; g < G; ++g)
#pragma unroll
            for (int off = LPI / 2; off > 0; off >>= 1) dot[g] += __shfl_xor_sync(gmask, dot[g], off, LPI);
        float vf[DPL];
#pragma unroll
        for (int k = 0; k < DPL / 8; ++k) {
            const uint32_t ws[4] = {vw[k].x, vw[k].y, vw[k].z, vw[k].w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&ws[e]));
                vf[8 * k + 2 * e] = f.x;
                vf[8 * k + 2 * e + 1] = f.y;
            }
        }
#pragma unroll
        for (int g = 0; g < G; ++g) {
            const float x = dot[g] * A.c2;
            const float mn = fmaxf(m[g], x);
            const float alpha = (m[g] == kNegInf2) ? 0.f : fast_exp2(m[g] - mn);
            const float p = fast_exp2(x - mn);
            m[g] = mn;
            l[g] = fmaf(l[g], alpha, p);
#pragma unroll
            for (int e = 0; e < DPL; ++e) o[g][e] = fmaf(o[g][e], alpha, p * vf[e]);
        }
    }
    // the warp's groups merged in order (butterfly over groups), then the
    // warps, then the chunks
#pragma unroll
    for (int off = LPI; off < 32; off <<= 1) {
#pragma unroll
        for (int g = 0; g < G; ++g) {
            const float m2 = __shfl_xor_sync(0xffffffffu, m[g], off);
            const float l2 = __shfl_xor_sync(0xffffffffu, l[g], off);
            const float M = fmaxf(m[g], m2);
            const float s1 = (m[g] == kNegInf2) ? 0.f : fast_exp2(m[g] - M);
            const float s2 = (m2 == kNegInf2) ? 0.f : fast_exp2(m2 - M);
            // the lower group's values first, whichever lane adds
            const bool low = (lane & off) == 0;
            const float sa = low ? s1 : s2, sb = low ? s2 : s1;
            const float la = low ? l[g] : l2, lb = low ? l2 : l[g];
            l[g] = fmaf(lb, sb, la * sa);
#pragma unroll
            for (int e = 0; e < DPL; ++e) {
                const float o2 = __shfl_xor_sync(0xffffffffu, o[g][e], off);
                const float oa = low ? o[g][e] : o2, ob = low ? o2 : o[g][e];
                o[g][e] = fmaf(ob, sb, oa * sa);
            }
            m[g] = M;
        }
    }
#pragma unroll
    for (int g = 0; g < G; ++g) {
        if (lane == 0) {
            wm[warp][g] = m[g];
            wl[warp][g] = l[g];
        }
        if (grp == 0) {
#pragma unroll
            for (int e = 0; e < DPL; e += 4)
                *reinterpret_cast<float4*>(&wo[warp][g][d0 + e]) = make_float4(o[g][e], o[g][e + 1], o[g][e + 2], o[g][e + 3]);
        }
    }
    __syncthreads();
    float* myp = A.part + (static_cast<int64_t>(u) * A.nchunk + c_id) * G * kRec;
    for (int x = tid; x < G * kHeadDim; x += kAttnWarps * 32) {
        const int g = x / kHeadDim, dd = x % kHeadDim;
        float M = kNegInf2;
#pragma unroll
        for (int w = 0; w < kAttnWarps; ++w) M = fmaxf(M, wm[w][g]);
        float O = 0.f, L = 0.f;
        if (M != kNegInf2) {
#pragma unroll
            for (int w = 0; w < kAttnWarps; ++w) {
                if (wm[w][g] == kNegInf2) continue;
                const float s = fast_exp2(wm[w][g] - M);
                O = fmaf(wo[w][g][dd], s, O);
                L = fmaf(wl[w][g], s, L);
            }
        }
        myp[g * kRec + 4 + dd] = O;
        if (dd == 0) {
            myp[g * kRec] = M;
            myp[g * kRec + 1] = L;
        }
    }
    __threadfence();
    __syncthreads();
    if (tid == 0) is_last = (atomicAdd(&A.ticket[u], 1u) == static_cast<uint32_t>(A.nchunk - 1));
    __syncthreads();
    if (!is_last) return;
    __threadfence();
    // the unit's chunks merged in order; a thread per (head, dim)
    const float* up = A.part + static_cast<int64_t>(u) * A.nchunk * G * kRec;
    for (int x = tid; x < G * kHeadDim; x += kAttnWarps * 32) {
        const int g = x / kHeadDim, dd = x % kHeadDim;
        float M = kNegInf2;
        for (int k = 0; k < A.nchunk; ++k) M = fmaxf(M, __ldcg(up + (static_cast<int64_t>(k) * G + g) * kRec));
        float O = 0.f, L = 0.f;
        if (M != kNegInf2) {
            for (int k = 0; k < A.nchunk; ++k) {
                const float* rec = up + (static_cast<int64_t>(k) * G + g) * kRec;
                const float mk = __ldcg(rec);
                if (mk == kNegInf2) continue;
                const float s = fast_exp2(mk - M);
                O = fmaf(__ldcg(rec + 4 + dd), s, O);
                L = fmaf(__ldcg(rec + 1), s, L);
            }
        }
        A.out[(static_cast<int64_t>(b) * A.Hq + h * G + g) * kHeadDim + dd] = __float2half_rn(L > 0.f ? O / L : 0.f);
    }
    if (tid == 0) A.ticket[u] = 0;
}

}  // namespace

int sel2_regions(int64_t slot_stride, int S) {
    return static_cast<int>((slot_stride / S + kScoreSegs - 1) / kScoreSegs);
}

int sel2_chunks(int units, int num_sms) {
    return std::max(1, std::min(kSel2MaxChunks, (2 * num_sms + units - 1) / units));
}

cudaError_t launch_decode_select(const DecodeSelectLaunch& L, cudaStream_t stream) {
    Sel2Args a;
    a.Hkv = L.shp.Hkv;
    a.Hq = L.shp.Hq;
    a.G = L.shp.G;
    a.S = L.shp.S;
    a.r = L.shp.r;
    a.c = L.shp.c;
    a.scale = L.scale;
    a.c2 = L.shp.c2;
    a.rate = L.rate;
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
    a.slot_stride = L.slot_stride;
    a.cscore = L.cscore;
    a.cslot = L.cslot;
    a.ccount = L.ccount;
    a.nreg_max = L.nreg_max;
    a.gather = L.gather;
    a.nsel = L.nsel;
    a.part = L.part;
    a.ticket = L.ticket;
    a.nchunk = L.nchunk;
    a.dbg_score = L.dbg_score;
    a.dbg_sel = L.dbg_sel;
    a.status = L.status;
    const int units = L.batch * L.shp.Hkv;
    cudaError_t e;
    prof_begin(stream, kProfSelScore);
    if (L.slot_stride > 0) {
        dim3 g1(static_cast<unsigned>(L.nreg_max), units);
        switch (L.shp.G) {
        case 1: e = launch_k(sel_score_kernel<1>, g1, dim3(kScoreThreads), 0, stream, a); break;
        case 2: e = launch_k(sel_score_kernel<2>, g1, dim3(kScoreThreads), 0, stream, a); break;
        case 4: e = launch_k(sel_score_kernel<4>, g1, dim3(kScoreThreads), 0, stream, a); break;
        case 8: e = launch_k(sel_score_kernel<8>, g1, dim3(kScoreThreads), 0, stream, a); break;
        default: return cudaErrorInvalidValue;
        }
        if (e != cudaSuccess) return e;
    }
    prof_end(stream, kProfSelScore);
    prof_begin(stream, kProfSelTop);
    e = launch_k(sel_topn_kernel, dim3(units), dim3(kTopThreads), (L.nreg_max + 1) * sizeof(int), stream, a);
    if (e != cudaSuccess) return e;
    prof_end(stream, kProfSelTop);
    prof_begin(stream, kProfSelAttn);
    dim3 g3(L.nchunk, units);
    switch (L.shp.G) {
    case 1: e = launch_k(sel_attn_kernel<1>, g3, dim3(kAttnWarps * 32), 0, stream, a); break;
    case 2: e = launch_k(sel_attn_kernel<2>, g3, dim3(kAttnWarps * 32), 0, stream, a); break;
    case 4: e = launch_k(sel_attn_kernel<4>, g3, dim3(kAttnWarps * 32), 0, stream, a); break;
    case 8: e = launch_k(sel_attn_kernel<8>, g3, dim3(kAttnWarps * 32), 0, stream, a); break;
    default: return cudaErrorInvalidValue;
    }
    if (e != cudaSuccess) return e;
    prof_end(stream, kProfSelAttn);
    return cudaGetLastError();
}

}  // namespace kv2d
