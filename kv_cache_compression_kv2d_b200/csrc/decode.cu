// decode.cu -- KV append and decode attention over the packed segments
// (sm_100a).
//
// MosaicKV ("MosaicKV: Serving Long-Context LLM with Dynamic Two-D KV Cache
// Compression", Sec. 5.3 PackedAttention and Fig. 6 packed sparse attention)
// runs decode attention directly on the compressed segments.  Here one unit
// (sequence b, KV head h) serves its G query heads from every byte it loads:
//   - a unit's work is its packed arena plus its dense tail
//     [comp_end, seq_len), 512 bytes per dense token; the units' byte
//     ranges, laid end to end over the batch, are cut into one equal share
//     per CTA (one CTA per SM), so every SM reads the same number of bytes
//     whatever the units' lengths; a CTA takes the segments whose first
//     byte falls in its share (counted on the descriptors) and the tail
//     tokens likewise, one unit after another when its share spans several;
//   - the CTA's range is cut into blocks of at most 8 tokens (a segment of
//     at most 8 tokens is one block); with W warps, warp w takes blocks w,
//     w + W, ... and runs q.k and p.v on the tensor cores (mma.sync
//     m16n8k16 / m16n8k8, fp16 in, fp32 accumulate; the G heads are the
//     rows of the tile);
//   - lane 0 of each warp has the TMA unit copy the bytes of its blocks
//     into a four-stage shared-memory ring (one bulk copy per contiguous
//     run, completion on a per-stage mbarrier), so a warp has three blocks
//     in flight while it computes a fourth; CH / BOTH keys are scattered
//     from their (index, value) pairs into a dense key tile;
//   - the per-block work is a chain of dependent steps (copy wait, q.k,
//     softmax shuffles, p.v), so the CTA runs 12 warps, three per
//     scheduler, to overlap the chains;
//   - scores meet an online softmax per head in the log2 domain; warps, then
//     the CTAs holding pieces of a unit, merge their (max, sum, output)
//     partials in a fixed order, the last CTA of a unit (atomic ticket)
//     writing the fp16 output.
#include "kernels.h"

namespace kv2d {

namespace {

constexpr int kDecWarps = 12;
constexpr int kDecThreads = kDecWarps * 32;
constexpr int kDecStages = 4;                       // stages per warp: 3 blocks in flight
// A stage holds one block of up to 8 tokens: 8 key rows, then 8 value rows,
// back to back.  Short blocks keep many stages in flight (12 warps x 3 x
// 4 KB per SM): the copy latency under load is microseconds, so the bytes in
// flight set the rate.  A quarter-warp's key reads meet 2 rows per bank
// group and its value reads 4.
constexpr int kDecRows = 8;
constexpr int kDecKStride = 256, kDecVStride = 256;
constexpr int kDecKBytes = kDecRows * kDecKStride;
constexpr int kDecSlotBytes = kDecKBytes + kDecRows * kDecVStride;
constexpr int kDecSmem = kDecWarps * kDecStages * kDecSlotBytes;
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
    int units;
    int kps;          // > 0: unit c / kps, piece c % kps of kps equal ones; 0: batch-wide shares
    int tbl_cap;      // blocks per table chunk (<= kTbl; >= 32, the most blocks of a segment)
    float* part;
    uint32_t* ticket;
    uint32_t* status;
};

constexpr int64_t kTailBytes = 2 * kHeadDim * 2;   // K + V row of one dense token

// The lengths of one unit, clamped into range (a value out of range sets
// KV2D_DEV_SEQ_RANGE when report is set): dense length T, compression end
// ce, segment count nsg, packed bytes U.
struct UnitLens {
    int T, ce, nsg;
    int64_t U;
};

__device__ __forceinline__ UnitLens unit_lens(const DecodeArgs& A, int u, bool report) {
    const int b = u / A.Hkv;
    UnitLens L;
    L.T = A.seq_len[b];
    L.ce = A.comp_end[b];
    L.nsg = A.n_segs[u];
    L.U = A.used_bytes[u];
    const int cap = A.dv.block_table ? A.dv.max_blocks * A.dv.block_size : A.dv.capacity;
    if (L.T < 0 || L.T > cap || L.ce < 0 || L.ce > L.T || L.nsg < 0 || L.nsg > A.max_segs || L.U < 0 ||
        L.U > A.arena_stride) {
        if (report) set_status(A.status, KV2D_DEV_SEQ_RANGE);
        L.T = max(0, min(L.T, cap));
        L.ce = max(0, min(L.ce, L.T));
        L.nsg = max(0, min(L.nsg, A.max_segs));
        L.U = max(static_cast<int64_t>(0), min(L.U, A.arena_stride));
    }
    return L;
}

// A unit's length in the batch-wide byte range the CTAs share: one byte that
// stands for the unit itself (so that every unit, even an empty one, has a
// CTA that writes its output), then its packed bytes, then 512 bytes per
// dense tail token.
__device__ __forceinline__ int64_t unit_span(const UnitLens& L) {
    return 1 + L.U + static_cast<int64_t>(L.T - L.ce) * kTailBytes;
}
constexpr int kDescRegs = 2048;                    // descriptors the counting pass holds in registers
constexpr int kTbl = kDecTableMax;                 // blocks in the block table (one chunk of a piece)

// ------------------------------------------------------ tensor-core decode
//
// Per warp, a block of up to 8 tokens goes through two mma.sync products
// (fp16 in, fp32 accumulate), lane (g = lane / 4, t = lane % 4):
//   S[16 x 8]  = Q[16 x 128] K^T      m16n8k16 x 8 (rows = the G query heads,
//                                     zero-padded; columns = the 8 tokens)
//   O^T[128 x 8] += V^T[128 x 8] P^T  m16n8k8 x 8 (rows = d, columns = the
//                                     heads; P^T is S's fragment as it lies)
// The q.k contraction runs over d in a fixed permuted order: mma k-index
// 2t+e of step ks <-> d = 8 (4 (ks / 2) + t) + 4 (ks % 2) + e and 2t+8+e <->
// the same + 2, so a lane's key data is the 16-byte chunks t, t+4, t+8, t+12
// of key row g.  In p.v, row g of tile i stands for d = 8g + i and row g + 8
// for d = 64 + 8g + i, so a lane's value data is chunks g and g + 8 of value
// rows 2t and 2t + 1, and its accumulators hold heads 2t and 2t + 1.

__device__ __forceinline__ void mma16816(float& d0, float& d1, uint32_t a0, uint32_t a2, uint32_t b0,
                                         uint32_t b1) {
    // rows 8..15 of the tile (accumulators 2, 3) are never used: they go to
    // scratch registers declared inside the asm
    asm volatile(
        "{\n\t.reg .f32 x2, x3;\n\t"
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, x2, x3}, {%2, %3, %4, %5}, "
        "{%6, %7}, {%8, %9, %10, %11};\n\t}"
        : "=f"(d0), "=f"(d1)
        : "r"(a0), "r"(0u), "r"(a2), "r"(0u), "r"(b0), "r"(b1), "f"(d0), "f"(d1), "f"(0.f), "f"(0.f));
}

// m16n8k8, all four accumulators live: D[16 x 8] += A[16 x 8] B[8 x 8].
__device__ __forceinline__ void mma16808(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t b0) {
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5}, {%6}, "
        "{%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(b0));
}

struct MmaState {
    float m;          // running max of this lane's head row g (log2 domain)
    float lp;         // this lane's share of that row's softmax sum
    float o[8][4];    // O[head 2t + (e & 1)][d = 8g + i + 64 (e >> 1)] at o[i][e]
};

__device__ __forceinline__ uint4 ld_nc16(const void* p) {
    return *reinterpret_cast<const uint4*>(p);
}

// One block of up to 8 token rows, n of them valid.  kw[i]: chunk 4i + t of
// key row g; vw[k][i]: chunk g + 8i of value row 2t + k.
//
// The running max moves only when a block max exceeds it by more than 8 (in
// log2 units), so the fp16 numerators stay <= 2^8 and most blocks skip the
// rescale of O; every partial carries the max it was scaled by.
__device__ __forceinline__ void mma_block(MmaState& st, const uint32_t (&qa)[8][2], const uint4 (&kw)[4],
                                          const uint4 (&vw)[2][2], int n, float c2) {
    const int lane = threadIdx.x & 31;
    const int t = lane & 3;
    // two accumulation chains (even and odd k-steps) halve the dependent
    // MMA latency
    float s0 = 0.f, s1 = 0.f, u0 = 0.f, u1 = 0.f;
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
        const uint4& w = kw[ks >> 1];
        const uint32_t b0 = (ks & 1) ? w.z : w.x;
        const uint32_t b1 = (ks & 1) ? w.w : w.y;
        if (ks & 1)
            mma16816(u0, u1, qa[ks][0], qa[ks][1], b0, b1);
        else
            mma16816(s0, s1, qa[ks][0], qa[ks][1], b0, b1);
    }
    s0 += u0;
    s1 += u1;
    // scores of tokens 2t, 2t + 1 of head row g, online softmax over the row
    const bool ok0 = 2 * t < n, ok1 = 2 * t + 1 < n;
    const float x0 = ok0 ? s0 * c2 : kNegInfF;
    const float x1 = ok1 ? s1 * c2 : kNegInfF;
    float bm = fmaxf(x0, x1);
    bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 1));
    bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 2));
    const bool move = bm > st.m + 8.f;               // st.m = -inf: any finite bm moves
    const float mn = move ? bm : st.m;
    const float alpha = move ? ((st.m == kNegInfF) ? 0.f : fast_exp2(st.m - mn)) : 1.f;
    st.m = mn;
    const float p0 = ok0 ? fast_exp2(x0 - mn) : 0.f;
    const float p1 = ok1 ? fast_exp2(x1 - mn) : 0.f;
    st.lp = st.lp * alpha + (p0 + p1);
    if (__any_sync(0xffffffffu, alpha != 1.f)) {
        // this lane's accumulators belong to heads 2t and 2t + 1, whose
        // factors sit in lanes 4 (2t) and 4 (2t + 1)
        const float a_lo = __shfl_sync(0xffffffffu, alpha, 8 * t);
        const float a_hi = __shfl_sync(0xffffffffu, alpha, 8 * t + 4);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            st.o[i][0] *= a_lo;
            st.o[i][1] *= a_hi;
            st.o[i][2] *= a_lo;
            st.o[i][3] *= a_hi;
        }
    }
    const __half2 pp = __floats2half2_rn(p0, p1);
    const uint32_t b0 = *reinterpret_cast<const uint32_t*>(&pp);
    // element i of chunk window ci of value rows 2t, 2t + 1, packed in pairs
    auto afrag = [&](int i, int ci) {
        const int wi = i >> 1;
        const uint32_t sel = (i & 1) ? 0x7632u : 0x5410u;
        auto word = [&](const uint4& q4) {
            return wi == 0 ? q4.x : wi == 1 ? q4.y : wi == 2 ? q4.z : q4.w;
        };
        return __byte_perm(word(vw[0][ci]), word(vw[1][ci]), sel);
    };
#pragma unroll
    for (int i = 0; i < 8; ++i) mma16808(st.o[i], afrag(i, 0), afrag(i, 1), b0);
}

// Contiguous global -> shared copy by the TMA unit (no tensor map, no
// multicast); 16-byte aligned addresses, size a multiple of 16; completion
// counted in bytes on the mbarrier.
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
                 "l"(src), "r"(bytes), "r"(bar)
                 : "memory");
}

// A block of up to 8 tokens of one warp.  kind & 3: 0 none, 1 dense rows
// (FULL / TOK segment or tail), 2 channel-sparse keys (CH / BOTH); kind & 4:
// the block is a whole segment whose sections are contiguous in the arena
// and arrive in one copy (dense: key rows, then value rows right after
// them; sparse: index bytes and key values end where the value rows start).
constexpr int kBlkOne = 4;
struct DecBlock {
    int kind, nlo;
    const uint8_t* ci;      // sparse: the block's index bytes
    int dkv;                // sparse: its key values start at ci + dkv
};

constexpr int kDescPerThread = kDescRegs / kDecThreads;   // descriptors each thread loads in the prologue

template <int G>
__global__ void __launch_bounds__(kDecThreads, 1) decode_kernel(const __grid_constant__ DecodeArgs A) {
    extern __shared__ __align__(16) uint8_t dec_smem[];
    const int cta = blockIdx.x, ncta = gridDim.x;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, t = lane & 3;
    __shared__ float wm[kDecWarps][G], wl[kDecWarps][G];
    __shared__ int wcnt[kDecWarps][2];
    __shared__ long long wsum[kDecWarps];
    __shared__ long long s_part[3];   // first unit, its start, last unit
    __shared__ __align__(8) uint64_t sbar[kDecWarps][kDecStages];
    __shared__ int is_last;
    // block table: entry i = descriptor of the segment holding block i of
    // the chunk, with the block's first token (segment-relative) in bits 40..55
    __shared__ uint64_t tbl[kTbl];
    // the warp partials reuse the stage buffers once every warp is done
    static_assert(sizeof(float) * kDecWarps * G * kHeadDim <= kDecSmem, "partials fit");

    float (*wo)[G][kHeadDim] = reinterpret_cast<float (*)[G][kHeadDim]>(dec_smem);

    pdl_wait();
    // ---- the batch-wide partition: the units' spans laid end to end, CTA c
    // takes bytes [lo_c, lo_{c+1}) with lo_c = floor(Wtot c / n) and works
    // on every unit from the one holding byte lo_c to the one holding byte
    // max(lo_c, lo_{c+1} - 1) (a "piece" of each); a segment or tail token
    // belongs to the CTA that holds its first byte.  A CTA whose range is
    // empty (fewer bytes than CTAs) still takes the unit holding lo_c, with
    // no work, so that the pieces of a unit are consecutive CTAs.
    const int units = A.units, kps = A.kps;
    long long Wtot = 0, GL = 0, GH = 0;
    if (kps == 0) {
        long long mine = 0;
        for (int u = tid; u < units; u += kDecThreads) mine += unit_span(unit_lens(A, u, false));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mine += __shfl_xor_sync(0xffffffffu, mine, o);
        if (lane == 0) wsum[warp] = mine;
        __syncthreads();
#pragma unroll
        for (int w = 0; w < kDecWarps; ++w) Wtot += wsum[w];
        GL = Wtot * cta / ncta;
        GH = Wtot * (cta + 1) / ncta;
        const long long Gend = GH > GL ? GH - 1 : GL;   // the last byte the CTA looks at
        long long base = 0;   // span of the units before the chunk
        for (int c0 = 0; c0 < units && base <= Gend; c0 += kDecThreads) {
            const int u = c0 + tid;
            const long long w = (u < units) ? unit_span(unit_lens(A, u, false)) : 0;
            long long x = w;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const long long y = __shfl_up_sync(0xffffffffu, x, o);
                if (lane >= o) x += y;
            }
            __syncthreads();   // wsum is free again
            if (lane == 31) wsum[warp] = x;
            __syncthreads();
            long long before = base, chunk = 0;
#pragma unroll
            for (int w2 = 0; w2 < kDecWarps; ++w2) {
                if (w2 < warp) before += wsum[w2];
                chunk += wsum[w2];
            }
            const long long incl = before + x, excl = incl - w;
            if (u < units && excl <= GL && GL < incl) {
                s_part[0] = u;
                s_part[1] = excl;
            }
            if (u < units && excl <= Gend && Gend < incl) s_part[2] = u;
            base += chunk;
        }
    } else if (tid == 0) {
        // few units: kps CTAs each, so that no CTA pays a second piece's
        // fixed costs (lengths, descriptors, merges)
        s_part[0] = s_part[2] = cta / kps;
        s_part[1] = 0;
    }
    if (tid < kDecWarps * kDecStages) {
        mbar_init(&sbar[tid / kDecStages][tid % kDecStages], 1);
        mbar_fence_init();
    }
    // value rows past a block's last token must hold finite numbers; the
    // copy engine writes these buffers next
    for (int i = tid; i < kDecSmem / 16; i += kDecThreads)
        reinterpret_cast<uint4*>(dec_smem)[i] = make_uint4(0, 0, 0, 0);
    fence_proxy_async();
    __syncthreads();
    const int u_first = static_cast<int>(s_part[0]), u_last = static_cast<int>(s_part[2]);
    long long P = s_part[1];   // start of the current unit's span
    // the last CTA c with lo_c <= x, and the first CTA c with lo_c >= x
    auto cta_at = [&](long long x) { return static_cast<int>(((x + 1) * ncta - 1) / Wtot); };
    auto cta_from = [&](long long x) { return static_cast<int>((x * ncta + Wtot - 1) / Wtot); };

    const float c2 = A.c2;
    const int S = A.S, r = A.r, c = A.c;
    const bool c8 = c <= 32 && (c & 7) == 0;       // the sparse fast path
    const int row8 = c8 ? (lane * 8) / c : 0;      // its key row for this lane
    const uint32_t wbase = smem_u32(dec_smem) + warp * (kDecStages * kDecSlotBytes);
    // stage s of this warp: key rows at kreg(s), value rows at kreg(s) +
    // kDecKBytes (see DecBlock for the one-copy layouts)
    auto kreg = [&](int stage) -> uint32_t { return wbase + stage * kDecSlotBytes; };
    const uint32_t bar0 = smem_u32(&sbar[warp][0]);
    auto lds16 = [&](uint32_t a) {
        uint4 v;
        asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                     : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                     : "r"(a));
        return v;
    };
    auto seg_ntok = [&](uint64_t d) {
        const int sty = static_cast<int>((d >> 32) & 255u);
        return (sty == KV2D_TOK || sty == KV2D_BOTH) ? r : S;
    };
    auto seg_dense = [&](uint64_t d) {
        const int sty = static_cast<int>((d >> 32) & 255u);
        return sty == KV2D_FULL || sty == KV2D_TOK;
    };
    // blocks this warp has consumed so far: block k of the warp uses stage
    // k % kDecStages and that stage's (k / kDecStages)-th barrier phase
    int kbase = 0;
    bool dead = false;   // a copy wait gave up: no more copies from this warp

    for (int u = u_first; u <= u_last; ++u) {
    const int b = u / A.Hkv, h = u % A.Hkv;
    // q fragments (rows g < G): chunk 4 (ks / 2) + t of head g, words of step ks
    uint32_t qa[8][2];
    {
        uint4 qw[4] = {make_uint4(0, 0, 0, 0), make_uint4(0, 0, 0, 0), make_uint4(0, 0, 0, 0),
                       make_uint4(0, 0, 0, 0)};
        if (g < G) {
            const __half* qrow = A.q + (static_cast<int64_t>(b) * A.Hq + h * G + g) * kHeadDim;
#pragma unroll
            for (int i = 0; i < 4; ++i) qw[i] = ld_nc16(qrow + 8 * (4 * i + t));
        }
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
            const uint4& w = qw[ks >> 1];
            qa[ks][0] = (ks & 1) ? w.z : w.x;
            qa[ks][1] = (ks & 1) ? w.w : w.y;
        }
    }
    // ---- one round trip: q, the unit's lengths and its first descriptors
    const uint64_t* D = A.desc + static_cast<int64_t>(u) * A.max_segs;
    const UnitLens Ln = unit_lens(A, u, tid == 0);
    const int T = Ln.T, ce = Ln.ce, nsg = Ln.nsg;
    const int64_t U = Ln.U;
    uint64_t dreg[kDescPerThread];
#pragma unroll
    for (int k = 0; k < kDescPerThread; ++k) {
        const int j = tid + k * kDecThreads;
        dreg[k] = (j < A.max_segs) ? D[j] : 0ull;
    }
    const int ntail = T - ce;
    // this CTA's piece of the unit, as offsets into its packed bytes and
    // tail (byte x of the unit is byte P + 1 + x of the batch-wide range)
    const long long span = unit_span(Ln);
    int64_t lo, hi;
    int first, last;   // the pieces of the unit are CTAs first .. last
    if (kps > 0) {
        const int sp = cta - u * kps;
        lo = span * sp / kps - 1;
        hi = span * (sp + 1) / kps - 1;
        first = u * kps;
        last = first + kps - 1;
    } else {
        lo = GL - P - 1;
        hi = GH - P - 1;
        // first: the first CTA whose last byte (first byte when it has none)
        // reaches P
        first = min(cta_from(P), cta_from(P + 1) - 1);
        last = cta_at(P + span - 1);
        P += span;
    }
    // segments whose first byte lies in [lo, hi)
    {
        int c_lo = 0, c_hi = 0;
#pragma unroll
        for (int k = 0; k < kDescPerThread; ++k) {
            const int j = tid + k * kDecThreads;
            if (j < nsg) {
                const int64_t off = static_cast<int64_t>(dreg[k] & 0xffffffffull) * 16;
                c_lo += off < lo;
                c_hi += off < hi;
            }
        }
        for (int j = tid + kDescPerThread * kDecThreads; j < nsg; j += kDecThreads) {
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
            wcnt[warp][0] = c_lo;
            wcnt[warp][1] = c_hi;
        }
    }
    __syncthreads();
    int j_lo = 0, j_hi = 0;
#pragma unroll
    for (int w = 0; w < kDecWarps; ++w) {
        j_lo += wcnt[w][0];
        j_hi += wcnt[w][1];
    }
    auto tail_at_or_after = [&](int64_t x) -> int {
        if (x <= U) return 0;
        const int64_t i = (x - U + kTailBytes - 1) / kTailBytes;
        return static_cast<int>(i < ntail ? i : static_cast<int64_t>(ntail));
    };
    const int t_lo = ce + tail_at_or_after(lo), t_hi = ce + tail_at_or_after(hi);
    const int ntb = (t_hi - t_lo + kDecRows - 1) / kDecRows;

    MmaState st;
    st.m = kNegInfF;
    st.lp = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int e = 0; e < 4; ++e) st.o[i][e] = 0.f;
    const uint8_t* ubase = A.arena + static_cast<int64_t>(u) * A.arena_stride;
    // first K row of a dense segment (its V rows follow its ntok K rows)
    auto seg_k = [&](uint64_t d) {
        const int sty = static_cast<int>((d >> 32) & 255u);
        return reinterpret_cast<const __half*>(ubase + static_cast<int64_t>(d & 0xffffffffull) * 16 +
                                               (sty == KV2D_TOK ? pad16(r) : 0));
    };

    // ---- the CTA's items, in order: every segment in blocks of up to 8
    // tokens, then the dense tail in blocks of 8.  Item i of a chunk belongs
    // to warp i % kDecWarps, so the order of every sum is fixed and the
    // output is deterministic.  The segments go through the block table in
    // chunks of whole segments (one chunk unless a piece has more than kTbl
    // blocks); a warp finds its block with one shared-memory load.
    int seg_next = j_lo;   // first segment not tabled yet
    for (bool last_chunk = false; !last_chunk;) {
    int n_tab = 0;         // blocks in the table
    {
        __shared__ int s_cut[2];
        if (tid == 0) s_cut[0] = -1;
        // chunks of kDecThreads segments aligned like the counting pass, so
        // that the descriptors it left in registers serve again
        for (int c0 = seg_next / kDecThreads * kDecThreads; c0 < j_hi; c0 += kDecThreads) {
            const int j = c0 + tid;
            const bool in = j >= seg_next && j < j_hi;
            uint64_t d = 0;
            if (in) {
                const int kk = c0 / kDecThreads;
                if (kk < kDescPerThread) {
#pragma unroll
                    for (int k = 0; k < kDescPerThread; ++k)
                        if (k == kk) d = dreg[k];
                } else {
                    d = D[j];
                }
            }
            const int nit = in ? (seg_ntok(d) + kDecRows - 1) / kDecRows : 0;
            int x = nit;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, x, o);
                if (lane >= o) x += y;
            }
            __syncthreads();   // wcnt is free
            if (lane == 31) wcnt[warp][0] = x;
            __syncthreads();
            int pos = n_tab + x - nit, tot = 0;
#pragma unroll
            for (int w2 = 0; w2 < kDecWarps; ++w2) {
                if (w2 < warp) pos += wcnt[w2][0];
                tot += wcnt[w2][0];
            }
            if (in) {
                if (pos + nit <= A.tbl_cap) {
                    for (int q = 0; q < nit; ++q) tbl[pos + q] = d | (static_cast<uint64_t>(q * kDecRows) << 40);
                } else if (pos <= A.tbl_cap) {   // the first segment that does not fit
                    s_cut[0] = pos;
                    s_cut[1] = j;
                }
            }
            __syncthreads();
            if (s_cut[0] >= 0) {
                n_tab = s_cut[0];
                seg_next = s_cut[1];
                break;
            }
            n_tab += tot;
            seg_next = min(c0 + kDecThreads, j_hi);
        }
        last_chunk = seg_next >= j_hi;
        __syncthreads();   // the table is complete
    }
    int g_next = warp;
    auto next_block = [&](int stage) -> DecBlock {
        DecBlock bk{0, 0, nullptr, 0};
        const int g_idx = g_next;
        g_next += kDecWarps;
        const __half* kh = nullptr;   // first K row of the block
        const __half* vh = nullptr;   // first V row of the block
        const __half* kv = nullptr;   // sparse: first key value of the block
        int n = 0;
        bool tail = false;
        uint64_t d = 0;
        int t0 = 0;
        if (g_idx < n_tab) {
            d = tbl[g_idx];
            t0 = static_cast<int>((d >> 40) & 0xffffu);
            d &= 0xffffffffffull;
            const int ntok = seg_ntok(d);
            n = min(kDecRows, ntok - t0);
            const int one = (ntok <= kDecRows) ? kBlkOne : 0;
            if (seg_dense(d)) {
                bk.kind = 1 | one;
                kh = seg_k(d) + static_cast<int64_t>(t0) * kHeadDim;
                vh = seg_k(d) + static_cast<int64_t>(ntok + t0) * kHeadDim;
            } else {
                bk.kind = 2 | (c <= 32 ? one : 0);
                const bool tok = ((d >> 32) & 255u) == KV2D_BOTH;
                const uint8_t* p0 = ubase + static_cast<int64_t>(d & 0xffffffffull) * 16 + (tok ? pad16(r) : 0);
                bk.ci = p0 + static_cast<int64_t>(t0) * c;
                kv = reinterpret_cast<const __half*>(p0 + pad16(static_cast<int64_t>(ntok) * c)) +
                     static_cast<int64_t>(t0) * c;
                bk.dkv = static_cast<int>(reinterpret_cast<const uint8_t*>(kv) - bk.ci);
                vh = reinterpret_cast<const __half*>(p0 + pad16(static_cast<int64_t>(ntok) * c) +
                                                     pad16(static_cast<int64_t>(ntok) * c * 2)) +
                     static_cast<int64_t>(t0) * kHeadDim;
            }
        } else if (last_chunk) {
            const int tb = g_idx - n_tab;
            if (tb < ntb) {
                bk.kind = 1;
                tail = true;
                t0 = t_lo + tb * kDecRows;
                n = min(kDecRows, t_hi - t0);
            }
        }
        bk.nlo = n;
        // Copies by the TMA unit.  Segment blocks: lane 0 copies a whole
        // short segment in one piece, else the block's key rows and value
        // rows (or a sparse block's two pair sections and its value rows) in
        // one piece each; the dense tail, whose rows need not be contiguous,
        // is copied row by row (lane l < 8: value row l, lane 16 + l: key
        // row l).
        if (bk.kind != 0) {
            const uint32_t K0 = kreg(stage), V0 = K0 + kDecKBytes, bar = bar0 + stage * 8;
            if (!tail) {
                if (lane == 0) {
                    const int kd = bk.kind & 3;
                    int npb = 0, nkb = 0;
                    if (kd == 2 && c <= 32) {
                        npb = pad16(n * c);
                        nkb = pad16(2 * n * c);
                    }
                    const uint32_t bytes = n * 256 * (kd == 1 ? 2 : 1) + npb + nkb;
                    mbar_expect_tx(&sbar[warp][stage], bytes);
                    if (bk.kind == (1 | kBlkOne)) {
                        bulk_g2s(K0, kh, bytes, bar);
                    } else if (bk.kind == (2 | kBlkOne)) {
                        bulk_g2s(V0 - npb - nkb, bk.ci, bytes, bar);
                    } else {
                        if (kd == 1) bulk_g2s(K0, kh, n * 256, bar);
                        bulk_g2s(V0, vh, n * 256, bar);
                        if (npb) {
                            bulk_g2s(K0, bk.ci, npb, bar);
                            bulk_g2s(K0 + 512, kv, nkb, bar);
                        }
                    }
                }
            } else {
                const int R = lane & 15;
                const bool krow_lane = lane >= 16;
                const __half* row = (R < n) ? dense_row(A.dv, krow_lane ? A.dv.k : A.dv.v, b, h, t0 + R, A.status)
                                            : nullptr;
                const uint32_t nrows = __popc(__ballot_sync(0xffffffffu, row != nullptr));
                if (lane == 0) mbar_expect_tx(&sbar[warp][stage], nrows * 256);
                __syncwarp();
                if (row) bulk_g2s(krow_lane ? K0 + R * kDecKStride : V0 + R * kDecVStride, row, 256, bar);
            }
        }
        return bk;
    };

    auto compute = [&](const DecBlock& bk, int stage) {
        const int kd = bk.kind & 3;
        const bool one = bk.kind & kBlkOne;
        const uint32_t K0 = kreg(stage);
        const uint32_t V0 = K0 + ((one && kd == 1) ? bk.nlo * 256 : kDecKBytes);
        if (kd == 2 && c8) {
            // c <= 32, a multiple of 8: lane l takes pairs 8l .. 8l + 7, all
            // in key row 8l / c; zero the 8 x 128 key tile, then scatter
            const int np = bk.nlo * c;
            const bool act = lane * 8 < np;
            uint2 iw = make_uint2(0, 0);
            uint4 va = make_uint4(0, 0, 0, 0);
            if (act) {
                const uint32_t nkb = one ? pad16(2 * np) : 0;
                const uint32_t P0 = one ? V0 - nkb - pad16(np) : K0;
                const uint32_t Q0 = one ? V0 - nkb : K0 + 512;
                asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(iw.x), "=r"(iw.y) : "r"(P0 + lane * 8));
                va = lds16(Q0 + lane * 16);
            }
            __syncwarp();
#pragma unroll
            for (int i = 0; i < kDecRows / 2; ++i)
                asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(K0 + (2 * i + (lane >> 4)) * kDecKStride +
                                                                             (lane & 15) * 16),
                             "r"(0u)
                             : "memory");
            __syncwarp();
            if (act) {
                const uint32_t row = K0 + row8 * kDecKStride;
                const uint32_t vws[4] = {va.x, va.y, va.z, va.w};
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    // indices are < 128; the mask keeps a corrupt byte inside the tile
                    const int ch = (((k < 4) ? iw.x : iw.y) >> (8 * (k & 3))) & 0x7f;
                    const uint16_t hv = static_cast<uint16_t>(vws[k >> 1] >> (16 * (k & 1)));
                    asm volatile("st.shared.u16 [%0], %1;" ::"r"(row + ch * 2), "h"(hv) : "memory");
                }
            }
            __syncwarp();
        } else if (kd == 2) {
            // the 8 x 128 key tile: zero it, then scatter the block's n * c
            // pairs into it; 16 pairs per lane and round
            const int np = bk.nlo * c;
            uint4 iw = make_uint4(0, 0, 0, 0), va = iw, vb = iw;
            if (c <= 32 && lane * 16 < np) {
                const uint32_t nkb = one ? pad16(2 * np) : 0;
                const uint32_t P0 = one ? V0 - nkb - pad16(np) : K0;
                const uint32_t Q0 = one ? V0 - nkb : K0 + 512;
                iw = lds16(P0 + lane * 16);
                va = lds16(Q0 + lane * 32);
                vb = lds16(Q0 + lane * 32 + 16);
            }
            __syncwarp();
#pragma unroll
            for (int i = 0; i < kDecRows / 2; ++i)
                asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(K0 + (2 * i + (lane >> 4)) * kDecKStride +
                                                                             (lane & 15) * 16),
                             "r"(0u)
                             : "memory");
            __syncwarp();
            for (int e0 = lane * 16; e0 < np; e0 += 32 * 16) {
                if (c > 32) {
                    iw = ld_nc16(bk.ci + e0);
                    const __half* kv = reinterpret_cast<const __half*>(bk.ci + bk.dkv);
                    va = ld_nc16(kv + e0);
                    vb = ld_nc16(kv + e0 + 8);
                }
                const uint32_t iws[4] = {iw.x, iw.y, iw.z, iw.w};
                const uint32_t vws[8] = {va.x, va.y, va.z, va.w, vb.x, vb.y, vb.z, vb.w};
                int rr = e0 / c, col = e0 - rr * c;
#pragma unroll
                for (int k = 0; k < 16; ++k) {
                    if (e0 + k < np) {
                        // indices are < 128; the mask keeps a corrupt byte inside the tile
                        const int ch = (iws[k >> 2] >> (8 * (k & 3))) & 0x7f;
                        const uint16_t hv = static_cast<uint16_t>(vws[k >> 1] >> (16 * (k & 1)));
                        asm volatile("st.shared.u16 [%0], %1;" ::"r"(K0 + rr * kDecKStride + ch * 2), "h"(hv) : "memory");
                    }
                    if (++col == c) {
                        col = 0;
                        ++rr;
                    }
                }
            }
            __syncwarp();
        }
        // key row g, value rows 2t and 2t + 1
        uint4 kw[4], vw[2][2];
#pragma unroll
        for (int i = 0; i < 4; ++i) kw[i] = lds16(K0 + g * kDecKStride + (4 * i + t) * 16);
#pragma unroll
        for (int k = 0; k < 2; ++k)
#pragma unroll
            for (int i = 0; i < 2; ++i) vw[k][i] = lds16(V0 + (2 * t + k) * kDecVStride + (g + 8 * i) * 16);
        mma_block(st, qa, kw, vw, bk.nlo, c2);
        // the stage is refilled next by the copy engine: after a scatter
        // (plain stores into the key rows) every writer orders its stores
        // before those copies; plain reads need no fence
        if (kd == 2) fence_proxy_async();
        __syncwarp();
    };

    {
        // the first kDecStages - 1 iterations only issue; block k is issued at
        // iteration k - (kDecStages - 1) into stage k % kDecStages and
        // computed at iteration k, after the stage's barrier completes its
        // (k / kDecStages)-th phase; f[j] holds block k + j
        constexpr int kAhead = kDecStages - 1;
        DecBlock f[kAhead];
#pragma unroll
        for (int j = 0; j < kAhead; ++j) f[j] = DecBlock{0, 0, nullptr, 0};
        for (int k = kbase - kAhead; !dead; ++k) {
            const DecBlock nb = next_block((k + kAhead) % kDecStages);
            if (k >= kbase) {
                if (f[0].kind == 0) {
                    kbase = k;   // every block after it is empty too: no copy in flight
                    break;
                }
                if (!mbar_wait(&sbar[warp][k % kDecStages], (k / kDecStages) & 1, A.status)) {
                    // give the copies this warp has in flight (blocks k + 1
                    // .. k + kAhead) one more bounded wait each before the
                    // stage buffers are reused; the outputs are undefined
                    // from here on (the status bit says so)
#pragma unroll
                    for (int j = 1; j <= kAhead; ++j) {
                        const DecBlock& fb = (j < kAhead) ? f[j] : nb;
                        if (fb.kind != 0)
                            mbar_wait(&sbar[warp][(k + j) % kDecStages], ((k + j) / kDecStages) & 1, A.status);
                    }
                    dead = true;
                    break;
                }
                compute(f[0], k % kDecStages);
            }
#pragma unroll
            for (int j = 0; j + 1 < kAhead; ++j) f[j] = f[j + 1];
            f[kAhead - 1] = nb;
        }
    }
    if (!last_chunk) __syncthreads();   // every warp is done with the table
    }   // chunks

    // ---- warp partials -> shared memory (lanes with g < G hold real rows)
    __syncthreads();   // every warp is done with its stage buffers
    float l = st.lp;
    l += __shfl_xor_sync(0xffffffffu, l, 1);
    l += __shfl_xor_sync(0xffffffffu, l, 2);
    if (g < G && t == 0) {
        wm[warp][g] = st.m;
        wl[warp][g] = l;
    }
    // lane (g, t) holds heads 2t, 2t + 1 at d = 8g + i and 64 + 8g + i
#pragma unroll
    for (int e = 0; e < 2; ++e) {
        const int hh = 2 * t + e;
        if (hh < G) {
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                wo[warp][hh][8 * g + i] = st.o[i][e];
                wo[warp][hh][64 + 8 * g + i] = st.o[i][2 + e];
            }
        }
    }
    __syncthreads();

    // ---- CTA partial: part[cta + u][g] = {M, L, 0, 0, O[d]} (16-byte
    // aligned O).  cta + u is unique: both grow along the batch-wide range,
    // so the pieces of unit u sit at first + u .. last + u, in order.
    constexpr int kRec = kHeadDim + 4;
    float* myp = A.part + (static_cast<int64_t>(cta) + u) * G * kRec;
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
    const int npieces = last - first + 1;
    if (tid == 0) is_last = (atomicAdd(&A.ticket[u], 1u) == static_cast<uint32_t>(npieces - 1));
    __syncthreads();
    if (is_last) {
    __threadfence();

    // ---- last CTA of the unit: merge the pieces in order.  A thread owns
    // 4 channels of one head and loads (M, L, O) of up to kMergeChunk pieces
    // at once; chunks merge online.
    if (tid < G * (kHeadDim / 4)) {
        constexpr int kMergeChunk = 20;
        const int gg = tid / (kHeadDim / 4), x4 = (tid % (kHeadDim / 4)) * 4;
        const float* up = A.part + (static_cast<int64_t>(first) + u) * G * kRec + gg * kRec;
        float Mrun = kNegInfF, Lrun = 0.f;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int s0 = 0; s0 < npieces; s0 += kMergeChunk) {
            float2 ml[kMergeChunk];
            float4 ov[kMergeChunk];
#pragma unroll
            for (int k = 0; k < kMergeChunk; ++k) {
                if (s0 + k < npieces) {
                    const float* rec = up + static_cast<int64_t>(s0 + k) * G * kRec;
                    ml[k] = __ldcg(reinterpret_cast<const float2*>(rec));
                    ov[k] = __ldcg(reinterpret_cast<const float4*>(rec + 4 + x4));
                } else {
                    ml[k] = make_float2(kNegInfF, 0.f);
                    ov[k] = make_float4(0.f, 0.f, 0.f, 0.f);
                }
            }
            float Mc = Mrun;
#pragma unroll
            for (int k = 0; k < kMergeChunk; ++k) Mc = fmaxf(Mc, ml[k].x);
            if (Mc == kNegInfF) continue;
            const float r = (Mrun == kNegInfF) ? 0.f : fast_exp2(Mrun - Mc);
            Lrun *= r;
            acc.x *= r;
            acc.y *= r;
            acc.z *= r;
            acc.w *= r;
#pragma unroll
            for (int k = 0; k < kMergeChunk; ++k) {
                if (ml[k].x == kNegInfF) continue;
                const float scl = fast_exp2(ml[k].x - Mc);
                Lrun = fmaf(ml[k].y, scl, Lrun);
                acc.x = fmaf(ov[k].x, scl, acc.x);
                acc.y = fmaf(ov[k].y, scl, acc.y);
                acc.z = fmaf(ov[k].z, scl, acc.z);
                acc.w = fmaf(ov[k].w, scl, acc.w);
            }
            Mrun = Mc;
        }
        const float inv = (Lrun > 0.f) ? 1.f / Lrun : 0.f;
        __half2 h01 = __floats2half2_rn(acc.x * inv, acc.y * inv);
        __half2 h23 = __floats2half2_rn(acc.z * inv, acc.w * inv);
        uint2 pk;
        pk.x = *reinterpret_cast<const uint32_t*>(&h01);
        pk.y = *reinterpret_cast<const uint32_t*>(&h23);
        *reinterpret_cast<uint2*>(A.out + (static_cast<int64_t>(b) * A.Hq + h * G + gg) * kHeadDim + x4) = pk;
    }
    if (tid == 0) A.ticket[u] = 0;
    }   // is_last

    // ---- the next piece's copies land where the warp partials were: put
    // finite numbers back
    __syncthreads();
    for (int i = tid; i < static_cast<int>(sizeof(float) * kDecWarps * G * kHeadDim / 16); i += kDecThreads)
        reinterpret_cast<uint4*>(dec_smem)[i] = make_uint4(0, 0, 0, 0);
    fence_proxy_async();
    __syncthreads();
    }   // pieces
}

}  // namespace

int decode_cta_count(int units, int64_t max_seq_len, int num_sms, int* kps) {
    // one CTA per SM, one wave; a unit of L tokens is cut into at most
    // min(64, L / 256) pieces.  With at least two SMs per unit every unit
    // gets the same number of CTAs; otherwise the batch's bytes are shared
    // out evenly.
    const int sms = std::min(num_sms, kMaxDecCtas);
    const int64_t by_len = std::max<int64_t>(1, std::min<int64_t>(64, (max_seq_len + 255) / 256));
    if (2 * static_cast<int64_t>(units) <= sms) {
        *kps = static_cast<int>(std::min<int64_t>(sms / units, by_len));
        return units * *kps;
    }
    *kps = 0;
    return static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(sms, units * by_len)));
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
    a.units = L.batch * L.shp.Hkv;
    a.kps = L.kps;
    a.tbl_cap = min(max(L.tbl_cap, 32), kTbl);
    a.part = L.part;
    a.ticket = L.ticket;
    a.status = L.status;
    cudaError_t e = cudaSuccess;
    dim3 grid(L.nctas);
    auto launch_dec = [&](auto kern) {
        cudaError_t r = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kDecSmem);
        if (r != cudaSuccess) return r;
        return launch_k(kern, grid, dim3(kDecThreads), kDecSmem, stream, a);
    };
    prof_begin(stream, kProfDecode);
    switch (L.shp.G) {
    case 2: e = launch_dec(decode_kernel<2>); break;
    case 4: e = launch_dec(decode_kernel<4>); break;
    case 8: e = launch_dec(decode_kernel<8>); break;
    default: return cudaErrorInvalidValue;
    }
    if (e != cudaSuccess) return e;
    prof_end(stream, kProfDecode);
    return cudaGetLastError();
}

}  // namespace kv2d
