// common.cuh -- device helpers shared by the kv2d kernels (sm_100a only).
//
// Thin wrappers over PTX: mbarriers with bounded waits, TMA tensor loads
// (no multicast), tcgen05 tensor-memory allocation / MMA / loads, and the
// 128-byte-swizzle shared-memory matrix descriptor that tcgen05.mma reads.
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "kv2d.h"

namespace kv2d {

constexpr int kHeadDim = 128;        // head dimension this build runs
constexpr int kKeyTile = 128;        // keys per scoring tile
constexpr int kMaxGW = 512;          // G * W rows per unit, upper bound
constexpr float kLog2e = 1.4426950408889634f;
constexpr unsigned long long kWaitNs = 2000000000ull;   // 2 s per wait

// ------------------------------------------------------------ status word

// The first 256 bytes of every workspace hold one uint32 of KV2D_DEV_* bits.
__device__ __forceinline__ void set_status(uint32_t* status, uint32_t bit) {
    if (status) atomicOr(status, bit);
}

// --------------------------------------------------------------- smem

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ unsigned long long global_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// ----------------------------------------------------------- mbarrier

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
                 : "memory");
}

__device__ __forceinline__ void mbar_fence_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Waits for the phase with the given parity to complete.  Gives up after
// kWaitNs of wall time, sets KV2D_DEV_TIMEOUT and returns false; the caller
// then stops issuing work so that the kernel ends.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, uint32_t* status) {
    if (mbar_try(bar, parity)) return true;
    unsigned long long t0 = global_ns();
    for (uint32_t i = 1;; ++i) {
        if (mbar_try(bar, parity)) return true;
        if ((i & 255u) == 0 && global_ns() - t0 > kWaitNs) {
            set_status(status, KV2D_DEV_TIMEOUT);
            return false;
        }
    }
}

// ---------------------------------------------------------------- TMA

// Orders this thread's earlier shared-memory accesses (generic proxy) before
// later accesses by the copy engine (async proxy) to the same bytes.
__device__ __forceinline__ void fence_proxy_async() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// 2-D / 4-D tiled bulk tensor load into this CTA's shared memory, completion
// counted in bytes on an mbarrier.  No multicast.
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int c0, int c1) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1)
        : "memory");
}

__device__ __forceinline__ void tma_load_4d(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int c0, int c1, int c2, int c3) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2),
        "r"(c3)
        : "memory");
}

__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ------------------------------------------------------------ tcgen05

// Allocates ncols (power of two >= 32) TMEM columns; the whole warp calls.
__device__ __forceinline__ void tmem_alloc(uint32_t* slot, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(slot)),
                 "r"(ncols)
                 : "memory");
}

__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T, fp16 inputs, fp32 accumulation.
__device__ __forceinline__ void umma_f16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                         uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrives once on bar when every tcgen05.mma this thread issued so far is done.
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
            smem_u32(bar))
        : "memory");
}

// 32 consecutive fp32 columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, "
        "[%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
          "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
          "=r"(r[31])
        : "r"(taddr));
}

__device__ __forceinline__ void tmem_ld_wait() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// tcgen05.wait::ld that also names the registers of the load it completes,
// so that no use of them can be scheduled above the wait.
__device__ __forceinline__ void tmem_ld_wait(uint32_t (&r)[32]) {
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]),
                   "+r"(r[6]), "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]),
                   "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15]), "+r"(r[16]), "+r"(r[17]),
                   "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]), "+r"(r[22]), "+r"(r[23]),
                   "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]),
                   "+r"(r[30]), "+r"(r[31])
                 :
                 : "memory");
}

// Shared-memory matrix descriptor for a K-major operand stored with the
// 128-byte swizzle: rows of 128 bytes (64 fp16), 8-row atoms of 1024 bytes,
// atoms stacked every 1024 bytes (stride byte offset).  Bits: start address
// >> 4 in [0,14), leading byte offset >> 4 in [16,30) (unused here, 1),
// stride byte offset >> 4 in [32,46), descriptor version 1 in [46,48),
// layout type 2 (128-byte swizzle) in [61,64).
__device__ __forceinline__ uint64_t sw128_kmajor_desc(uint32_t saddr) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4);
    d |= static_cast<uint64_t>(1) << 16;
    d |= static_cast<uint64_t>(1024 >> 4) << 32;
    d |= static_cast<uint64_t>(1) << 46;
    d |= static_cast<uint64_t>(2) << 61;
    return d;
}

// Instruction descriptor of kind::f16 with fp16 A and B (both K-major) and
// an fp32 accumulator: D format in [4,6), A/B formats in [7,10)/[10,13),
// N >> 3 in [17,23), M >> 4 in [24,29).
__host__ __device__ constexpr uint32_t idesc_f16_f32(int M, int N) {
    return (1u << 4) | (static_cast<uint32_t>(N >> 3) << 17) |
           (static_cast<uint32_t>(M >> 4) << 24);
}

// ------------------------------------------------------------- misc

__device__ __forceinline__ float fast_exp2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// 2^x on the FMA pipe (for x <= 0; below -126 the result is ~0): Cody-Waite
// range reduction x = n + f with n = round(x) by the 1.5 * 2^23 shifter and
// f in [-1/2, 1/2], then 2^f by a degree-5 polynomial whose coefficients were
// fitted to minimise the relative error on that interval (max 2.2e-7 with
// fp32 Horner steps), and n added to the exponent bits.  Used for part of
// the exponentials of the scoring epilogues so that the MUFU pipe is not the
// only one busy.
// Coefficients of the degree-5 fit on [-0.5, 0.5], highest degree first.
constexpr float kExp2P5 = 1.327646780e-03f;
constexpr float kExp2P4 = 9.675540961e-03f;
constexpr float kExp2P3 = 5.550713465e-02f;
constexpr float kExp2P2 = 2.402212024e-01f;
constexpr float kExp2P1 = 6.931469440e-01f;
constexpr float kExp2P0 = 1.000000119e+00f;

__device__ __forceinline__ float exp2_fma(float x) {
    x = fmaxf(x, -126.f);
    const float t = x + 12582912.f;
    const float f = x - (t - 12582912.f);
    float p = kExp2P5;
    p = fmaf(p, f, kExp2P4);
    p = fmaf(p, f, kExp2P3);
    p = fmaf(p, f, kExp2P2);
    p = fmaf(p, f, kExp2P1);
    p = fmaf(p, f, kExp2P0);
    return __int_as_float(__float_as_int(p) + ((__float_as_int(t) - 0x4B400000) << 23));
}

// Packed fp32 pairs (sm_100): each lane is rounded exactly as the scalar
// fused multiply-add / add / subtract of the same operands.
__device__ __forceinline__ float2 f2_fma(float2 a, float2 b, float2 c) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
        "fma.rn.f32x2 rd, ra, rb, rc;\n\t"
        "mov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
    return d;
}

__device__ __forceinline__ float2 f2_add(float2 a, float2 b) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "add.rn.f32x2 rd, ra, rb;\n\t"
        "mov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}

__device__ __forceinline__ float2 f2_sub(float2 a, float2 b) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "sub.rn.f32x2 rd, ra, rb;\n\t"
        "mov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}

// exp2_fma on a pair, the floating-point steps on packed pairs (each lane
// identical to exp2_fma).
__device__ __forceinline__ float2 exp2_fma2(float2 x) {
    x.x = fmaxf(x.x, -126.f);
    x.y = fmaxf(x.y, -126.f);
    const float2 sh = make_float2(12582912.f, 12582912.f);
    const float2 t = f2_add(x, sh);
    const float2 f = f2_sub(x, f2_sub(t, sh));
    float2 p = make_float2(kExp2P5, kExp2P5);
    p = f2_fma(p, f, make_float2(kExp2P4, kExp2P4));
    p = f2_fma(p, f, make_float2(kExp2P3, kExp2P3));
    p = f2_fma(p, f, make_float2(kExp2P2, kExp2P2));
    p = f2_fma(p, f, make_float2(kExp2P1, kExp2P1));
    p = f2_fma(p, f, make_float2(kExp2P0, kExp2P0));
    return make_float2(__int_as_float(__float_as_int(p.x) + ((__float_as_int(t.x) - 0x4B400000) << 23)),
                       __int_as_float(__float_as_int(p.y) + ((__float_as_int(t.y) - 0x4B400000) << 23)));
}

// Programmatic dependent launch: wait until the grids this one depends on
// have completed and their writes are visible (a no-op without a dependency).
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

__host__ __device__ constexpr int64_t pad16(int64_t x) { return (x + 15) / 16 * 16; }

// Per-call constants of the sequences in a batch (passed by value).
struct SeqPlan {
    int32_t T[KV2D_MAX_BATCH];      // tokens in the dense view
    int32_t r0[KV2D_MAX_BATCH];     // region start (comp_end)
    int32_t nseg[KV2D_MAX_BATCH];   // complete segments in the region
    int64_t Bu[KV2D_MAX_BATCH];     // byte budget of each unit of b
};

// Dense view of one layer as the kernels see it.
struct DenseView {
    const __half* k;
    const __half* v;
    int64_t stride_b, stride_h, stride_t;
    int32_t capacity;
    const int32_t* block_table;
    int32_t block_size, max_blocks;
    int64_t num_blocks;
    int32_t num_kv_heads;
};

// Row t of (b, h) in the dense view, or nullptr (with a status bit) when the
// block table points outside the pool.
template <typename T>
__device__ __forceinline__ T* dense_row(const DenseView& dv, T* base, int b, int h, int t,
                                        uint32_t* status) {
    if (dv.block_table == nullptr) {
        if (t < 0 || t >= dv.capacity) {
            set_status(status, KV2D_DEV_SEQ_RANGE);
            return nullptr;
        }
        return base + b * dv.stride_b + h * dv.stride_h + static_cast<int64_t>(t) * dv.stride_t;
    }
    int blk = t / dv.block_size;
    if (t < 0 || blk >= dv.max_blocks) {
        set_status(status, KV2D_DEV_SEQ_RANGE);
        return nullptr;
    }
    int phys = dv.block_table[static_cast<int64_t>(b) * dv.max_blocks + blk];
    if (phys < 0 || phys >= dv.num_blocks) {
        set_status(status, KV2D_DEV_BLOCK_TABLE);
        return nullptr;
    }
    return base + (static_cast<int64_t>(phys) * dv.num_kv_heads + h) * dv.block_size * kHeadDim +
           static_cast<int64_t>(t % dv.block_size) * kHeadDim;
}

}  // namespace kv2d
