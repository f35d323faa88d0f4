// pack.cu -- packed KV format of the compressed segments (sm_100a).
//
// MosaicKV ("MosaicKV: Serving Long-Context LLM with Dynamic Two-D KV Cache
// Compression", Fig. 6: packed KV format and flexible KV encoding) stores the
// mixed-strategy segments in a packed layout that attention reads directly.
// The pages give no byte layout; this library uses, per segment, sections
// zero-padded to 16 bytes:
//   FULL : K[S][d] | V[S][d]
//   TOK  : tidx[r] | K[r][d] | V[r][d]
//   CH   : cidx[S][c] | Kval[S][c] | V[S][d]
//   BOTH : tidx[r] | cidx[r][c] | Kval[r][c] | V[r][d]
// with Kval[t][j] = K[t][cidx[t][j]], uint8 indices ascending and tidx
// segment-relative.  One CTA writes one segment: whole K / V rows move as
// 16-byte vectors; the channel indices and Kval of a token are expanded from
// its 128-bit keep mask, one thread per 32-channel word, each word starting
// at the popcount of the words below it.
#include "kernels.h"

namespace kv2d {

namespace {

struct PackArgs {
    SeqPlan plan;
    int Hkv, S, r, c, max_nseg;
    DenseView dv;
    const uint8_t* tidx;
    const uint4* cmask;
    int64_t g_stride;
    const uint8_t* strat;
    const int32_t* unit_ok;
    const uint64_t* desc;
    int32_t max_segs;
    uint8_t* arena;
    int64_t arena_stride;
    uint32_t* status;
};

// Copies whole rows (256 bytes each): chunk c < nk * 16 is chunk c % 16 of
// key row c / 16 (rows kr, destination kdst); the next nv * 16 chunks are
// the value rows (vr, vdst).  A null row reads as zeros.  Four 16-byte loads
// are in flight per thread before their stores.
__device__ __forceinline__ void copy_rows2(const __half* const* kr, int nk, uint8_t* kdst,
                                           const __half* const* vr, int nv, uint8_t* vdst) {
    const int n = (nk + nv) * 16;
    for (int i0 = threadIdx.x; i0 < n; i0 += 4 * blockDim.x) {
        uint4 v[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const int idx = i0 + k * blockDim.x;
            v[k] = make_uint4(0, 0, 0, 0);
            if (idx < n) {
                const bool isk = idx < nk * 16;
                const int c = isk ? idx : idx - nk * 16;
                const __half* row = isk ? kr[c >> 4] : vr[c >> 4];
                if (row) v[k] = *reinterpret_cast<const uint4*>(row + (c & 15) * 8);
            }
        }
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const int idx = i0 + k * blockDim.x;
            if (idx < n) {
                const bool isk = idx < nk * 16;
                const int c = isk ? idx : idx - nk * 16;
                *reinterpret_cast<uint4*>((isk ? kdst : vdst) + (c >> 4) * 256 + (c & 15) * 16) = v[k];
            }
        }
    }
}

// 64 threads per segment: a TOK segment's 4 KB is one 16-byte load per
// thread and load slot, and up to 32 CTAs share an SM, so twice the bytes
// are in flight per SM as with 128-thread CTAs (measured: 580 -> 493 us at
// batch 16 x 128K).
constexpr int kPackThreads = 64;

__global__ void __launch_bounds__(kPackThreads) pack_kernel(const __grid_constant__ PackArgs A) {
    pdl_wait();
    const int j = blockIdx.x, u = blockIdx.y;
    const int b = u / A.Hkv, h = u % A.Hkv;
    if (j >= A.plan.nseg[b]) return;
    const int S = A.S, r = A.r, c = A.c;
    const int64_t slot = static_cast<int64_t>(u) * A.max_nseg + j;
    const int segbase = A.plan.r0[b] / S;
    // one round trip: the unit flag, the strategy, the descriptor and (on
    // speculation) this thread's token index
    const int ok = A.unit_ok[u];
    const int st = A.strat[slot];
    const uint64_t d = A.desc[static_cast<int64_t>(u) * A.max_segs + segbase + j];
    const int tk0 = (static_cast<int>(threadIdx.x) < r) ? A.tidx[slot * r + threadIdx.x] : 0;
    if (!ok) return;
    uint8_t* out = A.arena + static_cast<int64_t>(u) * A.arena_stride +
                   static_cast<int64_t>(d & 0xffffffffull) * 16;
    const int t0 = A.plan.r0[b] + j * S;
    __shared__ int toks[256];
    __shared__ const __half* krows[256];
    __shared__ const __half* vrows[256];
    const bool sparse_tok = (st == KV2D_TOK || st == KV2D_BOTH);
    const int ntok = sparse_tok ? r : S;
    for (int i = threadIdx.x; i < ntok; i += blockDim.x) {
        const int tk = sparse_tok ? (i == static_cast<int>(threadIdx.x) ? tk0 : A.tidx[slot * r + i]) : i;
        toks[i] = tk;
        krows[i] = dense_row(A.dv, A.dv.k, b, h, t0 + tk, A.status);
        vrows[i] = dense_row(A.dv, A.dv.v, b, h, t0 + tk, A.status);
    }
    __syncthreads();
    int64_t o = 0;
    if (sparse_tok) {
        for (int i = threadIdx.x; i < pad16(r); i += blockDim.x)
            out[i] = (i < r) ? static_cast<uint8_t>(toks[i]) : 0;
        o = pad16(r);
    }
    if (st == KV2D_FULL || st == KV2D_TOK) {
        // K rows then V rows, copied in one pass
        copy_rows2(krows, ntok, out + o, vrows, ntok, out + o + static_cast<int64_t>(ntok) * 256);
        return;
    }
    {
        const int n = ntok * c;
        const uint4* mbase = A.cmask + static_cast<int64_t>(u) * A.g_stride + static_cast<int64_t>(j) * S;
        uint8_t* ib = out + o;
        uint16_t* kv = reinterpret_cast<uint16_t*>(out + o + pad16(n));
        bool bad = false;
        for (int it = threadIdx.x; it < ntok * 4; it += blockDim.x) {
            const int i = it >> 2, wd = it & 3;
            const uint4 m4 = mbase[toks[i]];
            int k = i * c + (wd > 0 ? __popc(m4.x) : 0) + (wd > 1 ? __popc(m4.y) : 0) +
                    (wd > 2 ? __popc(m4.z) : 0);
            bad |= (__popc(m4.x) + __popc(m4.y) + __popc(m4.z) + __popc(m4.w)) != c;
            const int kend = (i + 1) * c;
            const __half* row = krows[i];
            for (uint32_t m = wd == 0 ? m4.x : wd == 1 ? m4.y : wd == 2 ? m4.z : m4.w; m && k < kend; m &= m - 1) {
                const int x = wd * 32 + __ffs(m) - 1;
                ib[k] = static_cast<uint8_t>(x);
                kv[k] = row ? __half_as_ushort(row[x]) : static_cast<uint16_t>(0);
                ++k;
            }
        }
        if (bad) atomicOr(A.status, KV2D_DEV_BAD_MASK);
        for (int i = n + threadIdx.x; i < pad16(n); i += blockDim.x) ib[i] = 0;
        for (int i = n + threadIdx.x; i < pad16(2 * n) / 2; i += blockDim.x) kv[i] = 0;
        o += pad16(n) + pad16(2 * n);
    }
    copy_rows2(nullptr, 0, nullptr, vrows, ntok, out + o);
}

}  // namespace

cudaError_t launch_pack(const PackLaunch& L, cudaStream_t stream) {
    if (L.max_nseg <= 0) return cudaSuccess;
    PackArgs a;
    a.plan = L.plan;
    a.Hkv = L.shp.Hkv;
    a.S = L.shp.S;
    a.r = L.shp.r;
    a.c = L.shp.c;
    a.max_nseg = L.max_nseg;
    a.dv = L.dv;
    a.tidx = L.tidx;
    a.cmask = L.cmask;
    a.g_stride = L.g_stride;
    a.strat = L.strat;
    a.unit_ok = L.unit_ok;
    a.desc = L.desc;
    a.max_segs = L.max_segs;
    a.arena = L.arena;
    a.arena_stride = L.arena_stride;
    a.status = L.status;
    dim3 grid(L.max_nseg, L.batch * L.shp.Hkv);
    prof_begin(stream, kProfPack);
    cudaError_t e = launch_k(pack_kernel, grid, dim3(kPackThreads), 0, stream, a);
    if (e != cudaSuccess) return e;
    prof_end(stream, kProfPack);
    return cudaGetLastError();
}

}  // namespace kv2d
