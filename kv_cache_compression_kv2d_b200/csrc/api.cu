// api.cu -- the C ABI of kv2d (declared in include/kv2d.h).
//
// Host side only: argument validation, budget feasibility, workspace
// carving, TMA descriptor encoding and kernel launches on the caller's
// stream.  No device memory is allocated and no stream is synchronised
// (except in kv2d_read_status, whose job that is).
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include "kernels.h"
#include "kv2d.h"

using namespace kv2d;

namespace {

thread_local std::string g_err;

kv2d_status fail(kv2d_status s, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_err = buf;
    return s;
}

kv2d_status ok() {
    g_err.clear();
    return KV2D_OK;
}

int64_t round_up(int64_t x, int64_t m) { return (x + m - 1) / m * m; }

// Returns KV2D_OK or the reason the parameters are unusable.
kv2d_status check_params(const kv2d_params* p) {
    if (!p) return fail(KV2D_ERR_INVALID_ARG, "params is NULL");
    if (p->head_dim != 64 && p->head_dim != 128 && p->head_dim != 256)
        return fail(KV2D_ERR_INVALID_ARG, "head_dim %d not in {64, 128, 256}", p->head_dim);
    if (p->num_q_heads <= 0 || p->num_kv_heads <= 0 || p->num_q_heads % p->num_kv_heads != 0)
        return fail(KV2D_ERR_INVALID_ARG, "num_q_heads %d must be a positive multiple of num_kv_heads %d",
                    p->num_q_heads, p->num_kv_heads);
    const int G = p->num_q_heads / p->num_kv_heads;
    if (p->segment_len < 16 || p->segment_len > 256 || p->segment_len % 16 != 0)
        return fail(KV2D_ERR_INVALID_ARG, "segment_len %d must be a multiple of 16 in [16, 256]",
                    p->segment_len);
    if (p->window < 1 || G * p->window > kMaxGW)
        return fail(KV2D_ERR_INVALID_ARG, "window %d: need 1 <= G*W <= %d (G = %d)", p->window,
                    kMaxGW, G);
    if (p->keep_tokens < 1 || p->keep_tokens > p->segment_len)
        return fail(KV2D_ERR_INVALID_ARG, "keep_tokens %d not in [1, S = %d]", p->keep_tokens,
                    p->segment_len);
    if (p->keep_channels < 1 || p->keep_channels > p->head_dim)
        return fail(KV2D_ERR_INVALID_ARG, "keep_channels %d not in [1, d = %d]", p->keep_channels,
                    p->head_dim);
    if (!(p->budget > 0.f) || !std::isfinite(p->budget))
        return fail(KV2D_ERR_INVALID_ARG, "budget must be a positive finite fraction");
    if (!(p->scale >= 0.f) || !std::isfinite(p->scale))
        return fail(KV2D_ERR_INVALID_ARG, "scale must be finite and >= 0 (0 selects 1/sqrt(d))");
    if (p->chunk_len != 0) {
        if (p->chunk_len < 3 || p->chunk_len > p->segment_len)
            return fail(KV2D_ERR_INVALID_ARG, "chunk_len %d: need 0 (off) or 3 <= chunk_len <= S = %d",
                        p->chunk_len, p->segment_len);
        if (p->chunk_budget < 1 || p->chunk_budget >= p->keep_tokens)
            return fail(KV2D_ERR_INVALID_ARG, "chunk_budget %d: need 1 <= chunk_budget < r = %d",
                        p->chunk_budget, p->keep_tokens);
        if (p->keep_tokens - p->chunk_budget > 33)
            return fail(KV2D_ERR_UNSUPPORTED, "Token2Chunk runs r - chunk_budget <= 33 core tokens, got %d",
                        p->keep_tokens - p->chunk_budget);
    }
    if (p->head_dim != kHeadDim)
        return fail(KV2D_ERR_UNSUPPORTED, "this build runs head_dim = %d only", kHeadDim);
    return KV2D_OK;
}

int64_t seg_bytes(const kv2d_params* p, int st) {
    const int64_t S = p->segment_len, d = p->head_dim, r = p->keep_tokens, c = p->keep_channels;
    switch (st) {
    case KV2D_FULL: return 4 * S * d;
    case KV2D_TOK: return pad16(r) + 4 * r * d;
    case KV2D_CH: return pad16(S * c) + pad16(2 * S * c) + 2 * S * d;
    case KV2D_BOTH: return pad16(r) + pad16(r * c) + pad16(2 * r * c) + 2 * r * d;
    default: return -1;
    }
}

float eff_scale(const kv2d_params* p) {
    return p->scale > 0.f ? p->scale : 1.0f / std::sqrt(static_cast<float>(p->head_dim));
}

UnitShape shape_of(const kv2d_params* p) {
    UnitShape s;
    s.Hkv = p->num_kv_heads;
    s.Hq = p->num_q_heads;
    s.G = p->num_q_heads / p->num_kv_heads;
    s.W = p->window;
    s.GW = s.G * s.W;
    s.GWpad = static_cast<int32_t>(round_up(s.GW, 128));
    s.S = p->segment_len;
    s.r = p->keep_tokens;
    s.c = p->keep_channels;
    s.c2 = eff_scale(p) * kLog2e;
    s.chunk_len = p->chunk_len;
    s.chunk_budget = p->chunk_len ? p->chunk_budget : 0;
    return s;
}

// Budget of one unit: floor(beta * (nseg * FULL bytes)) in fp64.
int64_t unit_budget(const kv2d_params* p, int nseg) {
    const int64_t full = seg_bytes(p, KV2D_FULL);
    return static_cast<int64_t>(
        std::floor(static_cast<double>(p->budget) * static_cast<double>(static_cast<int64_t>(nseg) * full)));
}

// ---- workspace layouts (every region 256-byte aligned)

struct Carver {
    size_t off = 0;
    size_t take(size_t bytes) {
        const size_t at = off;
        off = static_cast<size_t>(round_up(static_cast<int64_t>(off + bytes), 256));
        return at;
    }
};

constexpr int kMaxSplit1 = 64;

struct CompressLayout {
    size_t apart, part, s, g, cmask, tidx, E, hull, eff, db, strat, ok, total;
    int64_t s_stride, g_stride;
    int max_nseg;
};

CompressLayout compress_layout(const kv2d_params* p, int batch, int64_t max_region) {
    const UnitShape sh = shape_of(p);
    const int64_t units = static_cast<int64_t>(batch) * sh.Hkv;
    CompressLayout L;
    L.max_nseg = static_cast<int>(max_region / sh.S);
    L.s_stride = round_up(std::max<int64_t>(max_region, 1), 4);
    L.g_stride = std::max<int64_t>(static_cast<int64_t>(L.max_nseg) * sh.S, 1);
    const int64_t ns = std::max(L.max_nseg, 1);
    Carver c;
    c.take(256);   // status header
    L.apart = c.take(units * (sh.GWpad / 128) * kHeadDim * 4);
    L.part = c.take(units * sh.GWpad * kMaxSplit1 * 8);
    L.s = c.take(units * L.s_stride * 4);
    L.g = c.take(units * L.g_stride * 8);
    L.cmask = c.take(units * L.g_stride * 16);
    L.tidx = c.take(units * ns * sh.r);
    L.E = c.take(units * ns * 4 * 8);
    L.hull = c.take(units * ns * 8);
    L.eff = c.take(units * ns * 3 * 8);
    L.db = c.take(units * ns * 3 * 4);
    L.strat = c.take(units * ns);
    L.ok = c.take(units * 4);
    L.total = c.off;
    return L;
}

struct DecodeLayout {
    size_t ticket, part, total;
};

DecodeLayout decode_layout(const kv2d_params* p, int batch) {
    const UnitShape sh = shape_of(p);
    const int64_t units = static_cast<int64_t>(batch) * sh.Hkv;
    DecodeLayout L;
    Carver c;
    c.take(256);
    L.ticket = c.take(units * 4);
    L.part = c.take((units + kMaxDecCtas) * sh.G * (kHeadDim + 4) * 4);
    L.total = c.off;
    return L;
}

struct SelectLayout {
    size_t cscore, cslot, ccount, gather, nsel, ticket, part, total;
    int64_t slot_stride;
    int nreg;
};

// Workspace of kv2d_decode_attn_select: per unit the candidate scores and
// their slots compacted per region of 64 segments over (max_seq_len / S) * S
// candidate slots, the regions' counts, the kept items' gather entries, the
// kept count, a ticket, and the attention partials of up to kSel2MaxChunks
// chunks.
SelectLayout select_layout(const kv2d_params* p, int batch, int64_t max_seq_len) {
    const UnitShape sh = shape_of(p);
    const int64_t units = static_cast<int64_t>(batch) * sh.Hkv;
    SelectLayout L;
    L.slot_stride = round_up(std::max<int64_t>(max_seq_len / sh.S * sh.S, 1), 4);
    L.nreg = std::max(1, sel2_regions(L.slot_stride, sh.S));
    Carver c;
    c.take(256);
    L.cscore = c.take(units * L.slot_stride * 4);
    L.cslot = c.take(units * L.slot_stride * 4);
    L.ccount = c.take(units * L.nreg * 4);
    L.gather = c.take(units * L.slot_stride * 8);
    L.nsel = c.take(units * 4);
    L.ticket = c.take(units * 4);
    L.part = c.take(units * kSel2MaxChunks * sh.G * (kHeadDim + 4) * 4);
    L.total = c.off;
    return L;
}

// blocks per chunk of the decode kernel's block table (kv2d_set_decode_table_cap)
std::atomic<int> g_dec_table_cap{kDecTableMax};

int num_sms() {
    int dev = 0, n = 148;
    if (cudaGetDevice(&dev) == cudaSuccess)
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n > 0 ? n : 148;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    });
    return fn;
}

bool aligned(const void* ptr, size_t a) { return (reinterpret_cast<uintptr_t>(ptr) % a) == 0; }

kv2d_status check_dense(const kv2d_params* p, int batch, const kv2d_dense* kv) {
    if (!kv || !kv->k || !kv->v) return fail(KV2D_ERR_INVALID_ARG, "dense view or its K/V is NULL");
    if (!aligned(kv->k, 16) || !aligned(kv->v, 16))
        return fail(KV2D_ERR_INVALID_ARG, "dense K/V must be 16-byte aligned");
    if (kv->block_table) {
        if (kv->block_size < 16 || kv->block_size % 16 != 0 || kv->block_size > 256)
            return fail(KV2D_ERR_INVALID_ARG, "block_size %d must be a multiple of 16 in [16, 256]",
                        kv->block_size);
        if (kv->max_blocks <= 0 || kv->num_blocks <= 0)
            return fail(KV2D_ERR_INVALID_ARG, "paged view needs max_blocks > 0 and num_blocks > 0");
    } else {
        if (kv->capacity <= 0) return fail(KV2D_ERR_INVALID_ARG, "capacity must be > 0");
        if (kv->stride_t % 8 || kv->stride_h % 8 || kv->stride_b % 8 || kv->stride_t < p->head_dim)
            return fail(KV2D_ERR_INVALID_ARG, "strides must be multiples of 8 elements, stride_t >= d");
    }
    (void)batch;
    return KV2D_OK;
}

DenseView view_of(const kv2d_params* p, const kv2d_dense* kv) {
    DenseView dv;
    dv.k = static_cast<const __half*>(kv->k);
    dv.v = static_cast<const __half*>(kv->v);
    dv.stride_b = kv->stride_b;
    dv.stride_h = kv->stride_h;
    dv.stride_t = kv->stride_t;
    dv.capacity = kv->capacity;
    dv.block_table = kv->block_table;
    dv.block_size = kv->block_size;
    dv.max_blocks = kv->max_blocks;
    dv.num_blocks = kv->num_blocks;
    dv.num_kv_heads = p->num_kv_heads;
    return dv;
}

int dense_capacity(const kv2d_dense* kv) {
    if (kv->block_table) {
        const int64_t c = static_cast<int64_t>(kv->max_blocks) * kv->block_size;
        return static_cast<int>(std::min<int64_t>(c, INT32_MAX));
    }
    return kv->capacity;
}

// ---- optional event profiler: an event pair around every launch

struct ProfRec {
    int stage;
    cudaEvent_t a, b;
};

std::mutex g_prof_mu;
bool g_prof_on = false;
std::vector<ProfRec> g_prof_open;      // begun, not yet ended (one per stage)
std::vector<ProfRec> g_prof_done;

const char* const kStageNames[kProfStages] = {"score_pass1", "score_pass2", "chan_topc",  "seg_select",
                                              "budget",      "pack",        "append",     "decode",
                                              "sel_score",   "sel_topn",    "sel_attn"};

}  // namespace

namespace kv2d {

void prof_begin(cudaStream_t s, int stage) {
    std::lock_guard<std::mutex> lk(g_prof_mu);
    if (!g_prof_on) return;
    ProfRec r{stage, nullptr, nullptr};
    if (cudaEventCreate(&r.a) != cudaSuccess || cudaEventCreate(&r.b) != cudaSuccess) return;
    cudaEventRecord(r.a, s);
    g_prof_open.push_back(r);
}

void prof_end(cudaStream_t s, int stage) {
    std::lock_guard<std::mutex> lk(g_prof_mu);
    if (!g_prof_on) return;
    for (size_t i = g_prof_open.size(); i-- > 0;) {
        if (g_prof_open[i].stage != stage) continue;
        ProfRec r = g_prof_open[i];
        g_prof_open.erase(g_prof_open.begin() + static_cast<long>(i));
        cudaEventRecord(r.b, s);
        g_prof_done.push_back(r);
        return;
    }
}

}  // namespace kv2d

namespace {
// ---- fixed device scratch for kv2d_decode_attn_noalloc
//
// The array lives in every GPU's global memory from the moment the library's
// module is loaded on that GPU until the process exits.  Host code must not
// take its address directly (the host-side name is only a stand-in); the
// device address comes from cudaGetSymbolAddress, once per device.

constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;   // 8 MiB per GPU
constexpr int kNoAllocMaxDevices = 64;
// Fixed layout, the same for every call: bytes [0, 256) are unused, the
// per-unit tickets sit at [256, 256 + kNoAllocTicketBytes) and the per-CTA
// partials after them.  The tickets must read zero when a call starts;
// every completed call leaves the ones it used at zero, and no call ever
// writes anything else there, whatever its shape.
constexpr size_t kNoAllocTicketOff = 256;
constexpr size_t kNoAllocTicketBytes = size_t(64) << 10;   // 16384 units
constexpr size_t kNoAllocPartOff = kNoAllocTicketOff + kNoAllocTicketBytes;

// Per device: the id of the context the address was looked up in, and the
// address.  A device reset (cudaDeviceReset) ends that context and the
// module is loaded again, possibly elsewhere, in a new one; context ids are
// never reused within a process, so a changed id means the lookup is redone.
struct NoAllocSlot {
    unsigned long long ctx_id;
    void* ptr;
};
std::mutex g_noalloc_mu;
NoAllocSlot g_noalloc[kNoAllocMaxDevices] = {};

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

template <typename Fn>
Fn driver_fn(const char* name) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint(name, &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
        return reinterpret_cast<Fn>(ptr);
    return nullptr;
}

}  // namespace

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

namespace {

// Device address of the scratch array in the current device's current
// context, looked up on the first call per device (and again after the
// context changed).
kv2d_status noalloc_scratch(void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return fail(KV2D_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
    if (dev < 0 || dev >= kNoAllocMaxDevices)
        return fail(KV2D_ERR_UNSUPPORTED, "device ordinal %d beyond %d", dev, kNoAllocMaxDevices);
    static const CtxGetCurrentFn get_ctx = driver_fn<CtxGetCurrentFn>("cuCtxGetCurrent");
    static const CtxGetIdFn get_id = driver_fn<CtxGetIdFn>("cuCtxGetId");
    if (!get_ctx || !get_id) return fail(KV2D_ERR_CUDA, "the driver's context queries are unavailable");
    auto current_id = [&](unsigned long long* id) {
        CUcontext ctx = nullptr;
        return get_ctx(&ctx) == CUDA_SUCCESS && ctx && get_id(ctx, id) == CUDA_SUCCESS;
    };
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    NoAllocSlot& slot = g_noalloc[dev];
    unsigned long long id = 0;
    if (!slot.ptr || !current_id(&id) || slot.ctx_id != id) {
        // the lookup also makes the device's primary context current
        void* ptr = nullptr;
        e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
        if (e != cudaSuccess || !ptr)
            return fail(KV2D_ERR_CUDA, "cudaGetSymbolAddress of the decode scratch: %s",
                        cudaGetErrorString(e));
        if (!current_id(&id)) return fail(KV2D_ERR_CUDA, "cannot identify the current CUDA context");
        // the tickets start at zero in a fresh context (one-time set-up,
        // synchronous, before the array is first used)
        e = cudaMemset(static_cast<uint8_t*>(ptr) + kNoAllocTicketOff, 0, kNoAllocTicketBytes);
        if (e != cudaSuccess) return fail(KV2D_ERR_CUDA, "clearing the decode scratch tickets: %s",
                                          cudaGetErrorString(e));
        slot.ctx_id = id;
        slot.ptr = ptr;
    }
    *out = slot.ptr;
    return KV2D_OK;
}

}  // namespace

extern "C" {

int64_t kv2d_segment_bytes(const kv2d_params* p, int strategy) {
    const kv2d_status s = check_params(p);
    if (s != KV2D_OK && s != KV2D_ERR_UNSUPPORTED) return -1;
    return seg_bytes(p, strategy);
}

int64_t kv2d_arena_bytes(const kv2d_params* p, int64_t max_tokens) {
    const kv2d_status s = check_params(p);
    if ((s != KV2D_OK && s != KV2D_ERR_UNSUPPORTED) || max_tokens < 0) return -1;
    const int64_t nseg = max_tokens / p->segment_len;
    const double beta = std::min(1.0, static_cast<double>(p->budget));
    const double need = std::ceil(beta * static_cast<double>(nseg * seg_bytes(p, KV2D_FULL)));
    return round_up(static_cast<int64_t>(need) + 16, 256);
}

size_t kv2d_workspace_bytes(const kv2d_params* p, int op, int batch, int64_t max_tokens) {
    if (check_params(p) != KV2D_OK || batch < 1 || batch > KV2D_MAX_BATCH || max_tokens < 0) return 0;
    switch (op) {
    case KV2D_OP_COMPRESS: return compress_layout(p, batch, max_tokens).total;
    case KV2D_OP_DECODE: return decode_layout(p, batch).total;
    case KV2D_OP_APPEND: return 256;
    case KV2D_OP_DECODE_SELECT: return select_layout(p, batch, max_tokens).total;
    default: return 0;
    }
}

}  // extern "C"

namespace {

// The compression of kv2d_compress; with staged != NULL the new bookkeeping
// (n_segs, used_bytes, comp_end) goes to the staged record instead of the
// live one (the record is first set to the live values, so sequences
// without a new segment keep theirs).
kv2d_status compress_impl(const kv2d_params* p, int batch, const int32_t* seq_len_host,
                          const int32_t* comp_end_host, const kv2d_dense* kv, const void* q_window,
                          kv2d_ccache* cc, const kv2d_staged* staged, void* ws, size_t ws_bytes,
                          const kv2d_debug* dbg, void* stream) {
    kv2d_status st = check_params(p);
    if (st != KV2D_OK) return st;
    if (batch < 1 || batch > KV2D_MAX_BATCH)
        return fail(KV2D_ERR_INVALID_ARG, "batch %d not in [1, %d]", batch, KV2D_MAX_BATCH);
    if (!seq_len_host || !comp_end_host) return fail(KV2D_ERR_INVALID_ARG, "host length arrays are NULL");
    if ((st = check_dense(p, batch, kv)) != KV2D_OK) return st;
    if (!q_window || !aligned(q_window, 16))
        return fail(KV2D_ERR_INVALID_ARG, "q_window must be a 16-byte aligned device pointer");
    if (!cc || !cc->arena || !cc->desc || !cc->n_segs || !cc->used_bytes || !cc->comp_end)
        return fail(KV2D_ERR_INVALID_ARG, "compressed cache has a NULL pointer");
    if (!aligned(cc->arena, 256) || cc->arena_stride <= 0 || cc->arena_stride % 256)
        return fail(KV2D_ERR_INVALID_ARG, "arena must be 256-byte aligned with a stride that is a multiple of 256");
    if (!aligned(cc->desc, 8) || cc->max_segs <= 0)
        return fail(KV2D_ERR_INVALID_ARG, "descriptor table misaligned or max_segs <= 0");
    if (!ws || !aligned(ws, 256)) return fail(KV2D_ERR_WORKSPACE, "workspace must be 256-byte aligned");

    const UnitShape sh = shape_of(p);
    const int cap = dense_capacity(kv);
    SeqPlan plan;
    std::memset(&plan, 0, sizeof plan);
    int64_t max_region = 0;
    int max_nseg = 0;
    const int64_t min_bytes =
        std::min(std::min(seg_bytes(p, 0), seg_bytes(p, 1)), std::min(seg_bytes(p, 2), seg_bytes(p, 3)));
    for (int b = 0; b < batch; ++b) {
        const int T = seq_len_host[b], r0 = comp_end_host[b];
        if (T < 0 || T > cap)
            return fail(KV2D_ERR_INVALID_ARG, "seq_len[%d] = %d outside [0, capacity %d]", b, T, cap);
        if (r0 < 0 || r0 > T || r0 % sh.S)
            return fail(KV2D_ERR_INVALID_ARG, "comp_end[%d] = %d must be a multiple of S in [0, seq_len]", b, r0);
        const int region = T - r0;
        const int nseg = region / sh.S;
        if (nseg > 0 && sh.W > region)
            return fail(KV2D_ERR_INVALID_ARG, "window %d longer than the region %d of sequence %d", sh.W,
                        region, b);
        plan.T[b] = T;
        plan.r0[b] = r0;
        plan.nseg[b] = nseg;
        plan.Bu[b] = unit_budget(p, nseg);
        if (nseg > 0 && p->budget < 1.f && nseg * min_bytes > plan.Bu[b])
            return fail(KV2D_ERR_BUDGET_INFEASIBLE,
                        "sequence %d: %d segments need at least %lld bytes, budget is %lld", b, nseg,
                        static_cast<long long>(nseg * min_bytes), static_cast<long long>(plan.Bu[b]));
        if (r0 / sh.S + nseg > cc->max_segs)
            return fail(KV2D_ERR_CAPACITY, "sequence %d needs %d descriptors, max_segs is %d", b,
                        r0 / sh.S + nseg, cc->max_segs);
        const int64_t need = kv2d_arena_bytes(p, static_cast<int64_t>(r0) + static_cast<int64_t>(nseg) * sh.S);
        if (need > cc->arena_stride)
            return fail(KV2D_ERR_CAPACITY, "sequence %d may need %lld arena bytes per unit, stride is %lld",
                        b, static_cast<long long>(need), static_cast<long long>(cc->arena_stride));
        if (nseg > 0) max_region = std::max<int64_t>(max_region, region);
        max_nseg = std::max(max_nseg, nseg);
    }
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (staged) {
        if (!staged->n_segs || !staged->used_bytes || !staged->comp_end || !aligned(staged->used_bytes, 8))
            return fail(KV2D_ERR_INVALID_ARG, "staged record has a NULL or misaligned pointer");
        const size_t units = static_cast<size_t>(batch) * sh.Hkv;
        cudaError_t e0 = cudaMemcpyAsync(staged->n_segs, cc->n_segs, units * 4, cudaMemcpyDeviceToDevice, s);
        if (e0 == cudaSuccess)
            e0 = cudaMemcpyAsync(staged->used_bytes, cc->used_bytes, units * 8, cudaMemcpyDeviceToDevice, s);
        if (e0 == cudaSuccess)
            e0 = cudaMemcpyAsync(staged->comp_end, cc->comp_end, static_cast<size_t>(batch) * 4,
                                 cudaMemcpyDeviceToDevice, s);
        if (e0 != cudaSuccess) return fail(KV2D_ERR_CUDA, "staging copy: %s", cudaGetErrorString(e0));
    }
    if (max_nseg == 0) return ok();   // nothing complete to compress

    const CompressLayout WL = compress_layout(p, batch, max_region);
    if (ws_bytes < WL.total)
        return fail(KV2D_ERR_WORKSPACE, "workspace %zu bytes, need %zu", ws_bytes, WL.total);
    if (dbg && (dbg->s || dbg->g) && dbg->region_stride < max_region)
        return fail(KV2D_ERR_INVALID_ARG, "debug region_stride %lld < region %lld",
                    static_cast<long long>(dbg->region_stride), static_cast<long long>(max_region));
    if (dbg && dbg->E && dbg->seg_stride < max_nseg)
        return fail(KV2D_ERR_INVALID_ARG, "debug seg_stride %d < segments %d", dbg->seg_stride, max_nseg);

    auto encode = encode_fn();
    if (!encode) return fail(KV2D_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
    uint8_t* w = static_cast<uint8_t*>(ws);
    const int units = batch * sh.Hkv;

    ScoreLaunch SL;
    std::memset(&SL, 0, sizeof SL);
    SL.plan = plan;
    SL.shp = sh;
    SL.batch = batch;
    SL.dv = view_of(p, kv);
    SL.qw = static_cast<const __half*>(q_window);
    SL.paged = kv->block_table != nullptr;
    SL.max_region = static_cast<int>(max_region);
    SL.max_nseg = max_nseg;
    {
        cuuint64_t dims[2] = {static_cast<cuuint64_t>(kHeadDim),
                              static_cast<cuuint64_t>(batch) * sh.Hq * sh.W};
        cuuint64_t strides[1] = {static_cast<cuuint64_t>(kHeadDim) * 2};
        cuuint32_t box[2] = {64, 64};
        cuuint32_t es[2] = {1, 1};
        CUresult r = encode(&SL.qmap, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(q_window),
                            dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) return fail(KV2D_ERR_CUDA, "query tensor map encode failed (%d)", int(r));
    }
    {
        CUresult r;
        cuuint32_t es[4] = {1, 1, 1, 1};
        if (!SL.paged) {
            cuuint64_t dims[4] = {static_cast<cuuint64_t>(kHeadDim), static_cast<cuuint64_t>(kv->capacity),
                                  static_cast<cuuint64_t>(sh.Hkv), static_cast<cuuint64_t>(batch)};
            cuuint64_t strides[3] = {static_cast<cuuint64_t>(kv->stride_t) * 2,
                                     static_cast<cuuint64_t>(kv->stride_h) * 2,
                                     static_cast<cuuint64_t>(kv->stride_b) * 2};
            cuuint32_t box[4] = {64, static_cast<cuuint32_t>(kKeyTile), 1, 1};
            r = encode(&SL.kmap, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 4, kv->k, dims, strides, box, es,
                       CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                       CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        } else {
            cuuint64_t dims[4] = {static_cast<cuuint64_t>(kHeadDim), static_cast<cuuint64_t>(kv->block_size),
                                  static_cast<cuuint64_t>(sh.Hkv), static_cast<cuuint64_t>(kv->num_blocks)};
            cuuint64_t strides[3] = {static_cast<cuuint64_t>(kHeadDim) * 2,
                                     static_cast<cuuint64_t>(kHeadDim) * 2 * kv->block_size,
                                     static_cast<cuuint64_t>(kHeadDim) * 2 * kv->block_size * sh.Hkv};
            cuuint32_t box[4] = {64, 16, 1, 1};
            r = encode(&SL.kmap, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 4, kv->k, dims, strides, box, es,
                       CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                       CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        }
        if (r != CUDA_SUCCESS) return fail(KV2D_ERR_CUDA, "key tensor map encode failed (%d)", int(r));
    }
    // Grids fill whole waves: pass 1 runs two CTAs per SM, pass 2 one.  A
    // unit's keys are cut into ns splits so that the CTAs come as close as
    // possible to a whole number of waves (few splits: each costs a
    // pipeline fill and one lse partial per window row).
    const int nsm = num_sms();
    const int mtiles = sh.GWpad / 128;
    auto pick_splits = [](int64_t groups, int64_t slots, int64_t max_ns) {
        int64_t best = 1;
        double best_eff = 0.0;
        for (int64_t ns = 1; ns <= max_ns; ++ns) {
            const int64_t ctas = groups * ns;
            const int64_t waves = (ctas + slots - 1) / slots;
            const double eff = static_cast<double>(ctas) / static_cast<double>(waves * slots);
            if (eff > best_eff + 0.02) {
                best_eff = eff;
                best = ns;
            }
            if (eff >= 0.97 && ctas >= slots) break;
        }
        return best;
    };
    {
        const int64_t max_tiles = (max_region + kKeyTile - 1) / kKeyTile;
        const int64_t groups = static_cast<int64_t>(units) * mtiles;
        const int64_t ns = pick_splits(groups, 2 * nsm, std::min<int64_t>(max_tiles, kMaxSplit1));
        const int64_t tiles_per = (max_tiles + ns - 1) / ns;
        SL.kps1 = static_cast<int>(tiles_per * kKeyTile);
        SL.nsplit1 = static_cast<int>((max_tiles + tiles_per - 1) / tiles_per);
    }
    {
        const int64_t seg_tok = static_cast<int64_t>(max_nseg) * sh.S;
        const int64_t max_tiles = (seg_tok + kKeyTile - 1) / kKeyTile;
        const int64_t ns = pick_splits(units, nsm, std::min<int64_t>(max_tiles, 256));
        const int64_t tiles_per = (max_tiles + ns - 1) / ns;
        SL.kps2 = static_cast<int>(tiles_per * kKeyTile);
        SL.nsplit2 = static_cast<int>((max_tiles + tiles_per - 1) / tiles_per);
    }
    SL.apart = reinterpret_cast<float*>(w + WL.apart);
    SL.part = reinterpret_cast<float2*>(w + WL.part);
    SL.s = reinterpret_cast<float*>(w + WL.s);
    SL.s_stride = WL.s_stride;
    SL.g = reinterpret_cast<double*>(w + WL.g);
    SL.cmask = reinterpret_cast<uint4*>(w + WL.cmask);
    SL.g_stride = WL.g_stride;
    SL.status = reinterpret_cast<uint32_t*>(w);
    if (dbg) {
        SL.dbg_a = dbg->a;
        SL.dbg_lse = dbg->lse;
        SL.dbg_s = dbg->s;
        SL.dbg_g = dbg->g;
        SL.dbg_stride = dbg->region_stride;
    }
    cudaError_t e = launch_scoring(SL, s);
    if (e != cudaSuccess) return fail(KV2D_ERR_CUDA, "scoring launch: %s", cudaGetErrorString(e));

    SelectLaunch XL;
    std::memset(&XL, 0, sizeof XL);
    XL.plan = plan;
    XL.shp = sh;
    XL.batch = batch;
    XL.max_nseg = max_nseg;
    for (int k = 0; k < 4; ++k) {
        XL.bytes[k] = seg_bytes(p, k);
        XL.order[k] = k;
    }
    for (int i = 1; i < 4; ++i) {   // strategies by (bytes, id)
        const int v = XL.order[i];
        int j = i - 1;
        while (j >= 0 && (XL.bytes[XL.order[j]] > XL.bytes[v] ||
                          (XL.bytes[XL.order[j]] == XL.bytes[v] && XL.order[j] > v))) {
            XL.order[j + 1] = XL.order[j];
            --j;
        }
        XL.order[j + 1] = v;
    }
    XL.all_full = p->budget >= 1.f;
    XL.s = SL.s;
    XL.s_stride = WL.s_stride;
    XL.g = SL.g;
    XL.g_stride = WL.g_stride;
    XL.tidx = w + WL.tidx;
    XL.E = reinterpret_cast<double*>(w + WL.E);
    XL.hull = w + WL.hull;
    XL.eff = reinterpret_cast<double*>(w + WL.eff);
    XL.dbytes = reinterpret_cast<int32_t*>(w + WL.db);
    XL.strat = w + WL.strat;
    XL.unit_ok = reinterpret_cast<int32_t*>(w + WL.ok);
    XL.desc = static_cast<uint64_t*>(cc->desc);
    XL.max_segs = cc->max_segs;
    XL.n_segs = cc->n_segs;
    XL.used_bytes = cc->used_bytes;
    XL.comp_end = cc->comp_end;
    if (staged) {
        XL.out_n_segs = staged->n_segs;
        XL.out_used_bytes = staged->used_bytes;
        XL.out_comp_end = staged->comp_end;
    }
    XL.arena_stride = cc->arena_stride;
    XL.status = SL.status;
    if (dbg) {
        XL.dbg_E = dbg->E;
        XL.dbg_seg_stride = dbg->seg_stride;
    }
    e = launch_selection(XL, s);
    if (e != cudaSuccess) return fail(KV2D_ERR_CUDA, "selection launch: %s", cudaGetErrorString(e));

    PackLaunch PL;
    std::memset(&PL, 0, sizeof PL);
    PL.plan = plan;
    PL.shp = sh;
    PL.batch = batch;
    PL.max_nseg = max_nseg;
    PL.dv = SL.dv;
    PL.tidx = XL.tidx;
    PL.cmask = SL.cmask;
    PL.g_stride = WL.g_stride;
    PL.strat = XL.strat;
    PL.unit_ok = XL.unit_ok;
    PL.desc = XL.desc;
    PL.max_segs = cc->max_segs;
    PL.arena = static_cast<uint8_t*>(cc->arena);
    PL.arena_stride = cc->arena_stride;
    PL.status = SL.status;
    e = launch_pack(PL, s);
    if (e != cudaSuccess) return fail(KV2D_ERR_CUDA, "pack launch: %s", cudaGetErrorString(e));
    (void)units;
    return ok();
}

}  // namespace

extern "C" {

kv2d_status kv2d_compress(const kv2d_params* p, int batch, const int32_t* seq_len_host,
                          const int32_t* comp_end_host, const kv2d_dense* kv, const void* q_window,
                          kv2d_ccache* cc, void* ws, size_t ws_bytes, const kv2d_debug* dbg,
                          void* stream) {
    return compress_impl(p, batch, seq_len_host, comp_end_host, kv, q_window, cc, nullptr, ws, ws_bytes,
                         dbg, stream);
}

kv2d_status kv2d_compress_staged(const kv2d_params* p, int batch, const int32_t* seq_len_host,
                                 const int32_t* comp_end_host, const kv2d_dense* kv,
                                 const void* q_window, kv2d_ccache* cc, const kv2d_staged* staged,
                                 void* ws, size_t ws_bytes, const kv2d_debug* dbg, void* stream) {
    if (!staged) return fail(KV2D_ERR_INVALID_ARG, "staged record is NULL");
    return compress_impl(p, batch, seq_len_host, comp_end_host, kv, q_window, cc, staged, ws, ws_bytes,
                         dbg, stream);
}

kv2d_status kv2d_switch(const kv2d_params* p, int batch, kv2d_ccache* cc, const kv2d_staged* staged,
                        void* stream) {
    kv2d_status st = check_params(p);
    if (st != KV2D_OK) return st;
    if (batch < 1 || batch > KV2D_MAX_BATCH)
        return fail(KV2D_ERR_INVALID_ARG, "batch %d not in [1, %d]", batch, KV2D_MAX_BATCH);
    if (!cc || !cc->n_segs || !cc->used_bytes || !cc->comp_end)
        return fail(KV2D_ERR_INVALID_ARG, "compressed cache has a NULL pointer");
    if (!staged || !staged->n_segs || !staged->used_bytes || !staged->comp_end)
        return fail(KV2D_ERR_INVALID_ARG, "staged record has a NULL pointer");
    const int units = batch * p->num_kv_heads;
    cudaError_t e = launch_publish(units, batch, staged->n_segs, staged->used_bytes, staged->comp_end,
                                   cc->n_segs, cc->used_bytes, cc->comp_end, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return fail(KV2D_ERR_CUDA, "switch launch: %s", cudaGetErrorString(e));
    return ok();
}

kv2d_status kv2d_append(const kv2d_params* p, int batch, const kv2d_dense* kv, const void* k_new,
                        const void* v_new, int32_t* seq_len_dev, void* ws, size_t ws_bytes,
                        void* stream) {
    kv2d_status st = check_params(p);
    if (st != KV2D_OK) return st;
    if (batch < 1 || batch > KV2D_MAX_BATCH)
        return fail(KV2D_ERR_INVALID_ARG, "batch %d not in [1, %d]", batch, KV2D_MAX_BATCH);
    if ((st = check_dense(p, batch, kv)) != KV2D_OK) return st;
    if (!k_new || !v_new || !seq_len_dev || !aligned(k_new, 16) || !aligned(v_new, 16))
        return fail(KV2D_ERR_INVALID_ARG, "k_new / v_new / seq_len must be 16-byte aligned device pointers");
    if (!ws || !aligned(ws, 256) || ws_bytes < 256)
        return fail(KV2D_ERR_WORKSPACE, "append needs a 256-byte aligned workspace of 256 bytes");
    AppendLaunch L;
    L.batch = batch;
    L.Hkv = p->num_kv_heads;
    L.dv = view_of(p, kv);
    L.k = static_cast<__half*>(kv->k);
    L.v = static_cast<__half*>(kv->v);
    L.k_new = static_cast<const __half*>(k_new);
    L.v_new = static_cast<const __half*>(v_new);
    L.seq_len = seq_len_dev;
    L.status = static_cast<uint32_t*>(ws);
    cudaError_t e = launch_append(L, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return fail(KV2D_ERR_CUDA, "append launch: %s", cudaGetErrorString(e));
    return ok();
}

kv2d_status kv2d_decode_attn(const kv2d_params* p, int batch, const kv2d_ccache* cc,
                             const kv2d_dense* kv, const int32_t* seq_len_dev,
                             int32_t max_seq_len_host, const void* q, void* out, void* ws,
                             size_t ws_bytes, void* stream) {
    kv2d_status st = check_params(p);
    if (st != KV2D_OK) return st;
    const UnitShape sh = shape_of(p);
    if (sh.G != 2 && sh.G != 4 && sh.G != 8)
        return fail(KV2D_ERR_UNSUPPORTED, "decode runs G = Hq/Hkv in {2, 4, 8}, got %d", sh.G);
    if (batch < 1 || batch > KV2D_MAX_BATCH)
        return fail(KV2D_ERR_INVALID_ARG, "batch %d not in [1, %d]", batch, KV2D_MAX_BATCH);
    if ((st = check_dense(p, batch, kv)) != KV2D_OK) return st;
    if (!cc || !cc->arena || !cc->desc || !cc->n_segs || !cc->used_bytes || !cc->comp_end)
        return fail(KV2D_ERR_INVALID_ARG, "compressed cache has a NULL pointer");
    if (!aligned(cc->arena, 256) || cc->arena_stride % 256)
        return fail(KV2D_ERR_INVALID_ARG, "arena must be 256-byte aligned with a multiple-of-256 stride");
    if (!seq_len_dev || !q || !out || !aligned(q, 16) || !aligned(out, 16))
        return fail(KV2D_ERR_INVALID_ARG, "seq_len / q / out must be 16-byte aligned device pointers");
    if (max_seq_len_host < 0 || max_seq_len_host > dense_capacity(kv))
        return fail(KV2D_ERR_INVALID_ARG, "max_seq_len %d outside [0, capacity]", max_seq_len_host);
    const DecodeLayout WL = decode_layout(p, batch);
    if (!ws || !aligned(ws, 256) || ws_bytes < WL.total)
        return fail(KV2D_ERR_WORKSPACE, "decode workspace %zu bytes, need %zu (256-byte aligned)",
                    ws_bytes, WL.total);
    uint8_t* w = static_cast<uint8_t*>(ws);
    DecodeLaunch L;
    L.shp = sh;
    L.batch = batch;
    L.scale_log2 = sh.c2;
    L.dv = view_of(p, kv);
    L.arena = static_cast<const uint8_t*>(cc->arena);
    L.arena_stride = cc->arena_stride;
    L.desc = static_cast<const uint64_t*>(cc->desc);
    L.max_segs = cc->max_segs;
    L.n_segs = cc->n_segs;
    L.used_bytes = cc->used_bytes;
    L.comp_end = cc->comp_end;
    L.seq_len = seq_len_dev;
    L.q = static_cast<const __half*>(q);
    L.out = static_cast<__half*>(out);
    L.nctas = decode_cta_count(batch * sh.Hkv, max_seq_len_host, num_sms(), &L.kps);
    L.tbl_cap = g_dec_table_cap.load();
    L.part = reinterpret_cast<float*>(w + WL.part);
    L.ticket = reinterpret_cast<uint32_t*>(w + WL.ticket);
    L.status = reinterpret_cast<uint32_t*>(w);
    cudaError_t e = launch_decode(L, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return fail(KV2D_ERR_CUDA, "decode launch: %s", cudaGetErrorString(e));
    return ok();
}

kv2d_status kv2d_decode_attn_noalloc(const kv2d_params* p, int batch, const kv2d_ccache* cc,
                                     const kv2d_dense* kv, const int32_t* seq_len_dev,
                                     int32_t max_seq_len_host, const void* q, void* out,
                                     uint32_t* status_dev, void* stream) {
    kv2d_status st = check_params(p);
    if (st != KV2D_OK) return st;
    const UnitShape sh = shape_of(p);
    if (sh.G != 2 && sh.G != 4 && sh.G != 8)
        return fail(KV2D_ERR_UNSUPPORTED, "decode runs G = Hq/Hkv in {2, 4, 8}, got %d", sh.G);
    if (batch < 1 || batch > KV2D_MAX_BATCH)
        return fail(KV2D_ERR_INVALID_ARG, "batch %d not in [1, %d]", batch, KV2D_MAX_BATCH);
    if ((st = check_dense(p, batch, kv)) != KV2D_OK) return st;
    if (!cc || !cc->arena || !cc->desc || !cc->n_segs || !cc->used_bytes || !cc->comp_end)
        return fail(KV2D_ERR_INVALID_ARG, "compressed cache has a NULL pointer");
    if (!aligned(cc->arena, 256) || cc->arena_stride % 256)
        return fail(KV2D_ERR_INVALID_ARG, "arena must be 256-byte aligned with a multiple-of-256 stride");
    if (!seq_len_dev || !q || !out || !aligned(q, 16) || !aligned(out, 16))
        return fail(KV2D_ERR_INVALID_ARG, "seq_len / q / out must be 16-byte aligned device pointers");
    if (status_dev && !aligned(status_dev, 4))
        return fail(KV2D_ERR_INVALID_ARG, "status_dev must be 4-byte aligned");
    if (max_seq_len_host < 0 || max_seq_len_host > dense_capacity(kv))
        return fail(KV2D_ERR_INVALID_ARG, "max_seq_len %d outside [0, capacity]", max_seq_len_host);
    const int64_t units = static_cast<int64_t>(batch) * sh.Hkv;
    int kps = 0;
    const int nctas = decode_cta_count(static_cast<int>(units), max_seq_len_host, num_sms(), &kps);
    const size_t part_bytes = static_cast<size_t>(units + nctas) * sh.G * (kHeadDim + 4) * 4;
    if (static_cast<size_t>(units) * 4 > kNoAllocTicketBytes || kNoAllocPartOff + part_bytes > kNoAllocScratchBytes)
        return fail(KV2D_ERR_WORKSPACE,
                    "decode needs %zu bytes of scratch partials and %lld tickets for %lld units on %d "
                    "CTAs; the built-in scratch holds %zu bytes of partials and %zu tickets",
                    part_bytes, static_cast<long long>(units), static_cast<long long>(units), nctas,
                    kNoAllocScratchBytes - kNoAllocPartOff, kNoAllocTicketBytes / 4);
    void* scratch = nullptr;
    if ((st = noalloc_scratch(&scratch)) != KV2D_OK) return st;
    uint8_t* w = static_cast<uint8_t*>(scratch);
    DecodeLaunch L;
    L.shp = sh;
    L.batch = batch;
    L.scale_log2 = sh.c2;
    L.dv = view_of(p, kv);
    L.arena = static_cast<const uint8_t*>(cc->arena);
    L.arena_stride = cc->arena_stride;
    L.desc = static_cast<const uint64_t*>(cc->desc);
    L.max_segs = cc->max_segs;
    L.n_segs = cc->n_segs;
    L.used_bytes = cc->used_bytes;
    L.comp_end = cc->comp_end;
    L.seq_len = seq_len_dev;
    L.q = static_cast<const __half*>(q);
    L.out = static_cast<__half*>(out);
    L.nctas = nctas;
    L.kps = kps;
    L.tbl_cap = g_dec_table_cap.load();
    L.part = reinterpret_cast<float*>(w + kNoAllocPartOff);
    L.ticket = reinterpret_cast<uint32_t*>(w + kNoAllocTicketOff);   // left at zero by every call
    L.status = status_dev;   // NULL: device faults are not recorded anywhere
    cudaError_t e = launch_decode(L, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return fail(KV2D_ERR_CUDA, "decode launch: %s", cudaGetErrorString(e));
    return ok();
}

kv2d_status kv2d_decode_attn_select(const kv2d_params* p, int batch, const kv2d_ccache* cc,
                                    const kv2d_dense* kv, const int32_t* seq_len_dev,
                                    int32_t max_seq_len_host, const void* q, void* out,
                                    float select_rate, void* ws, size_t ws_bytes, float* dbg_score,
                                    uint8_t* dbg_sel, void* stream) {
    kv2d_status st = check_params(p);
    if (st != KV2D_OK) return st;
    const UnitShape sh = shape_of(p);
    if (sh.G > 8) return fail(KV2D_ERR_UNSUPPORTED, "token-selection decode runs G <= 8, got %d", sh.G);
    if (batch < 1 || batch > KV2D_MAX_BATCH)
        return fail(KV2D_ERR_INVALID_ARG, "batch %d not in [1, %d]", batch, KV2D_MAX_BATCH);
    if ((st = check_dense(p, batch, kv)) != KV2D_OK) return st;
    if (!cc || !cc->arena || !cc->desc || !cc->n_segs || !cc->used_bytes || !cc->comp_end)
        return fail(KV2D_ERR_INVALID_ARG, "compressed cache has a NULL pointer");
    if (!aligned(cc->arena, 256) || cc->arena_stride % 256)
        return fail(KV2D_ERR_INVALID_ARG, "arena must be 256-byte aligned with a multiple-of-256 stride");
    if (!seq_len_dev || !q || !out || !aligned(q, 16) || !aligned(out, 16))
        return fail(KV2D_ERR_INVALID_ARG, "seq_len / q / out must be 16-byte aligned device pointers");
    if (max_seq_len_host < 0 || max_seq_len_host > dense_capacity(kv))
        return fail(KV2D_ERR_INVALID_ARG, "max_seq_len %d outside [0, capacity]", max_seq_len_host);
    if (!(select_rate > 0.f) || !std::isfinite(select_rate))
        return fail(KV2D_ERR_INVALID_ARG, "select_rate must be a positive finite fraction");
    if (cc->arena_stride >= (int64_t(1) << 36))
        return fail(KV2D_ERR_UNSUPPORTED, "selection decode runs arenas below 64 GB per unit");
    const SelectLayout WL = select_layout(p, batch, max_seq_len_host);
    if (WL.nreg > 12000)
        return fail(KV2D_ERR_UNSUPPORTED, "selection decode runs at most 12000 x 64 segments per sequence");
    if (!ws || !aligned(ws, 256) || ws_bytes < WL.total)
        return fail(KV2D_ERR_WORKSPACE, "selection decode workspace %zu bytes, need %zu (256-byte aligned)",
                    ws_bytes, WL.total);
    uint8_t* w = static_cast<uint8_t*>(ws);
    DecodeSelectLaunch L;
    L.shp = sh;
    L.batch = batch;
    L.scale = eff_scale(p);
    L.rate = static_cast<double>(select_rate);
    L.dv = view_of(p, kv);
    L.arena = static_cast<const uint8_t*>(cc->arena);
    L.arena_stride = cc->arena_stride;
    L.desc = static_cast<const uint64_t*>(cc->desc);
    L.max_segs = cc->max_segs;
    L.n_segs = cc->n_segs;
    L.used_bytes = cc->used_bytes;
    L.comp_end = cc->comp_end;
    L.seq_len = seq_len_dev;
    L.q = static_cast<const __half*>(q);
    L.out = static_cast<__half*>(out);
    L.slot_stride = WL.slot_stride;
    L.cscore = reinterpret_cast<float*>(w + WL.cscore);
    L.cslot = reinterpret_cast<int32_t*>(w + WL.cslot);
    L.ccount = reinterpret_cast<int32_t*>(w + WL.ccount);
    L.nreg_max = WL.nreg;
    L.gather = reinterpret_cast<uint2*>(w + WL.gather);
    L.nsel = reinterpret_cast<int32_t*>(w + WL.nsel);
    L.part = reinterpret_cast<float*>(w + WL.part);
    L.ticket = reinterpret_cast<uint32_t*>(w + WL.ticket);
    L.nchunk = sel2_chunks(batch * sh.Hkv, num_sms());
    L.dbg_score = dbg_score;
    L.dbg_sel = dbg_sel;
    L.status = reinterpret_cast<uint32_t*>(w);
    cudaError_t e = launch_decode_select(L, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return fail(KV2D_ERR_CUDA, "selection decode launch: %s", cudaGetErrorString(e));
    return ok();
}

kv2d_status kv2d_read_status(void* ws, void* stream, uint32_t* bits) {
    if (!ws) return fail(KV2D_ERR_INVALID_ARG, "workspace is NULL");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint32_t v = 0;
    cudaError_t e = cudaStreamSynchronize(s);
    if (e == cudaSuccess) e = cudaMemcpy(&v, ws, sizeof v, cudaMemcpyDeviceToHost);
    if (e == cudaSuccess) e = cudaMemset(ws, 0, sizeof v);
    if (e != cudaSuccess) return fail(KV2D_ERR_CUDA, "status read: %s", cudaGetErrorString(e));
    if (bits) *bits = v;
    if (v) return fail(KV2D_ERR_DEVICE_FAULT, "device status bits 0x%x", v);
    return ok();
}

const char* kv2d_last_error(void) { return g_err.c_str(); }

const char* kv2d_version(void) { return "kv2d 0.1.0 (sm_100a)"; }

kv2d_status kv2d_set_decode_table_cap(int cap) {
    if (cap != 0 && (cap < 32 || cap > kDecTableMax))
        return fail(KV2D_ERR_INVALID_ARG, "decode table cap %d not 0 or in [32, %d]", cap, kDecTableMax);
    g_dec_table_cap.store(cap == 0 ? kDecTableMax : cap);
    return ok();
}

kv2d_status kv2d_profile_enable(int on) {
    std::lock_guard<std::mutex> lk(g_prof_mu);
    g_prof_on = on != 0;
    return ok();
}

int kv2d_profile_read(double* ms, int64_t* launches, int max_stages) {
    std::vector<ProfRec> done;
    {
        std::lock_guard<std::mutex> lk(g_prof_mu);
        done.swap(g_prof_done);
    }
    const int n = std::min(max_stages, static_cast<int>(kProfStages));
    for (int i = 0; i < n; ++i) {
        if (ms) ms[i] = 0.0;
        if (launches) launches[i] = 0;
    }
    for (const ProfRec& r : done) {
        float t = 0.f;
        if (cudaEventSynchronize(r.b) == cudaSuccess && cudaEventElapsedTime(&t, r.a, r.b) == cudaSuccess &&
            r.stage < n) {
            if (ms) ms[r.stage] += t;
            if (launches) launches[r.stage] += 1;
        }
        cudaEventDestroy(r.a);
        cudaEventDestroy(r.b);
    }
    return n;
}

const char* kv2d_profile_stage_name(int stage) {
    return (stage >= 0 && stage < kProfStages) ? kStageNames[stage] : nullptr;
}

}  // extern "C"
