// kernels.h -- host-side launch interface between the C ABI (api.cu) and the
// kernel files.  Internal to the library.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

#include "common.cuh"

namespace kv2d {

// Kernel stages the optional event profiler tells apart.
enum ProfStage {
    kProfPass1 = 0,
    kProfPass2,
    kProfChan,
    kProfSegSelect,
    kProfBudget,
    kProfPack,
    kProfAppend,
    kProfDecode,
    kProfSelScore,
    kProfSelTop,
    kProfSelAttn,
    kProfStages
};

// Records a CUDA event pair around one launch when profiling is on
// (defined in api.cu; a no-op otherwise).
void prof_begin(cudaStream_t s, int stage);
void prof_end(cudaStream_t s, int stage);

// Launches kernel on stream with programmatic stream serialization, so that
// its launch overlaps the tail of the previous kernel in the stream; every
// kernel calls pdl_wait() before it reads what earlier work wrote.
template <typename... KArgs, typename... Args>
cudaError_t launch_k(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                     Args&&... args) {
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg;
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

struct UnitShape {
    int32_t Hkv, Hq, G, W, GW, GWpad;
    int32_t S, r, c;
    float c2;   // softmax scale * log2(e)
    int32_t chunk_len, chunk_budget;   // Token2Chunk (chunk_len 0: plain top-r)
};

// ---- scoring (score.cu)
struct ScoreLaunch {
    SeqPlan plan;
    UnitShape shp;
    int batch;
    DenseView dv;
    const __half* qw;          // [B][Hq][W][d]
    CUtensorMap qmap;          // 2-D map over qw rows, box 64 x 64
    CUtensorMap kmap;          // 4-D map over K, box 64 x (128 | 16)
    int paged;
    int max_region;            // longest region of the call (tokens)
    int max_nseg;
    // workspace
    float* apart;              // [units][GWpad / 128][d]
    float2* part;              // [units][GWpad][nsplit1]
    int nsplit1, kps1;
    float* s;                  // [units][s_stride]
    int64_t s_stride;
    int nsplit2, kps2;
    double* g;                 // [units][g_stride]
    uint4* cmask;              // [units][g_stride]: bit x set iff channel x is kept
    int64_t g_stride;
    uint32_t* status;
    // debug
    float* dbg_a;
    float* dbg_lse;
    float* dbg_s;
    double* dbg_g;
    int64_t dbg_stride;
};
cudaError_t launch_scoring(const ScoreLaunch& L, cudaStream_t stream);
int score_pass1_smem_bytes();
int score_pass2_smem_bytes(int gwpad);

// ---- selection (select.cu)
struct SelectLaunch {
    SeqPlan plan;
    UnitShape shp;
    int batch, max_nseg;
    int64_t bytes[4];          // payload bytes per strategy
    int32_t order[4];          // strategies by (bytes, id)
    int all_full;              // beta >= 1
    const float* s;
    int64_t s_stride;
    const double* g;
    int64_t g_stride;
    uint8_t* tidx;             // [units][max_nseg][r]
    double* E;                 // [units][max_nseg][4]
    uint8_t* hull;             // [units][max_nseg][8]: nv, verts[4]
    double* eff;               // [units][max_nseg][3]
    int32_t* dbytes;           // [units][max_nseg][3]
    uint8_t* strat;            // [units][max_nseg]
    int32_t* unit_ok;          // [units]
    // compressed cache
    uint64_t* desc;            // [units][max_segs]
    int32_t max_segs;
    int32_t* n_segs;
    int64_t* used_bytes;
    int32_t* comp_end;
    // where the new bookkeeping goes; NULL: the live fields above (a staged
    // compression leaves the live ones untouched until it is published)
    int32_t* out_n_segs;
    int64_t* out_used_bytes;
    int32_t* out_comp_end;
    int64_t arena_stride;
    uint32_t* status;
    double* dbg_E;
    int32_t dbg_seg_stride;
};
cudaError_t launch_selection(const SelectLaunch& L, cudaStream_t stream);
cudaError_t launch_publish(int units, int batch, const int32_t* st_n_segs, const int64_t* st_used,
                           const int32_t* st_comp_end, int32_t* n_segs, int64_t* used, int32_t* comp_end,
                           cudaStream_t stream);

// ---- packing (pack.cu)
struct PackLaunch {
    SeqPlan plan;
    UnitShape shp;
    int batch, max_nseg;
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
cudaError_t launch_pack(const PackLaunch& L, cudaStream_t stream);

// ---- append and decode (decode.cu)
struct AppendLaunch {
    int batch, Hkv;
    DenseView dv;
    __half* k;
    __half* v;
    const __half* k_new;
    const __half* v_new;
    int32_t* seq_len;
    uint32_t* status;
};
cudaError_t launch_append(const AppendLaunch& L, cudaStream_t stream);

struct DecodeLaunch {
    UnitShape shp;
    int batch;
    float scale_log2;
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
    int nctas;                 // grid size, at most kMaxDecCtas
    int kps;                   // CTAs per unit, or 0: batch-wide byte shares
    int tbl_cap;               // blocks per block-table chunk, in [32, kDecTableMax]
    float* part;               // [nctas + units][G][4 + d]: M, L, 0, 0, O[d]
    uint32_t* ticket;          // [units]
    uint32_t* status;
};
constexpr int kMaxDecCtas = 512;
constexpr int kDecTableMax = 4096;
cudaError_t launch_decode(const DecodeLaunch& L, cudaStream_t stream);
int decode_cta_count(int units, int64_t max_seq_len, int num_sms, int* kps);

// ---- decode with decode-time token selection (stage2.cu)
struct DecodeSelectLaunch {
    UnitShape shp;
    int batch;
    float scale;               // softmax scale (natural log domain)
    double rate;               // token selection rate
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
    int64_t slot_stride;       // candidate slots per unit: (max_seq_len / S) * S
    float* cscore;             // [units][slot_stride]: scores compacted per region
    int32_t* cslot;            // [units][slot_stride]
    int32_t* ccount;           // [units][nreg_max]
    int nreg_max;              // regions of 64 segments per unit
    uint2* gather;             // [units][slot_stride]: kept items
    int32_t* nsel;             // [units]
    float* part;               // [units][nchunk][G][4 + d]
    uint32_t* ticket;          // [units]
    int nchunk;                // attention chunks per unit, <= kSel2MaxChunks
    float* dbg_score;
    uint8_t* dbg_sel;
    uint32_t* status;
};
constexpr int kSel2MaxChunks = 64;
cudaError_t launch_decode_select(const DecodeSelectLaunch& L, cudaStream_t stream);
int sel2_chunks(int units, int num_sms);
int sel2_regions(int64_t slot_stride, int S);

}  // namespace kv2d
