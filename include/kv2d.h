/*
 * kv2d.h -- C ABI of the kv2d library: dynamic two-dimensional KV-cache
 * compression and decode attention over the compressed cache, for NVIDIA
 * B200 (sm_100a).
 *
 * The method is the one of "MosaicKV: Serving Long-Context LLM with Dynamic
 * Two-D KV Cache Compression" (pith.science summary of arXiv 2607.00760):
 *   - Core claim: importance is identified for the elements of every KV
 *     vector and a compression strategy is chosen per KV-cache segment;
 *   - Fig. 5: the cache is partitioned into segments and a compression
 *     strategy is generated per segment;
 *   - Fig. 6: Stage-1 keeps the top important elements of each vector; a
 *     packed KV format and a flexible encoding hold the result;
 *   - Fig. 7 / Sec. 5.3 (PackedAttention): decode attention runs directly on
 *     the packed segments.
 * Token importance is the attention mass that a window of recent queries
 * gives each key, as in "KARA: Efficient Reasoning LLM Serving via
 * Sliding-Window KV Cache Compression" (pith.science review of arXiv
 * 2607.01237), "What carries the argument"; the same page's periodic
 * compression of the trailing region is what repeated kv2d_compress calls
 * over [comp_end, seq_len) implement.
 *
 * Where the pages leave a step open the library takes these readings:
 *   a_d    = mean over the G*W window rows of |q_d|            (per KV head)
 *   s_t    = sum over window rows of softmax weight on key t   (causal,
 *            normalised over the scored region [comp_end, seq_len))
 *   C_t    = the c channels of largest |k_t,d| * a_d, ties to the lower d
 *   g_t    = share of sum_d |k_t,d| a_d carried by the dropped channels
 *   R_j    = the r tokens of segment j with the largest s_t, ties to lower t
 *            (or, with chunk_len > 0, Kara's Token2Chunk variant: the top
 *            r - alpha tokens, then whole gaps between consecutive ones of
 *            span <= gamma by summed s_t while they fit alpha, then the best
 *            tokens left; "KARA" page, "What carries the argument")
 *   E_FULL = 0, E_TOK = sum_{t not in R} s_t, E_CH = sum_t s_t g_t,
 *   E_BOTH = E_TOK + sum_{t in R} s_t g_t            (lost attention mass)
 *   choice = greedy over each segment's lower convex hull in (bytes, E),
 *            steps in (efficiency desc, segment asc, step asc) order while
 *            they fit floor(beta * nseg * FULL_bytes), stopping at the first
 *            that does not; beta >= 1 keeps every segment FULL.
 *
 * Units.  One unit u = b * num_kv_heads + h is one (sequence, KV head).
 * Query head of (h, g) is h * G + g with G = num_q_heads / num_kv_heads.
 *
 * Memory.  Every buffer is allocated and owned by the caller; the library
 * never allocates device memory, never synchronises a stream inside
 * kv2d_compress / kv2d_append / kv2d_decode_attn, and keeps no state between
 * calls except a thread-local error string and two process-wide switches of
 * its aids (kv2d_profile_enable, kv2d_set_decode_table_cap); the fixed
 * scratch of kv2d_decode_attn_noalloc is described with that call.  All
 * device work is enqueued on the caller's stream.  fp16 means IEEE binary16.
 *
 * Errors.  Every entry point validates its arguments on the host before it
 * launches anything and returns a kv2d_status; kv2d_last_error() gives the
 * reason in words.  Faults that only the device can see (a block-table entry
 * out of range, a full arena, an exhausted wait) never trap: the kernel
 * skips the access and sets a status word in the workspace, which
 * kv2d_read_status() returns.
 */
#ifndef KV2D_H
#define KV2D_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define KV2D_API __attribute__((visibility("default")))
#else
#define KV2D_API
#endif

#define KV2D_MAX_BATCH 128

typedef enum kv2d_status {
    KV2D_OK = 0,
    KV2D_ERR_INVALID_ARG = 1,        /* a size, pointer or stride is wrong  */
    KV2D_ERR_BUDGET_INFEASIBLE = 2,  /* cheapest strategies exceed budget   */
    KV2D_ERR_WORKSPACE = 3,          /* ws too small or misaligned          */
    KV2D_ERR_CUDA = 4,               /* a CUDA runtime call failed          */
    KV2D_ERR_DEVICE_FAULT = 5,       /* device status word was set          */
    KV2D_ERR_UNSUPPORTED = 6,        /* valid but not built (e.g. d != 128) */
    KV2D_ERR_CAPACITY = 7            /* arena or descriptor table too small */
} kv2d_status;

/* Strategy ids stored in the descriptors. */
enum { KV2D_FULL = 0, KV2D_TOK = 1, KV2D_CH = 2, KV2D_BOTH = 3 };

/* Operations for kv2d_workspace_bytes. */
enum { KV2D_OP_COMPRESS = 0, KV2D_OP_DECODE = 1, KV2D_OP_APPEND = 2, KV2D_OP_DECODE_SELECT = 3 };

/* Device status bits (kv2d_read_status ORs them into *bits). */
enum {
    KV2D_DEV_BLOCK_TABLE = 1,   /* a block-table entry was out of range   */
    KV2D_DEV_CAPACITY = 2,      /* an arena would have overflowed          */
    KV2D_DEV_TIMEOUT = 4,       /* a bounded wait gave up                  */
    KV2D_DEV_SEQ_RANGE = 8,     /* a sequence length was out of range      */
    KV2D_DEV_BAD_MASK = 16      /* a channel keep-mask without exactly c
                                   bits (an internal invariant; the packed
                                   indices of that token were truncated)   */
};

typedef struct kv2d_params {
    int32_t head_dim;       /* d; this build runs d = 128                    */
    int32_t num_q_heads;    /* Hq                                            */
    int32_t num_kv_heads;   /* Hkv; G = Hq / Hkv must be 1, 2, 4 or 8        */
    int32_t segment_len;    /* S: a multiple of 16 in [16, 256]              */
    int32_t window;         /* W: window queries, 1 <= G*W <= 512            */
    int32_t keep_tokens;    /* r: 1 <= r <= S                                */
    int32_t keep_channels;  /* c: 1 <= c <= d                                */
    float budget;           /* beta > 0: byte budget / FULL bytes            */
    float scale;            /* softmax scale; 0 selects 1/sqrt(d)            */
    int32_t chunk_len;      /* Token2Chunk: longest chunk gamma in tokens,
                               3 <= gamma <= S; 0 = plain top-r              */
    int32_t chunk_budget;   /* Token2Chunk: tokens alpha that chunks may add
                               per segment, 1 <= alpha < r and r - alpha <=
                               33 (ignored when chunk_len is 0)              */
} kv2d_params;

/* Dense (uncompressed) K/V view of one layer.  Two layouts:
 *  contiguous (block_table == NULL): element (b, h, t, x) of K lives at
 *      k + b*stride_b + h*stride_h + t*stride_t + x  (fp16 elements);
 *      stride_t, stride_h, stride_b are multiples of 8; capacity = tokens per
 *      (b, h) row that the allocation holds.
 *  paged (block_table != NULL): a pool of num_blocks blocks laid out
 *      [num_blocks][Hkv][block_size][d]; token t of sequence b is row
 *      t % block_size of physical block block_table[b * max_blocks +
 *      t / block_size].  block_size is a multiple of 16 in [16, 256]. */
typedef struct kv2d_dense {
    void* k;
    void* v;
    int64_t stride_b, stride_h, stride_t;
    int32_t capacity;
    const int32_t* block_table;
    int32_t block_size;
    int32_t max_blocks;
    int64_t num_blocks;
} kv2d_dense;

/* Compressed cache of one layer (caller-owned device memory).
 *  arena:      units * arena_stride bytes; the unit's packed segments are
 *              appended at offset used_bytes[u]; base 256-byte aligned,
 *              arena_stride a multiple of 256 (see kv2d_arena_bytes).
 *  desc:       units * max_segs descriptors of 8 bytes:
 *              {uint32 offset/16, uint8 strategy, 3 zero bytes}.
 *  n_segs:     [units] int32, segments stored per unit.
 *  used_bytes: [units] int64, payload bytes stored per unit.
 *  comp_end:   [batch] int32, first token of sequence b that is not yet
 *              compressed (a multiple of S).
 * Zero n_segs, used_bytes and comp_end before the first compression. */
typedef struct kv2d_ccache {
    void* arena;
    int64_t arena_stride;
    void* desc;
    int32_t max_segs;
    int32_t* n_segs;
    int64_t* used_bytes;
    int32_t* comp_end;
} kv2d_ccache;

/* Optional intermediate results of kv2d_compress (device pointers; any may
 * be NULL).  Rows are per unit; region_stride >= the longest region of the
 * call (tokens), seg_stride >= its segment count.
 *  a   [units][d]                  float  window statistics a_d
 *  lse [batch][Hq][W]              float  natural-log normaliser of each
 *                                         window row over the region
 *  s   [units][region_stride]      float  token mass s_t, t - comp_end
 *  g   [units][region_stride]      double dropped-importance share g_t
 *  E   [units][seg_stride][4]      double error proxies per segment */
typedef struct kv2d_debug {
    float* a;
    float* lse;
    float* s;
    double* g;
    double* E;
    int64_t region_stride;
    int32_t seg_stride;
} kv2d_debug;

/* Payload bytes of one segment for strategy KV2D_FULL..KV2D_BOTH, every
 * section padded to 16 bytes (MosaicKV Fig. 6, packed KV format; layout:
 * FULL K[S][d] | V[S][d];  TOK tidx[r] | K[r][d] | V[r][d];
 * CH cidx[S][c] | Kval[S][c] | V[S][d];  BOTH tidx[r] | cidx[r][c] |
 * Kval[r][c] | V[r][d]; indices are uint8, ascending, segment-relative for
 * tidx).  Returns -1 for invalid params or strategy. */
KV2D_API int64_t kv2d_segment_bytes(const kv2d_params* p, int strategy);

/* Arena bytes per unit that always hold the compression of max_tokens
 * tokens at the params' budget, rounded up to 256.  -1 if invalid. */
KV2D_API int64_t kv2d_arena_bytes(const kv2d_params* p, int64_t max_tokens);

/* Workspace bytes for op (KV2D_OP_*) on a batch whose longest region
 * (compress) or sequence (decode) has max_tokens tokens.  0 if invalid. */
KV2D_API size_t kv2d_workspace_bytes(const kv2d_params* p, int op, int batch, int64_t max_tokens);

/* kv2d_compress -- compress, for every sequence b < batch and KV head, the
 * complete segments of the region [comp_end_host[b], seq_len_host[b]),
 * scored by the last W queries of that sequence (MosaicKV Fig. 5 and Fig. 6;
 * Kara's windowed scoring and periodic trailing-region compression).
 *   seq_len_host  [batch] host int32: tokens in the dense view.
 *   comp_end_host [batch] host int32: must equal the device cc->comp_end.
 *   kv            dense view (read only here).
 *   q_window      device fp16 [batch][Hq][W][d]: queries at positions
 *                 seq_len-W .. seq_len-1 (post-RoPE, like the keys).
 *   cc            compressed cache; segments are appended, n_segs,
 *                 used_bytes and comp_end advance on the device.
 *   ws, ws_bytes  device scratch of kv2d_workspace_bytes(p, COMPRESS, ...)
 *                 bytes, 256-byte aligned; its first 256 bytes hold the
 *                 status word (zero it once before first use).
 *   dbg           optional intermediate outputs, or NULL.
 * Host checks, before any launch: params (see kv2d_params), batch in
 * [1, KV2D_MAX_BATCH], W <= region length, segment and arena capacity, and
 * budget feasibility (nseg * cheapest bytes > budget ->
 * KV2D_ERR_BUDGET_INFEASIBLE).  Asynchronous on stream. */
KV2D_API kv2d_status kv2d_compress(const kv2d_params* p, int batch, const int32_t* seq_len_host,
                          const int32_t* comp_end_host, const kv2d_dense* kv,
                          const void* q_window, kv2d_ccache* cc, void* ws, size_t ws_bytes,
                          const kv2d_debug* dbg, void* stream);

/* Staged bookkeeping of a compression that is not yet published (device
 * memory, caller-owned): n_segs [units], used_bytes [units] (8-byte
 * aligned), comp_end [batch]. */
typedef struct kv2d_staged {
    int32_t* n_segs;
    int64_t* used_bytes;
    int32_t* comp_end;
} kv2d_staged;

/* kv2d_compress_staged / kv2d_switch -- compression that does not block
 * decode (MosaicKV Fig. 1 and Fig. 5: a switching mechanism replaces the
 * temporary version of a new segment with the compressed one without
 * blocking the decode stage; here the temporary version is the dense view
 * itself, so no CPU copy is involved).
 *   kv2d_compress_staged does what kv2d_compress does, but writes the new
 *   segments' bookkeeping into *staged and leaves cc->n_segs, used_bytes
 *   and comp_end untouched: the new packed bytes go past used_bytes and the
 *   new descriptors past n_segs, which decode never reads.  It may run on
 *   a second stream while kv2d_decode_attn / kv2d_append run on the decode
 *   stream: decode keeps attending the old segments and reads the tokens
 *   being compressed from the dense view (the region [comp_end, seq_len) a
 *   compression reads is never written by append).  *staged first receives
 *   the live values (stream-ordered copies), then the new ones.
 *   kv2d_switch publishes *staged as the live bookkeeping with one small
 *   kernel on the given stream.  The caller orders it after the staged
 *   compression (an event) and before the next decode that should see the
 *   new segments, and issues no other compression of the same cache until
 *   the switch.  Arguments and errors otherwise as kv2d_compress. */
KV2D_API kv2d_status kv2d_compress_staged(const kv2d_params* p, int batch,
                                          const int32_t* seq_len_host, const int32_t* comp_end_host,
                                          const kv2d_dense* kv, const void* q_window,
                                          kv2d_ccache* cc, const kv2d_staged* staged, void* ws,
                                          size_t ws_bytes, const kv2d_debug* dbg, void* stream);
KV2D_API kv2d_status kv2d_switch(const kv2d_params* p, int batch, kv2d_ccache* cc,
                                 const kv2d_staged* staged, void* stream);

/* kv2d_append -- write one new token per (sequence, KV head) into the dense
 * view at position seq_len_dev[b], then increment seq_len_dev[b] (the
 * decode stage's KV growth that later compressions consume; MosaicKV
 * Fig. 1, recompressing new segments).
 *   k_new, v_new  device fp16 [batch][Hkv][d].
 *   seq_len_dev   device int32 [batch], updated in place.
 *   ws            at least kv2d_workspace_bytes(p, APPEND, ...) bytes; a
 *                 write beyond capacity or the block table is skipped and
 *                 sets KV2D_DEV_SEQ_RANGE / KV2D_DEV_BLOCK_TABLE. */
KV2D_API kv2d_status kv2d_append(const kv2d_params* p, int batch, const kv2d_dense* kv, const void* k_new,
                        const void* v_new, int32_t* seq_len_dev, void* ws, size_t ws_bytes,
                        void* stream);

/* kv2d_decode_attn -- attention of each query head over its unit's
 * compressed segments [0, comp_end) and dense tokens [comp_end, seq_len)
 * (MosaicKV Sec. 5.3, PackedAttention):
 *   FULL/TOK/dense: logit = scale * q . k;   CH/BOTH: logit = scale *
 *   sum_j q[cidx_j] * Kval_j (dropped channels add nothing); softmax over
 *   every kept token; out = sum_t p_t v_t.
 *   seq_len_dev       device int32 [batch].
 *   max_seq_len_host  host upper bound of seq_len (fixes the grid, so the
 *                     call can be captured in a CUDA graph).
 *   q                 device fp16 [batch][Hq][d].
 *   out               device fp16 [batch][Hq][d].
 *   ws, ws_bytes      kv2d_workspace_bytes(p, DECODE, batch, max_seq_len)
 *                     bytes; per-CTA partials and per-unit tickets live
 *                     here.
 *                     Zero it once before its first use; every completed
 *                     call leaves the tickets at zero again.
 * Deterministic: the batch's bytes are cut into one share per CTA (a
 * function of the data and the SM count only); fixed merge order.
 * If a call sets KV2D_DEV_TIMEOUT (a copy into shared memory never
 * completed), its outputs are undefined. */
KV2D_API kv2d_status kv2d_decode_attn(const kv2d_params* p, int batch, const kv2d_ccache* cc,
                             const kv2d_dense* kv, const int32_t* seq_len_dev,
                             int32_t max_seq_len_host, const void* q, void* out, void* ws,
                             size_t ws_bytes, void* stream);

/* kv2d_decode_attn_select -- decode attention with decode-time,
 * query-aware token selection over the packed segments (MosaicKV Fig. 6
 * caption: stage 2 runs during the decode stage before each attention
 * layer; Sec. 5.3, PackedAttention: sequence compression and attention in
 * every decode layer; Fig. 8: token selection rates of 6.25 % and 12.5 %).
 * Readings the library takes where the pages give no rule:
 *   candidates  every token the unit's packed segments keep, slot j*S + i
 *               for token i of segment j; the dense tail [comp_end,
 *               seq_len) is always attended;
 *   score       the largest over the unit's G query heads of the logit
 *               scale * q_g . k (the stored key: whole for FULL / TOK, its
 *               kept channels for CH / BOTH), in fp32;
 *   count       n_sel = min(candidates, ceil(select_rate * n_segs * S)),
 *               select_rate taken as the double of the float given;
 *   choice      the n_sel largest scores, ties to the lower slot;
 *   attention   softmax of each head over the kept candidates and the
 *               dense tail; out = sum_t p_t v_t (fp16).
 *   select_rate       > 0 and finite; >= 1 keeps every candidate (the
 *                     result is then kv2d_decode_attn's, up to rounding).
 *   ws, ws_bytes      kv2d_workspace_bytes(p, KV2D_OP_DECODE_SELECT, batch,
 *                     max_seq_len_host) bytes, 256-byte aligned; zero it
 *                     once before first use (tickets return to zero after
 *                     every completed call).
 *   dbg_score, dbg_sel  optional device outputs [units][slots], slots =
 *                     (max_seq_len_host / S) * S rounded up to a multiple
 *                     of 4: the fp32 score of every candidate slot (-inf
 *                     past a segment's kept tokens) and a 0/1 flag per slot
 *                     (1 = kept); written for slots < n_segs * S.
 * Other arguments and errors as kv2d_decode_attn; G <= 8. */
KV2D_API kv2d_status kv2d_decode_attn_select(const kv2d_params* p, int batch,
                                             const kv2d_ccache* cc, const kv2d_dense* kv,
                                             const int32_t* seq_len_dev, int32_t max_seq_len_host,
                                             const void* q, void* out, float select_rate,
                                             void* ws, size_t ws_bytes, float* dbg_score,
                                             uint8_t* dbg_sel, void* stream);

/* kv2d_decode_attn_noalloc -- the same decode attention as kv2d_decode_attn,
 * for callers that cannot obtain device memory at all: a plugin that runs
 * inside a host process which owns every allocation, a runtime whose memory
 * plan is fixed before the first request, or code that must not call
 * cudaMalloc because that call can synchronise the device in the middle of a
 * latency-critical loop.  There is no counterpart on the pages; it is an
 * interface convenience only.
 *   It takes no workspace.  Its per-CTA partials and per-unit tickets live
 *   in a fixed 8 MiB array in the library's own device memory, which every
 *   GPU that loads the library holds until the process exits.  Its layout
 *   is the same for every call: a ticket per unit in a fixed 64 KiB region
 *   (at most 16384 units, batch x Hkv), then the partials, (units + CTAs) x
 *   G x (d + 4) x 4 bytes (CTAs <= the SM count) in the remaining
 *   8 MiB - 64 KiB - 256 bytes; larger calls return KV2D_ERR_WORKSPACE
 *   before launching.
 *   The first call on each device looks up the array's device address with
 *   the CUDA runtime (which makes the device's primary context current) and
 *   zeroes the ticket region with a synchronous cudaMemset; make that first
 *   call outside any stream capture.  The address is kept per device
 *   together with the id of the context it belongs to, and the set-up is
 *   repeated when that context has changed (after cudaDeviceReset).
 *   All calls on a device share the one array and each leaves its partials
 *   behind; every completed call leaves its per-unit tickets at zero again,
 *   and no call writes anything else into the ticket region.  Calls whose
 *   kernels overlap on the GPU (two streams, or two host threads) race on the
 *   array and give wrong results: serialise them.
 *   status_dev: optional device uint32; device-side faults OR their
 *   KV2D_DEV_* bits into it.  NULL: faults are not recorded anywhere.
 * Other arguments, layouts and errors as kv2d_decode_attn.  Allocates no
 * memory: no cudaMalloc / cudaFree and no allocating library call. */
KV2D_API kv2d_status kv2d_decode_attn_noalloc(const kv2d_params* p, int batch,
                                              const kv2d_ccache* cc, const kv2d_dense* kv,
                                              const int32_t* seq_len_dev, int32_t max_seq_len_host,
                                              const void* q, void* out, uint32_t* status_dev,
                                              void* stream);

/* Synchronises stream, returns the device status bits of ws in *bits and
 * clears them.  KV2D_ERR_DEVICE_FAULT if any bit was set. */
KV2D_API kv2d_status kv2d_read_status(void* ws, void* stream, uint32_t* bits);

/* Optional event profiler (a tracing aid, off by default).  While enabled,
 * every kernel launch of every call is bracketed by a CUDA event pair on the
 * caller's stream.  kv2d_profile_read() waits for those events, writes per
 * stage the summed milliseconds (ms[i]) and launch counts (launches[i]) for
 * the first max_stages stages, forgets them, and returns the number of
 * stages; kv2d_profile_stage_name() names stage i (NULL past the end). */
KV2D_API kv2d_status kv2d_profile_enable(int on);
KV2D_API int kv2d_profile_read(double* ms, int64_t* launches, int max_stages);
KV2D_API const char* kv2d_profile_stage_name(int stage);

/* Testing aid: caps the number of blocks (8-token slices of segments) the
 * decode kernel tables per chunk of a CTA's share (cap in [32, 4096]; 0
 * restores the default 4096), so that small inputs reach the path that
 * handles shares larger than one chunk.  Affects later decode calls of the
 * process; results do not depend on it.  KV2D_ERR_INVALID_ARG outside the
 * range. */
KV2D_API kv2d_status kv2d_set_decode_table_cap(int cap);

/* Human-readable reason of the calling thread's last non-OK status. */
KV2D_API const char* kv2d_last_error(void);

/* Library version string. */
KV2D_API const char* kv2d_version(void);

#ifdef __cplusplus
}
#endif
#endif /* KV2D_H */
