/*
 * minfer.h -- C ABI of libminfer.so: MInference dynamic sparse attention
 * prefill (MInference 1.0, arXiv 2407.02490) on NVIDIA B200 (sm_100a).
 *
 * The method (MInference 1.0 abstract; hotpaper.ai summary "key idea";
 * aifetchly "MInference 1.0 Guide", "The Three Fundamental Attention
 * Topologies" and "Technical Deep Dive") has two stages per attention head:
 *   1. an online sparse index: Vertical-Slash (VS) heads score every key
 *      column and every diagonal from the last `last_q` queries and keep the
 *      top ones; Block-Sparse (BS) heads score 64-token mean-pooled query and
 *      key blocks and keep the top key blocks per query block;
 *   2. causal softmax attention computed only over the selected columns and
 *      diagonals, blocks, or (A-shape heads) sink tokens plus a local window.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - q is [Hq][N][d], k and v are [Hkv][N][d], out is [Hq][N][d]: contiguous
 *    row-major bf16 (mi_bf16 = raw bf16 bits) in DEVICE memory owned by the
 *    caller.  Query head h reads KV head floor(h * Hkv / Hq) (grouped-query
 *    attention, contiguous groups).
 *  - Supported shapes: d in {64, 128}; N a multiple of 64 with N >= 64;
 *    Hq a multiple of Hkv; 1 <= Hq <= MI_MAX_HEADS.  Others return
 *    MI_ERR_UNSUPPORTED (shape) or MI_ERR_INVALID_ARG (inconsistent).
 *  - `heads` is a HOST array of `n_heads` query-head ids (each processed at
 *    most once); NULL means all Hq heads in order.  Per-head index arrays
 *    (v_idx, s_idx, blk_idx, blk_cnt, scores) are indexed by POSITION in that
 *    list; out / lse are indexed by absolute head.  Heads not listed are not
 *    touched.
 *  - `scale` is the softmax scale; pass 0 for the default 1/sqrt(d).
 *  - `ws` / `ws_bytes`: caller-owned device workspace, at least the size
 *    mi_workspace_bytes() returns for the same arguments, 256-byte aligned.
 *    The library allocates no memory of any kind.
 *  - `stream` is a cudaStream_t (as void*); all work is enqueued on it,
 *    asynchronously.  No entry point synchronises the device or the stream
 *    or copies device data to the host.
 *  - Every entry point validates its arguments on the host first.  On any
 *    error nothing is launched and the status says why; MI_ERR_CUDA keeps the
 *    cudaError_t in thread-local storage (mi_last_cuda_error()).
 *  - `err_count` (optional, device int32, may be NULL): the attention entry
 *    points add the number of index entries they skipped (out of range) to
 *    it; if a device-side wait ever gives up (a bounded wait, never expected
 *    in a correct run) bit 30 is set in it.
 *  - Budgets larger than the candidate count are clamped (vertical_size and
 *    slash_size to N, topk to the number of causal blocks): "budgets that
 *    cover everything" give dense causal attention.
 */
#ifndef MINFER_H
#define MINFER_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t mi_bf16; /* raw bf16 bit pattern */

enum {
    MI_OK = 0,
    MI_ERR_INVALID_ARG = 1, /* null pointer, negative size, Hq % Hkv != 0, bad head id */
    MI_ERR_UNSUPPORTED = 2, /* d not in {64,128}, N % 64 != 0, N < last_q, too many heads */
    MI_ERR_WORKSPACE = 3,   /* ws too small or misaligned */
    MI_ERR_CUDA = 4         /* a CUDA call failed; see mi_last_cuda_error() */
};

/* Per-head patterns of the router.  DENSE is plain causal attention over every
 * key j <= i: the class the offline profiler assigns to the few heads no
 * sparse pattern fits (guide, "Phase 1: The Offline Pattern Profiler" and
 * "Phase 2: The Online Dynamic Kernel Router"), and the prefill MInference is
 * measured against (guide, "Prefill Latency Benchmark"). */
enum { MI_PATTERN_ASHAPE = 0, MI_PATTERN_VS = 1, MI_PATTERN_BS = 2, MI_PATTERN_DENSE = 3 };

enum {
    MI_OP_VS_INDEX = 1,
    MI_OP_BS_INDEX = 2,
    MI_OP_VS_ATTN = 3,
    MI_OP_BS_ATTN = 4,
    MI_OP_ASHAPE_ATTN = 5,
    MI_OP_DENSE_ATTN = 6
};

#define MI_MAX_HEADS 256
#define MI_BLOCK 64

/* How a Vertical-Slash head's selected diagonals become attended keys:
 *  MI_SLASH_BLOCKS -- every 64x64 tile a diagonal touches is computed whole
 *    (the tile lists of the guide's "Vertical-Slash Kernel Mechanics");
 *  MI_SLASH_RANGES -- diagonal o gives query block bq (rows 64 bq .. 64 bq + 63)
 *    the 64 keys 64 bq - o .. 64 bq + 63 - o, causally masked: the keys
 *    its rows reach along the diagonal, as one unaligned range per block
 *    (fewer keys than the tiles; see mi_vs_range_attn). */
enum { MI_SLASH_BLOCKS = 0, MI_SLASH_RANGES = 1 };

/* Per-pattern parameters of one layer (all heads of a pattern share them). */
typedef struct {
    int last_q;        /* VS: number of final queries that score columns/diagonals */
    int vertical_size; /* VS: columns kept per head */
    int slash_size;    /* VS: diagonals kept per head */
    int topk_blocks;   /* BS: key blocks kept per 64-row query block */
    int sink;          /* A-shape: keys 0..sink-1 always kept */
    int window;        /* A-shape: keys i-window+1 .. i kept for row i */
    int slash_tiles;   /* VS: MI_SLASH_BLOCKS (0, the default) or MI_SLASH_RANGES */
} mi_params;

/* Stage boundaries recorded by mi_prefill_layer when stage_events != NULL:
 * START | index kernels | INDEX_DONE | slash/vertical prep | PREP_DONE |
 * the one sparse-attention launch | ATTN_DONE. */
enum {
    MI_STAGE_START = 0,
    MI_STAGE_INDEX_DONE = 1,
    MI_STAGE_PREP_DONE = 2,
    MI_STAGE_ATTN_DONE = 3,
    MI_STAGE_EVENTS = 4
};

/* Static description of a status code; never NULL. */
const char* mi_status_str(int status);

/* cudaError_t of the last MI_ERR_CUDA returned on this thread (0 if none). */
int mi_last_cuda_error(void);

/* Library version, e.g. "minfer 0.1 sm_100a". */
const char* mi_version(void);

/*
 * Workspace bytes for one call of `op` with these shapes (n_heads <= 0 means
 * all Hq heads).  Arguments the op does not use are ignored.  Returns 0 for
 * arguments the op would reject.
 */
size_t mi_workspace_bytes(int op, int Hq, int Hkv, int N, int d, int n_heads, int last_q,
                          int vertical_size, int slash_size, int topk_blocks);

/*
 * Workspace bytes for mi_prefill_layer.  `pattern` is the host pattern table
 * [Hq] (NULL: budget for any table).
 */
size_t mi_prefill_workspace_bytes(int Hq, int Hkv, int N, int d, const int8_t* pattern,
                                  const mi_params* p);

/*
 * Vertical-Slash index (hotpaper.ai "key idea"; guide "2. The Vertical-Slash
 * Pattern").  For each listed head h and each of the last L = last_q rows
 * i = N-L .. N-1: row softmax of scale * q_i . k_j over j <= i; vertical[j]
 * sums the probabilities of column j over the L rows, slash[o] sums those of
 * diagonal o = i - j.  The products q_i . k_j run on the tensor cores (exact
 * bf16 products, fp32 accumulation); the softmax argument and the column and
 * diagonal sums are carried to fp64 accuracy.  Scores are ranked as fp32.
 * The top vertical_size columns and top slash_size diagonals (ties: lower
 * index first) are written sorted ascending:
 *   v_idx [n_heads][vertical_size], s_idx [n_heads][slash_size] (int32,
 *   device); entries past min(budget, N) are set to -1.
 *   v_score, s_score [n_heads][N] fp32 (device, optional): the scores.
 * Requires 1 <= last_q <= N.
 */
int mi_vs_index(const mi_bf16* q, const mi_bf16* k, int Hq, int Hkv, int N, int d, float scale,
                int last_q, int vertical_size, int slash_size, const int32_t* heads, int n_heads,
                int32_t* v_idx, int32_t* s_idx, float* v_score, float* s_score, void* ws,
                size_t ws_bytes, void* stream);

/*
 * Block-Sparse index (hotpaper.ai "key idea": 64-token mean pooling; guide
 * "Block-Sparse Kernel Mechanics": block score against the mean key of each
 * block, keep the top-k).  Qm[b] / Km[b] are means of 64 rows; for query
 * block bq the candidates are key blocks bk <= bq with score
 * scale * Qm[bq] . Km[bk] (fp64 means and fp64 dot products).  The top
 * min(topk, bq+1) (ties: lower block first) are written sorted ascending:
 *   blk_idx [n_heads][N/64][topk] int32 (device; unused entries -1),
 *   blk_cnt [n_heads][N/64] int32 (device).
 * `block` must be 64.
 */
int mi_bs_index(const mi_bf16* q, const mi_bf16* k, int Hq, int Hkv, int N, int d, float scale,
                int block, int topk, const int32_t* heads, int n_heads, int32_t* blk_idx,
                int32_t* blk_cnt, void* ws, size_t ws_bytes, void* stream);

/*
 * Vertical-Slash sparse attention (guide, "Vertical-Slash Kernel
 * Mechanics": online softmax over the gathered columns and the diagonals).
 * Row i attends key j <= i iff j is one of the head's vertical columns, or
 * the 64x64 tile holding (i, j) is touched by one of its slash diagonals
 * (diagonal o touches the tiles with block-diagonal delta = bq - bk,
 * |o - 64 delta| <= 63; such tiles are computed whole, causally masked).
 * A key is never counted twice.  v_idx [n_heads][vertical_size] and
 * s_idx [n_heads][slash_size] (device int32) may be unsorted and may repeat
 * entries; entries outside [0, N) are skipped (counted in err_count).
 * out [Hq][N][d] bf16; lse [Hq][N] fp32 natural-log sum of exp (optional).
 * A row with no allowed key gets out = 0 and lse = -inf.
 */
int mi_vs_sparse_attn(const mi_bf16* q, const mi_bf16* k, const mi_bf16* v, int Hq, int Hkv,
                      int N, int d, float scale, const int32_t* v_idx, int vertical_size,
                      const int32_t* s_idx, int slash_size, const int32_t* heads, int n_heads,
                      mi_bf16* out, float* lse, int32_t* err_count, void* ws, size_t ws_bytes,
                      void* stream);

/*
 * Vertical-Slash sparse attention with range slash tiles (MI_SLASH_RANGES):
 * the guide's cost model for this pattern ("2. The Vertical-Slash Pattern":
 * work in proportion to the kept columns and diagonals) with the diagonals
 * streamed as contiguous key runs ("Vertical-Slash Kernel Mechanics").
 * Row i of query block bq = i / 64 attends key j <= i iff j is one of the
 * head's vertical columns, or some selected diagonal o has
 * 64 bq - o <= j <= 64 bq + 63 - o.  The kept keys of a block are a union
 * of such 64-key runs; the kernel covers it with 64-key tiles that start at
 * any key, so an isolated diagonal costs one tile per query block instead of
 * the two 64x64 tiles it touches.  Arguments, layouts, workspace
 * (mi_workspace_bytes with MI_OP_VS_ATTN) and errors as for
 * mi_vs_sparse_attn.
 */
int mi_vs_range_attn(const mi_bf16* q, const mi_bf16* k, const mi_bf16* v, int Hq, int Hkv,
                     int N, int d, float scale, const int32_t* v_idx, int vertical_size,
                     const int32_t* s_idx, int slash_size, const int32_t* heads, int n_heads,
                     mi_bf16* out, float* lse, int32_t* err_count, void* ws, size_t ws_bytes,
                     void* stream);

/*
 * Block-sparse attention (guide, "3. The Block-Sparse Pattern": only the
 * selected 64x64 tiles are computed).  Row i of query block bq = i / 64
 * attends key j <= i iff j / 64 is among the first blk_cnt[bq] entries of
 * blk_idx[bq] (device int32, layouts as produced by mi_bs_index; entries may
 * be unsorted or repeated; entries outside [0, bq] are skipped and counted).
 * `block` must be 64.  out / lse as for mi_vs_sparse_attn.
 */
int mi_block_sparse_attn(const mi_bf16* q, const mi_bf16* k, const mi_bf16* v, int Hq, int Hkv,
                         int N, int d, float scale, const int32_t* blk_idx,
                         const int32_t* blk_cnt, int topk, int block, const int32_t* heads,
                         int n_heads, mi_bf16* out, float* lse, int32_t* err_count, void* ws,
                         size_t ws_bytes, void* stream);

/*
 * A-shape attention (guide, "1. The A-Shape Pattern": attention sinks plus a
 * local causal band).  Row i attends key j <= i iff j < sink or
 * i - j < window (the window counts the query itself).  sink >= 0,
 * window >= 1.  out / lse as for mi_vs_sparse_attn.
 */
int mi_ashape_attn(const mi_bf16* q, const mi_bf16* k, const mi_bf16* v, int Hq, int Hkv, int N,
                   int d, float scale, int sink, int window, const int32_t* heads, int n_heads,
                   mi_bf16* out, float* lse, int32_t* err_count, void* ws, size_t ws_bytes,
                   void* stream);

/*
 * Dense causal attention: row i attends every key j <= i, on the same engine
 * as the sparse entry points (every causal 64x64 tile computed).  No
 * workspace is needed (ws may be NULL).  out / lse as for mi_vs_sparse_attn.
 */
int mi_dense_attn(const mi_bf16* q, const mi_bf16* k, const mi_bf16* v, int Hq, int Hkv, int N,
                  int d, float scale, const int32_t* heads, int n_heads, mi_bf16* out,
                  float* lse, int32_t* err_count, void* ws, size_t ws_bytes, void* stream);

/*
 * One attention layer with a per-head pattern table (guide, "Phase 2: The
 * Online Dynamic Kernel Router"): `pattern` is a HOST int8 [Hq] of
 * MI_PATTERN_* codes.  Builds the VS and BS indices for the heads that need
 * them, then runs one sparse-attention launch over all heads, each with its
 * own pattern; all on `stream`, no host-device synchronisation.
 * stage_events (optional): MI_STAGE_EVENTS cudaEvent_t handles (as void*),
 * recorded on `stream` at the stage boundaries.
 */
int mi_prefill_layer(const mi_bf16* q, const mi_bf16* k, const mi_bf16* v, int Hq, int Hkv,
                     int N, int d, float scale, const int8_t* pattern, const mi_params* p,
                     mi_bf16* out, float* lse, int32_t* err_count, void* ws, size_t ws_bytes,
                     void* stream, void* const* stage_events);

/*
 * mi_prefill_layer with one mi_params per head: `params` is a HOST array of
 * Hq entries, read for each head according to its pattern (the pages' offline
 * pattern profiler sets them per head; guide, "Phase 1: The Offline Pattern
 * Profiler").  Vertical-Slash
 * heads may differ in vertical_size and slash_size but must share last_q;
 * Block-Sparse heads may differ in topk_blocks; A-shape heads in sink and
 * window.  MI_ERR_INVALID_ARG for VS heads with different last_q.  The
 * workspace is mi_prefill_workspace_bytes_heads() of the same arguments
 * (0 if they are invalid).  Everything else as for mi_prefill_layer.
 */
size_t mi_prefill_workspace_bytes_heads(int Hq, int Hkv, int N, int d, const int8_t* pattern,
                                        const mi_params* params);
int mi_prefill_layer_heads(const mi_bf16* q, const mi_bf16* k, const mi_bf16* v, int Hq,
                           int Hkv, int N, int d, float scale, const int8_t* pattern,
                           const mi_params* params, mi_bf16* out, float* lse,
                           int32_t* err_count, void* ws, size_t ws_bytes, void* stream,
                           void* const* stage_events);

/*
 * mi_vs_index without a workspace argument.  The paper has no counterpart:
 * this entry point exists for callers that cannot provide device scratch --
 * e.g. an inference server that reserves nearly all HBM for its KV-cache pool
 * and forbids new allocations on the request path, or host code on a
 * latency-critical path where cudaMalloc's implicit synchronisation is not
 * acceptable.  It computes exactly what mi_vs_index computes (same kernels,
 * same results), with its scratch in a 16 MiB array inside the library that
 * every GPU which loads the library holds until the process exits.  It
 * allocates nothing.
 *  - Capacity: the call needs the bytes mi_workspace_bytes(MI_OP_VS_INDEX,
 *    ...) reports for the same arguments; beyond 16 MiB it returns
 *    MI_ERR_UNSUPPORTED and launches nothing (for example 8 heads at
 *    N = 131072 fit, 32 heads at N = 131072 do not).
 *  - Every call shares that one array.  Calls whose work overlaps on the GPU
 *    (other streams, other host threads, concurrent graph replays) race on
 *    it; serialise them, e.g. on one stream.
 *  - The first call on each device looks up the array's device address and
 *    caches it; make that first call before any stream capture on the device.
 *    A device reset (cudaDeviceReset) invalidates the cached address: do not
 *    call this entry point again in a process that reset the device.
 * All other arguments, outputs and errors as for mi_vs_index.
 */
int mi_vs_index_static(const mi_bf16* q, const mi_bf16* k, int Hq, int Hkv, int N, int d,
                       float scale, int last_q, int vertical_size, int slash_size,
                       const int32_t* heads, int n_heads, int32_t* v_idx, int32_t* s_idx,
                       float* v_score, float* s_score, void* stream);

/*
 * Diagnostics (not on the hot path; synchronous).  The sparse-attention
 * kernel and the tensor-core Vertical-Slash score passes bound every wait;
 * the first wait that gives up is recorded as
 * {launch sequence, site, block, thread, group or tile, parity, 0 or block y,
 * 0} with site in 1..7 for attention (1 producer/stage-free, 2 MMA/Q,
 * 3 MMA/stage-full, 4 MMA/P-ready, 5 softmax/stage-full, 6 softmax/S-ready,
 * 7 softmax/O-done) and 11..15 for the score passes (11 producer/stage-free,
 * 12 MMA/Q, 13 MMA/stage-full, 14 MMA/accumulator-free, 15 epilogue/
 * accumulator-full), and 21..27 for the key-major Block-Sparse engine
 * (21 producer, 22-24 MMA issue, 25-27 softmax); site 0 means no wait
 * gave up.  The row-major attention record is returned when it holds one,
 * else the key-major one, else the score passes'.  Reading copies the record
 * to `record8` (host int32 [8]) and clears all three.  A correct run never
 * records anything.
 */
int mi_debug_wait_failure(int32_t* record8);

/*
 * Diagnostics: the clock budget (in SM cycles) of every abortable wait inside
 * the kernels launched after this call; cycles <= 0 restores the default of
 * about half a second.  Waits that guard the release of tensor memory or the
 * landing of copies in flight keep the full budget whatever is set here, so
 * a launch whose waits give up still ends cleanly: it sets bit 30 of its
 * err_count, records the site for mi_debug_wait_failure, writes zero rows,
 * and leaves the device usable.  For tests of that failure path only; a
 * small budget makes correct launches give up.  Process-wide, not thread-safe
 * against concurrent launches.
 */
int mi_debug_set_wait_budget(long long cycles);

/*
 * Engine for Block-Sparse heads in the launches that follow (process-wide):
 *   MI_BS_ENGINE_ROW (0, the default) -- the row-major engine every pattern
 *     uses: 128 query rows per tensor-core tile (two 64-row query blocks),
 *     each 64-key chunk the union of the two blocks' chosen blocks;
 *   MI_BS_ENGINE_KEY (1) -- the key-major engine for d = 128: one 64-row
 *     query block per work item, two of ITS chosen key blocks per 128-key
 *     tile (S^T = K Q^T, O^T += V^T P^T), so no computed score is unused.
 * Both follow the Block-Sparse definition of MInference 1.0 (aifetchly
 * guide, "3. The Block-Sparse Pattern") and give the same results up to
 * rounding order.  The row-major engine is the faster one on the Block-Sparse
 * workloads measured so far; the key-major one is kept for comparison.
 * Returns MI_ERR_INVALID_ARG for any other value.  Not thread-safe against
 * concurrent launches.
 */
#define MI_BS_ENGINE_ROW 0
#define MI_BS_ENGINE_KEY 1
int mi_set_bs_engine(int engine);

#ifdef __cplusplus
}
#endif

#endif /* MINFER_H */
