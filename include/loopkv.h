/*
 * loopkv.h -- C ABI of the LoopKV decode hot path on B200 (sm_100a).
 *
 * LoopKV (arXiv 2611.04137) compresses the KV cache of a looped transformer per
 * (loop, layer) "cell": each cell stores its history as 4-bit codes, as 2-bit codes,
 * or reads the final loop's history of the same layer (LoopKV paper, §3 "System
 * Design", §3.1 C1, §3.2 C2).  At decode time every loop reads all key codes,
 * computes exact softmax weights, and fetches the low 2-bit plane of a value only
 * for tokens whose weight is at least tau times the row maximum (§3.3 C3).
 *
 * This header is the whole boundary: plain pointers and sizes, no framework types.
 *
 * Conventions
 *   - Every function returns LOOPKV_OK (0) or a negative LOOPKV_ERR_* code; no
 *     exception crosses the ABI.  loopkv_strerror() names a code.
 *   - "device pointer" = memory on the current CUDA device; "host pointer" = CPU
 *     memory.  `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Kernels run asynchronously on that stream; argument checks that
 *     need no device data happen before launch and return an error without
 *     launching.  Errors found on the device (non-finite inputs, a full tail, an
 *     exhausted pool, an out-of-range block id, a timed-out wait) are OR-ed into a
 *     device status word that loopkv_status() reads and clears.
 *   - Ownership: the caller owns every q/k/v/out buffer and the device buffer given
 *     to loopkv_alloc (it must outlive the cache).  The library owns plan and cache
 *     handles and the descriptors it keeps on the host.
 *   - All device addresses the kernels use are fixed for the life of a cache, so a
 *     sequence of append / flush / decode calls can be captured in a CUDA graph and
 *     replayed (the paper replays a whole decode step as one graph, §3.4).
 *   - Shapes: H = n_heads, D = head_dim (64 or 128), tokens of a cell are paged in
 *     16-token blocks; a K quantization group is 32 tokens = two blocks.
 */
#ifndef LOOPKV_H
#define LOOPKV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- status codes ------------------------------------------------------- */
#define LOOPKV_OK 0
#define LOOPKV_ERR_INVALID_ARG (-1)    /* null pointer, index out of range, bad value */
#define LOOPKV_ERR_SHAPE (-2)          /* sizes inconsistent with the config */
#define LOOPKV_ERR_PLAN (-3)           /* share cell in the final loop, bad mode */
#define LOOPKV_ERR_POOL_EXHAUSTED (-4) /* no free 16-token block left */
#define LOOPKV_ERR_NONFINITE (-5)      /* NaN or Inf in a quantized group */
#define LOOPKV_ERR_RANGE (-6)          /* fp16 zero point or scale overflows */
#define LOOPKV_ERR_TIMEOUT (-7)        /* a bounded device wait gave up */
#define LOOPKV_ERR_CUDA (-8)           /* a CUDA runtime call failed */
#define LOOPKV_ERR_TAIL_FULL (-9)      /* append to a full window (W + 32 tokens) not yet flushed */
#define LOOPKV_ERR_STATE (-10)         /* ingest into a non-empty (cell, request), bad block id */
#define LOOPKV_ERR_EMPTY_ROW (-11)     /* decode of a row with no token at all */
#define LOOPKV_ERR_NO_DEVICE (-12)     /* no CUDA device of compute capability 10.x */
#define LOOPKV_ERR_INFEASIBLE (-13)    /* plan search: no plan meets the budgets */

/* Device status word bits (loopkv_status); each maps to one code above. */
#define LOOPKV_DEV_NONFINITE 0x01u
#define LOOPKV_DEV_RANGE 0x02u
#define LOOPKV_DEV_POOL_EXHAUSTED 0x04u
#define LOOPKV_DEV_TAIL_FULL 0x08u
#define LOOPKV_DEV_STATE 0x10u
#define LOOPKV_DEV_TIMEOUT 0x20u
#define LOOPKV_DEV_EMPTY_ROW 0x40u

/* ---- enums -------------------------------------------------------------- */
/* Storage option of a cell (LoopKV paper, §3 and §3.4 "Layout"). */
typedef enum {
    LOOPKV_CELL_4B = 0,   /* own 4-bit KIVI-style codes; V split into hi/lo 2-bit planes */
    LOOPKV_CELL_2B = 1,   /* own 2-bit KIVI-style codes */
    LOOPKV_CELL_SHARE = 2 /* reads the final loop's history at the same layer (§3.2) */
} loopkv_cell_mode;

/* Which weight the threshold tau is compared with (LoopKV paper, §3.3). */
typedef enum {
    LOOPKV_TAU_REL_MAX = 0,  /* hot iff exp(s_t - m) >= tau, m = exact row max (default) */
    LOOPKV_TAU_ABS_PROB = 1, /* hot iff exp(s_t - m) / sum_u exp(s_u - m) >= tau */
    /* The paper's streaming rule (§3.3: the reader tests tokens against a running maximum
     * that starts at a seed, the sink maximum).  Each reading warp takes its 32-token groups
     * in order; the running maximum starts at the row's largest sink score (minus infinity
     * without a sink) and takes each group's largest score before that group's tokens are
     * tested: hot iff exp(s_t - m_run) >= tau.  A superset of the REL_MAX set; which tokens
     * it adds depends on the split of the row over the reading warps (group g of the row is
     * read by CTA g mod C of the cluster, as its local group g / C, and local group i by warp
     * i mod 4 in increasing i; C from loopkv_decode_shape).  The seed travels with the row
     * statistics the cluster exchanges anyway, so no reader waits for it. */
    LOOPKV_TAU_STREAM = 2
} loopkv_tau_mode;

/* Element type of q, k, v inputs and of the unquantized tail. */
typedef enum { LOOPKV_DTYPE_BF16 = 0, LOOPKV_DTYPE_F32 = 1 } loopkv_dtype;

/* ---- configuration and handles ------------------------------------------ */
typedef struct {
    int n_layers;           /* layers of the looped block */
    int n_loops;            /* loops per token; the last one is the "final loop" */
    int n_heads;            /* KV heads H (multi-head attention, no GQA) */
    int head_dim;           /* D: 64 or 128 */
    int max_batch;          /* request slots per cell */
    int max_blocks_per_seq; /* capacity of a cell's history in 16-token blocks (even) */
    int in_dtype;           /* loopkv_dtype */
    /* Unquantized near region of every (cell, request) (LoopKV paper §2.3 and §3.4: the
     * attention sink and the recent window stay BF16, and a 32-token page is quantized when
     * it leaves the window).  sink_tokens: the first tokens of a sequence, never quantized
     * (0..64, a multiple of 32; the paper uses 32).  window_tokens: W, multiple of 32, 0..512
     * (the paper uses 256).  The window holds the most recent W to W + 31 tokens after a
     * flush; loopkv_flush quantizes its oldest page once it holds W + 32.  The history (the
     * quantized pages) lies between sink and window in sequence order.  Both 0 (the zero
     * default of older callers): no sink, and a tail of up to 32 tokens quantized as soon as
     * it is full. */
    int sink_tokens;
    int window_tokens;
} loopkv_config;

typedef struct loopkv_plan loopkv_plan;   /* opaque: config + per-cell modes + tau */
typedef struct loopkv_cache loopkv_cache; /* opaque: pools, tails, block tables */

/* Bytes of KV history per token summed over all cells (LoopKV paper §2.2, §3.3).
 * A 4-bit cell stores 2.5 KiB per token at H = 16, D = 128 (K codes, K meta, V hi,
 * V lo, V meta) and reads 2.0 KiB + 0.5 KiB for a hot token; a 2-bit cell stores and
 * reads 1.5 KiB; a share cell stores nothing and reads its source's pages. */
typedef struct {
    double stored_bytes_per_token;
    double read_bytes_per_token; /* at the given hot fractions */
    double read_bytes_all_hot;   /* every lo plane read (tau = 0) */
    double read_bytes_all_cold;  /* no lo plane read */
    double bf16_bytes_per_token; /* the same cells kept as BF16 K and V */
} loopkv_byte_report;

/* Device addresses of one cell, for inspection (tests, tools). */
typedef struct {
    int mode;                /* loopkv_cell_mode of this cell */
    int src_cell;            /* cell whose history pages are read (self or final loop) */
    int src_mode;            /* storage mode of src_cell (4B or 2B) */
    int head_main_bytes;     /* bytes of one head's main region in a block of src_cell */
    int head_lo_bytes;       /* bytes of one head's lo-plane region (4B) or 0 */
    const uint8_t *main_pool;   /* device: block b, head h at b*H*head_main_bytes + h*head_main_bytes */
    const uint8_t *lo_pool;     /* device: block b, head h at (b*H + h)*head_lo_bytes */
    const int32_t *block_table; /* device [max_batch][max_blocks_per_seq] of src_cell */
    const int32_t *hist_len;    /* device [max_batch] history tokens of src_cell */
    const int32_t *tail_len;    /* device [max_batch] unquantized (near) tokens of this cell:
                                 * sink fill + window length */
    const int32_t *win_start;   /* device [max_batch] ring slot of the oldest window token */
    const void *tail;           /* device [max_batch][2 (K,V)][H][near_cap][D] in in_dtype: near
                                 * token slots; slots 0..sink-1 the sink, then the window ring of
                                 * window_tokens + 32 slots (see loopkv_config) */
    int near_cap;               /* sink_tokens + window_tokens + 32 */
    int64_t pool_blocks;        /* capacity of the pool in blocks */
} loopkv_cell_view;

/* ---- plan ---------------------------------------------------------------- */
/*
 * Build a plan: one storage option per cell, as the paper's offline planner produces it
 * (LoopKV paper §3; loopkv_plan_search below is one such planner).  modes[n_loops *
 * n_layers] is loop-major: cell (loop, layer) at loop * n_layers + layer.  Cells of the
 * final loop must be 4B or 2B; a share cell
 * reads cell (n_loops - 1, layer).  tau >= 0; tau = 0 reads every lo plane, tau > 1
 * none.  Returns LOOPKV_ERR_PLAN / LOOPKV_ERR_INVALID_ARG / LOOPKV_ERR_SHAPE.
 */
int loopkv_plan_create(const loopkv_config *cfg, const uint8_t *modes, float tau, int tau_mode,
                       loopkv_plan **out);
void loopkv_plan_free(loopkv_plan *plan);

/*
 * Sliding-window attention for one layer (the Dory model's recurrent block mixes
 * full-attention and sliding-window layers, LoopKV paper §2.1): every cell of `layer`
 * attends only to the last window_tokens positions of its sequence (sink, history pages
 * and window in sequence order); 0 restores full attention (the default).  The refine set,
 * row maximum and output then run over those tokens only, and a decode reads only the
 * history pages that reach into the window.  Storage is unchanged (older pages are kept).
 * Applies to decodes made with this plan after the call.  Such decodes are launched
 * without programmatic dependent launch.  Returns LOOPKV_ERR_INVALID_ARG for a bad layer or a
 * negative window.
 */
int loopkv_plan_set_window(loopkv_plan *plan, int layer, int window_tokens);

/*
 * Byte accounting of a plan (LoopKV paper §2.2 and §3.3: KiB stored and read per
 * token).  hot_fraction: host [n_loops * n_layers] fraction of history tokens read
 * with their lo plane per reading cell, or NULL for 1.0 (every lo plane read).
 * Host-only; touches no device.
 */
int loopkv_plan_bytes(const loopkv_plan *plan, const float *hot_fraction, loopkv_byte_report *out);

/*
 * Offline plan search (LoopKV paper §3.1 "Allocation"): choose one storage option per
 * cell of loops 0 .. n_loops-2 -- LOOPKV_CELL_4B, LOOPKV_CELL_2B, or LOOPKV_CELL_SHARE
 * (reads the final loop's cell of the same layer, §3.2) -- that minimizes the bytes read
 * per token subject to
 *     sum over all cells of damage[cell][option] <= damage_budget, and
 *     stored bytes per token <= storage_budget (no storage budget if <= 0).
 * Cells of the final loop keep 4-bit codes.  Bytes per token and head: 4-bit stores and
 * reads 1.25 D (every lo plane counted), 2-bit 0.75 D, share stores 0 and reads 1.25 D.
 * Damages add up over cells (the paper's profile: summed single-cell damages predict a
 * plan's KL).  Among the plans with the fewest reads the result has the least damage, then
 * the least storage; remaining ties are broken deterministically.  Exact (dynamic program
 * over cells).  Host-only; touches no device.
 *   damage:    host [n_loops * n_layers][3] (loop-major cells, option index =
 *              loopkv_cell_mode), finite and >= 0; of final-loop cells only the 4B entry
 *              is read.
 *   modes_out: host [n_loops * n_layers], the plan's modes for loopkv_plan_create.
 *   report:    may be NULL; read / stored bytes per token and total damage of the plan.
 * Returns LOOPKV_OK, LOOPKV_ERR_INVALID_ARG, or LOOPKV_ERR_INFEASIBLE (modes_out then
 * untouched).
 */
typedef struct {
    double read_bytes_per_token;   /* every lo plane read */
    double stored_bytes_per_token;
    double damage;                 /* sum over all cells, final loop included */
} loopkv_plan_search_report;

int loopkv_plan_search(const loopkv_config *cfg, const double *damage, double damage_budget,
                       double storage_budget, uint8_t *modes_out, loopkv_plan_search_report *report);

/* Device bytes a cache needs so that every non-share cell can hold max_batch x
 * max_blocks_per_seq blocks.  Host-only. */
int loopkv_required_bytes(const loopkv_plan *plan, size_t *bytes);

/* ---- cache --------------------------------------------------------------- */
/*
 * Carve a cache out of a caller-owned device buffer (the paper carves its history
 * pools out of the engine's KV budget, §4 "vLLM integration").  dev_buf must be
 * 256-byte aligned.  If dev_bytes is below loopkv_required_bytes the 4-bit and
 * 2-bit block pools are shrunk in proportion and blocks are handed out on demand
 * (paged); running out later raises LOOPKV_DEV_POOL_EXHAUSTED.  Initialises the
 * device state on `stream` (lengths zero, free lists full).  The cache keeps a copy
 * of the plan.
 */
int loopkv_alloc(const loopkv_plan *plan, void *dev_buf, size_t dev_bytes, void *stream,
                 loopkv_cache **out);
void loopkv_free(loopkv_cache *cache);

/*
 * Bulk history of one request in one cell (prefill).  k, v: device [T][H][D] in
 * in_dtype.  The (cell, request) must be empty (else LOOPKV_DEV_STATE and nothing is
 * written).  The first min(T, sink) tokens fill the sink; of the remaining R, the first
 * 32 * floor((R - W) / 32) (none if R < W) are quantized into 16-token blocks by the same
 * kernel as loopkv_flush, and the last go to the window (W to W + 31 of them, or all R
 * when R < W); with sink = W = 0 that is T mod 32 tokens.  A share cell stores only its
 * sink and window; its history is the final loop's (LoopKV paper §3.2), which must be
 * ingested with the same T before decoding.
 */
int loopkv_ingest(loopkv_cache *cache, int loop, int layer, int req, const void *k, const void *v,
                  int T, void *stream);

/*
 * Append one token per request to a cell's unquantized near region (LoopKV paper §3.4:
 * sink and window stay BF16; share cells keep their own, §3.2): into the sink while it is
 * not full, else into the window.  k, v: device [B][H][D] in in_dtype for requests
 * req_ids[0..B-1] (host array) or 0..B-1 when req_ids is NULL.  A window already holding
 * W + 32 tokens raises LOOPKV_DEV_TAIL_FULL for that request and drops its token: call
 * loopkv_flush first.
 */
int loopkv_append(loopkv_cache *cache, int loop, int layer, const void *k, const void *v,
                  const int32_t *req_ids, int B, void *stream);

/*
 * loopkv_append for callers that cannot allocate device memory: engines that hand all
 * device memory to their own arena up front (so no further allocation can succeed), or
 * code on a decode loop that cannot take the device-wide synchronisation an allocation may
 * cause.  The LoopKV paper has no counterpart; this is an interface convenience.
 *
 * Same arguments, results and device-side errors as loopkv_append.  The request ids go to
 * the device through a fixed array inside the library (LOOPKV_NOALLOC_MAX_IDS int32, 16 KiB,
 * which every GPU that loads the library keeps until the process exits) instead of the
 * cache's staging words, and the call allocates nothing: no cudaMalloc, no cudaFree, no
 * allocating library routine.
 *   - B > LOOPKV_NOALLOC_MAX_IDS (or > max_batch) returns LOOPKV_ERR_SHAPE before any
 *     device work.
 *   - The first call on a device looks up the array's device address with the device
 *     current (cudaGetSymbolAddress) and keeps it; make that first call before any stream
 *     capture.  A failed look-up returns LOOPKV_ERR_CUDA.
 *   - Every call shares the one array and leaves its ids there; each call writes all B ids
 *     it reads, so nothing has to start at zero.  Calls whose copies and kernels overlap on
 *     the GPU (different streams, no ordering between them) race on the array: order them.
 */
#define LOOPKV_NOALLOC_MAX_IDS 4096
int loopkv_append_noalloc(loopkv_cache *cache, int loop, int layer, const void *k, const void *v,
                          const int32_t *req_ids, int B, void *stream);

/*
 * Window exit: in every (cell, request) whose window holds W + 32 tokens, quantize its
 * oldest 32 into two new 16-token blocks of the cell (K per channel over the 32 tokens, V
 * per token over 32 channels, fp16 scale/zero, V split into hi/lo planes) and drop them
 * from the window; a share cell only drops them (LoopKV paper §3.2; §3.4 "Layout", where
 * pages are quantized as they leave the window, ahead of the step's graph).  Blocks come
 * from the device free list, so the call needs no host round trip and can sit inside a
 * captured graph.
 */
int loopkv_flush(loopkv_cache *cache, void *stream);

/* Release every block of request slot `req` in every cell and zero its lengths. */
int loopkv_reset_request(loopkv_cache *cache, int req, void *stream);

/*
 * Fused decode attention for cell (loop, layer), one launch (LoopKV paper §3.4 "One
 * launch per cell").  q: device [B][H][D] in in_dtype for request slots 0..B-1;
 * out: device [B][H][D] fp32.  Per (request, head) row: scores over the full keys of
 * the history the cell reads (own pages, or the final loop's for a share cell) and
 * over its own sink and window; exact row max m; refine set S = history tokens of a 4-bit
 * source whose weight passes tau; values decoded as z + s*(4h+l) for tokens in S,
 * z + s*(4h+1.5) for the other 4-bit tokens, z + s*code for 2-bit cells, raw for the
 * sink and window; out = sum_t exp(s_t - m) v_t / sum_t exp(s_t - m).  When S does not depend on
 * m (2-bit source, or tau <= 0) the launch accumulates with a running maximum instead;
 * the result is the same up to fp32 rounding.  A decode uses no device scratch, so
 * decodes of different cells may run on different streams.  The first call for a batch
 * size queries the device occupancy to pick the launch shape (cached in the cache
 * object); make it before capturing a stream.  Calls on one cache may come from several
 * host threads (the host bookkeeping is locked).
 * A decode may start while the previous kernel on its stream is finishing (programmatic
 * dependent launch); it reads q and the tails, and writes out, only after that kernel has
 * completed.  It reads lengths, block tables and pools earlier, so a decode that directly
 * follows a loopkv_flush, loopkv_ingest or loopkv_reset_request on the same stream is
 * launched without the overlap.
 */
int loopkv_decode(const loopkv_plan *plan, int loop, int layer, const void *q,
                  const loopkv_cache *cache, float *out, int B, void *stream);

/*
 * loopkv_decode that also exports, per row, the refine set and the softmax
 * statistics.  s_bitmap: device uint32 [B][H][max_blocks_per_seq / 2]; bit t % 32 of
 * word t / 32 is set iff history token t is in S (words past the history are left
 * untouched).  row_max: device fp32 [B][H], m in natural-log units; row_sum: device
 * fp32 [B][H], sum_t exp(s_t - m).  Any of the three may be NULL.
 */
int loopkv_decode_debug(const loopkv_plan *plan, int loop, int layer, const void *q,
                        const loopkv_cache *cache, float *out, int B, void *stream,
                        uint32_t *s_bitmap, float *row_max, float *row_sum);

/* Synchronise `stream`, return the device status word in *device_status (a bit set
 * of LOOPKV_DEV_*) and clear it.  Returns the first matching LOOPKV_ERR_* code, or
 * LOOPKV_OK when the word is zero. */
int loopkv_status(loopkv_cache *cache, void *stream, int *device_status);

/*
 * Bounded device waits and a fault-injection hook for testing them.  Every wait of a decode
 * kernel on data it has requested (a pipeline stage's bytes) gives up after wait_limit_ns
 * (default 500 ms): the kernel then records LOOPKV_DEV_TIMEOUT, issues no further copies,
 * waits (again bounded) for the copies it already issued, and returns, so the stream and
 * the context stay usable; loopkv_status reports LOOPKV_ERR_TIMEOUT.  The outputs of a
 * decode that timed out are meaningless.
 * inject: LOOPKV_INJECT_NONE, or LOOPKV_INJECT_STALLED_STAGE: in later decodes one warp of
 * the first CTA arms its first stage for bytes that it never requests, so that wait runs
 * out (the LoopKV paper's reader gives up on a late publisher, §3.4; this makes the give-up
 * path testable without any fault).  Applies to decodes launched after the call.
 * Returns LOOPKV_ERR_INVALID_ARG for a zero limit or an unknown inject value.
 */
#define LOOPKV_INJECT_NONE 0
#define LOOPKV_INJECT_STALLED_STAGE 1
int loopkv_set_wait_policy(loopkv_cache *cache, uint64_t wait_limit_ns, int inject);

/* Device addresses of cell (loop, layer). */
int loopkv_cell_view_get(const loopkv_cache *cache, int loop, int layer, loopkv_cell_view *out);

/* Decode launch shape chosen for a batch of B requests (cluster size, CTAs, shared
 * memory per CTA) when the source cell is 4-bit, for reporting: the single-pass reader
 * when the plan's tau <= 0 (every token refined), else the exact-maximum reader.
 * Queries the occupancy of the current device (LOOPKV_ERR_NO_DEVICE without one). */
int loopkv_decode_shape(const loopkv_plan *plan, int B, int *cluster_size, int *ctas, int *smem_bytes);

const char *loopkv_strerror(int code);

/* Library version, major * 10000 + minor * 100 + patch. */
int loopkv_version(void);

#ifdef __cplusplus
}
#endif
#endif /* LOOPKV_H */
