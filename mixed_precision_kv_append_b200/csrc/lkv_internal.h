// lkv_internal.h -- structures and launchers shared by the CUDA sources of libloopkv.
// Not part of the ABI.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "loopkv.h"
#include "loopkv_format.h"

namespace lkv {

// Device-side state of a cache, carved from the caller's buffer.
struct DevState {
    uint32_t *status;     // [1] LOOPKV_DEV_* bits
    int32_t *ctrl;        // [8] per-call control words (ingest admission flag)
    int32_t *hist_len;    // [n_cells][max_batch]
    int32_t *tail_len;    // [n_cells][max_batch] near tokens (sink fill + window length)
    int32_t *win_start;   // [n_cells][max_batch] window ring slot of the oldest window token
    int32_t *block_table; // [n_cells][max_batch][max_blocks]
    int32_t *free4;       // free stack of the 4-bit pool, ids [0, n4)
    int32_t *top4;        // number of free ids in free4
    int32_t *free2;
    int32_t *top2;
    int64_t n4, n2;       // pool capacities in blocks
    uint8_t *tail;        // [n_cells][max_batch][2][H][near_cap][D] elements of in_dtype
    int sink, wring;      // sink slots, window ring slots (window_tokens + 32)
    int near_cap;         // sink + wring
    uint8_t *main4;       // [n4][H][LKV_HEAD_MAIN_4B(D)]
    uint8_t *lo4;         // [n4][H][LKV_HEAD_LO_4B(D)]
    uint8_t *main2;       // [n2][H][LKV_HEAD_MAIN_2B(D)]
};

// Arguments of one fused decode launch (one cell).
struct DecodeArgs {
    const void *q;              // [B][H][D] in_dtype
    float *out;                 // [B][H][D]
    const uint8_t *main;        // pool of the source cell's storage mode
    const uint8_t *lo;          // lo pool (4-bit sources)
    const int32_t *block_table; // source cell [max_batch][max_blocks]
    const int32_t *hist_len;    // source cell [max_batch]
    const int32_t *tail_len;    // own cell [max_batch] near tokens
    const int32_t *win_start;   // own cell [max_batch] ring slot of the oldest window token
    const uint8_t *tail;        // own cell [max_batch][2][H][near_cap][D]
    uint32_t *status;
    uint32_t *s_bitmap;         // optional [B][H][bitmap_words]
    float *row_max;             // optional [B][H]
    float *row_sum;             // optional [B][H]
    int64_t pool_blocks;
    int H;
    int rows;                   // B * H (request, head) rows
    int max_blocks;
    int bitmap_words;
    int cap_groups;             // score capacity per CTA, in 32-token groups
    float qscale;               // log2(e) / sqrt(D)
    float tau;
    int tau_mode;
    int sink, wring, near_cap;  // near region geometry (see DevState)
    int attn_window;            // sliding attention window of the cell's layer in tokens, 0 = full
    unsigned long long wait_ns; // limit of every bounded wait, in nanoseconds
    int inject;                 // LOOPKV_INJECT_*: LOOPKV_INJECT_NONE in normal operation
};

struct DecodeShape {
    int cluster;   // CTAs per cluster; a cluster reads one (request, head) row at a time
    int clusters;  // persistent clusters in the grid
    int stages;    // ring slots per warp (a power of two)
    int stages_log2;
    int score_bufs; // 1, or 2 when a cluster reads several rows
    int min_ctas;   // register budget of the kernel build: CTAs per SM (4 or 5)
    int smem;      // dynamic shared memory bytes per CTA
    int threads;
    int cap;       // score capacity per CTA and row, in 32-token groups
    int pdl;       // launch with programmatic stream serialization (overlap the previous launch)
    int onepass;   // single-pass kernel (refine set independent of the row maximum)
};

// Launchers (defined in the .cu files).  Return LOOPKV_OK or an error code.
// pdl: launch with programmatic stream serialization (see launch_shape in decode_kernel.cu); the
// caller passes false when the previous launch on the stream may have written lengths, block
// tables or pools, which the kernel reads before its grid dependency wait.
int launch_decode(const DecodeArgs &a, int bits, int D, int dtype, const DecodeShape &shp, bool pdl,
                  cudaStream_t s);
// onepass: the rows' refine set does not depend on the row maximum (2-bit source, or a
// 4-bit source read with tau <= 0), so the single-pass kernel may read them.
DecodeShape decode_shape(int bits, int D, int dtype, int rows, int max_blocks, int near_cap, bool onepass);

int launch_init_state(const DevState &st, cudaStream_t s);
int launch_append(const DevState &st, int cell, int H, int D, int dtype, int max_batch, const void *k,
                  const void *v, const int32_t *req_ids_dev, int B, cudaStream_t s);
int launch_flush(const DevState &st, const uint8_t *cell_modes_dev, int n_cells, int H, int D, int dtype,
                 int max_batch, int max_blocks, cudaStream_t s);
int launch_ingest(const DevState &st, int cell, int mode, int H, int D, int dtype, int max_batch,
                  int max_blocks, int req, const void *k, const void *v, int T, cudaStream_t s);
int launch_reset(const DevState &st, const uint8_t *cell_modes_dev, int n_cells, int max_batch, int max_blocks,
                 int req, cudaStream_t s);

// What an entry point defined outside runtime.cu needs to know about a cache.
struct CacheInfo {
    DevState st;
    int n_loops, n_layers, n_heads, head_dim, in_dtype, max_batch;
};
int cache_info(const loopkv_cache *cache, CacheInfo *out);

}  // namespace lkv
