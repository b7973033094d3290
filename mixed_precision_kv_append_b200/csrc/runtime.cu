// runtime.cu -- host side of libloopkv: plans, byte accounting, cache carving and
// the C ABI entry points declared in loopkv.h.
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdlib>
#include <cstring>
#include <map>
#include <mutex>
#include <new>
#include <tuple>
#include <vector>

#include "lkv_device.cuh"
#include "lkv_internal.h"

struct loopkv_plan {
    loopkv_config cfg;
    std::vector<uint8_t> modes;
    std::vector<int> layer_window; // sliding attention window per layer in tokens, 0 = full
    float tau;
    int tau_mode;
    int n_cells() const { return cfg.n_loops * cfg.n_layers; }
    int cell(int loop, int layer) const { return loop * cfg.n_layers + layer; }
    // A share cell reads the final loop's cell at the same layer (LoopKV paper §3.2).
    int src_cell(int c) const
    {
        return modes[c] == LOOPKV_CELL_SHARE ? cell(cfg.n_loops - 1, c % cfg.n_layers) : c;
    }
};

// Unquantized slots per (cell, request): the sink, then a window ring of window + 32.
static int near_cap(const loopkv_config &c) { return c.sink_tokens + c.window_tokens + 32; }

struct loopkv_cache {
    loopkv_plan plan;
    // Host bookkeeping shared by calls from several host threads, under `mu`:
    //   shapes: decode launch shapes by (storage bits, batch, single-pass), computed once
    //           (occupancy queries must not run while a stream is being captured);
    //   state_written: per stream, whether the last call of this library on it launched a
    //           kernel that writes lengths, block tables or pools (flush, ingest, reset).  A
    //           decode reads those before its grid dependency wait, so a decode right after
    //           such a launch does not overlap it (no programmatic dependent launch).
    std::mutex mu;
    std::map<std::tuple<int, int, bool, int>, lkv::DecodeShape> shapes;
    std::map<void *, bool> state_written;
    unsigned long long wait_ns = lkv::kDefaultWaitNs;
    int inject = LOOPKV_INJECT_NONE;
    void mark_state_written(void *stream)
    {
        std::lock_guard<std::mutex> lock(mu);
        state_written[stream] = true;
    }
    // Whether a decode on `stream` may overlap the previous launch; clears the mark.
    bool decode_may_overlap(void *stream)
    {
        std::lock_guard<std::mutex> lock(mu);
        auto it = state_written.find(stream);
        const bool written = it != state_written.end() && it->second;
        if (written)
            it->second = false;
        return !written;
    }
    // window: the layer's sliding attention window (0: full attention).  A window bounds the
    // history groups a row reads to (window + sink) / 32 + 1 (the first may be partly before the
    // window), so those reads take the shape of that shorter row.
    lkv::DecodeShape shape(int bits, int B, bool onepass, int window)
    {
        int mb = plan.cfg.max_blocks_per_seq;
        if (window > 0)
            mb = std::min(mb, 2 * ((window + plan.cfg.sink_tokens + 31) / 32 + 1));
        std::lock_guard<std::mutex> lock(mu);
        auto key = std::make_tuple(bits, B, onepass, mb);
        auto it = shapes.find(key);
        if (it == shapes.end())
            it = shapes.emplace(key, lkv::decode_shape(bits, plan.cfg.head_dim, plan.cfg.in_dtype, B * plan.cfg.n_heads,
                                                       mb, near_cap(plan.cfg), onepass))
                     .first;
        return it->second;
    }
    lkv::DevState st;
    uint8_t *modes_dev;
    int32_t *req_stage; // [max_batch] request ids of the last loopkv_append with req_ids
    uint8_t *base;
    size_t bytes;
    int esz;
};

namespace {

constexpr size_t kAlign = 256;
size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

int dtype_size(int dt) { return dt == LOOPKV_DTYPE_BF16 ? 2 : 4; }

int head_main_bytes(int bits, int D) { return bits == 4 ? LKV_HEAD_MAIN_4B(D) : LKV_HEAD_MAIN_2B(D); }

// Whether a read's refine set is fixed before any score is known: a 2-bit source has no lo
// plane (S empty), a 4-bit source read with tau <= 0 refines every token.  Such reads go to
// the single-pass kernel (running maximum), the others to the exact-maximum kernel.
bool single_pass(int bits, float tau) { return bits == 2 || !(tau > 0.f); }

int check_config(const loopkv_config *c)
{
    if (!c)
        return LOOPKV_ERR_INVALID_ARG;
    if (c->n_layers <= 0 || c->n_loops <= 0 || c->n_heads <= 0 || c->max_batch <= 0 || c->max_blocks_per_seq <= 0)
        return LOOPKV_ERR_SHAPE;
    if (c->head_dim != 64 && c->head_dim != 128)
        return LOOPKV_ERR_SHAPE;
    if (c->max_blocks_per_seq % 2)
        return LOOPKV_ERR_SHAPE;
    if (c->in_dtype != LOOPKV_DTYPE_BF16 && c->in_dtype != LOOPKV_DTYPE_F32)
        return LOOPKV_ERR_INVALID_ARG;
    if ((int64_t)c->n_heads * c->max_batch > 65535)
        return LOOPKV_ERR_SHAPE;
    if (c->sink_tokens < 0 || c->sink_tokens > 64 || c->sink_tokens % 32 || c->window_tokens < 0 ||
        c->window_tokens > 512 || c->window_tokens % 32)
        return LOOPKV_ERR_SHAPE;
    return LOOPKV_OK;
}

struct Layout {
    size_t status, ctrl, reqs, hist, tail_len, win_start, table, free4, top4, free2, top2, tail, main4, lo4, main2, modes,
        end;
    int64_t n4, n2;
};

// Offsets of every region inside the caller's buffer for pool capacities n4, n2.
Layout layout(const loopkv_plan &p, int64_t n4, int64_t n2)
{
    const loopkv_config &c = p.cfg;
    const int64_t cells = p.n_cells();
    Layout L;
    size_t o = 0;
    L.status = o;
    o = align_up(o + 4);
    L.ctrl = o;
    o = align_up(o + 32);
    L.reqs = o;
    o = align_up(o + 4 * (int64_t)c.max_batch);
    L.hist = o;
    o = align_up(o + 4 * cells * c.max_batch);
    L.tail_len = o;
    o = align_up(o + 4 * cells * c.max_batch);
    L.win_start = o;
    o = align_up(o + 4 * cells * c.max_batch);
    L.table = o;
    o = align_up(o + 4 * cells * c.max_batch * (int64_t)c.max_blocks_per_seq);
    L.modes = o;
    o = align_up(o + cells);
    L.free4 = o;
    o = align_up(o + 4 * n4);
    L.top4 = o;
    o = align_up(o + 4);
    L.free2 = o;
    o = align_up(o + 4 * n2);
    L.top2 = o;
    o = align_up(o + 4);
    L.tail = o;
    o = align_up(o + (size_t)cells * c.max_batch * 2 * c.n_heads * near_cap(c) * c.head_dim * dtype_size(c.in_dtype));
    L.main4 = o;
    o = align_up(o + (size_t)n4 * c.n_heads * LKV_HEAD_MAIN_4B(c.head_dim));
    L.lo4 = o;
    o = align_up(o + (size_t)n4 * c.n_heads * LKV_HEAD_LO_4B(c.head_dim));
    L.main2 = o;
    o = align_up(o + (size_t)n2 * c.n_heads * LKV_HEAD_MAIN_2B(c.head_dim));
    L.end = o;
    L.n4 = n4;
    L.n2 = n2;
    return L;
}

void full_pools(const loopkv_plan &p, int64_t &n4, int64_t &n2)
{
    n4 = n2 = 0;
    const int64_t per = (int64_t)p.cfg.max_batch * p.cfg.max_blocks_per_seq;
    for (int cidx = 0; cidx < p.n_cells(); ++cidx) {
        if (p.modes[cidx] == LOOPKV_CELL_4B)
            n4 += per;
        else if (p.modes[cidx] == LOOPKV_CELL_2B)
            n2 += per;
    }
}

int cuda_err(cudaError_t e) { return e == cudaSuccess ? LOOPKV_OK : LOOPKV_ERR_CUDA; }

int check_cell(const loopkv_plan *p, int loop, int layer)
{
    if (loop < 0 || loop >= p->cfg.n_loops || layer < 0 || layer >= p->cfg.n_layers)
        return LOOPKV_ERR_INVALID_ARG;
    return LOOPKV_OK;
}

int check_device()
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess)
        return LOOPKV_ERR_NO_DEVICE;
    int major = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
        return LOOPKV_ERR_NO_DEVICE;
    return major == 10 ? LOOPKV_OK : LOOPKV_ERR_NO_DEVICE;
}

}  // namespace

int lkv::cache_info(const loopkv_cache *cache, lkv::CacheInfo *out)
{
    if (!cache || !out)
        return LOOPKV_ERR_INVALID_ARG;
    const loopkv_config &c = cache->plan.cfg;
    out->st = cache->st;
    out->n_loops = c.n_loops;
    out->n_layers = c.n_layers;
    out->n_heads = c.n_heads;
    out->head_dim = c.head_dim;
    out->in_dtype = c.in_dtype;
    out->max_batch = c.max_batch;
    return LOOPKV_OK;
}

extern "C" {

int loopkv_version(void) { return 100; }

const char *loopkv_strerror(int code)
{
    switch (code) {
    case LOOPKV_OK:
        return "ok";
    case LOOPKV_ERR_INVALID_ARG:
        return "invalid argument";
    case LOOPKV_ERR_SHAPE:
        return "shape inconsistent with the config";
    case LOOPKV_ERR_PLAN:
        return "invalid plan (share cell in the final loop or unknown mode)";
    case LOOPKV_ERR_POOL_EXHAUSTED:
        return "block pool exhausted";
    case LOOPKV_ERR_NONFINITE:
        return "non-finite value in a quantized group";
    case LOOPKV_ERR_RANGE:
        return "fp16 zero point or scale out of range";
    case LOOPKV_ERR_TIMEOUT:
        return "a bounded device wait timed out";
    case LOOPKV_ERR_CUDA:
        return "CUDA runtime error";
    case LOOPKV_ERR_TAIL_FULL:
        return "tail already holds 32 tokens (flush first)";
    case LOOPKV_ERR_STATE:
        return "cache state does not allow the operation";
    case LOOPKV_ERR_EMPTY_ROW:
        return "decode row with no token";
    case LOOPKV_ERR_NO_DEVICE:
        return "no CUDA device of compute capability 10.x";
    case LOOPKV_ERR_INFEASIBLE:
        return "no plan meets the damage and storage budgets";
    default:
        return "unknown error";
    }
}

int loopkv_plan_create(const loopkv_config *cfg, const uint8_t *modes, float tau, int tau_mode, loopkv_plan **out)
{
    if (!out || !modes)
        return LOOPKV_ERR_INVALID_ARG;
    *out = nullptr;
    int rc = check_config(cfg);
    if (rc)
        return rc;
    if (!(tau >= 0.f) || std::isinf(tau))
        return LOOPKV_ERR_INVALID_ARG;
    if (tau_mode != LOOPKV_TAU_REL_MAX && tau_mode != LOOPKV_TAU_ABS_PROB && tau_mode != LOOPKV_TAU_STREAM)
        return LOOPKV_ERR_INVALID_ARG;
    const int n = cfg->n_loops * cfg->n_layers;
    for (int c = 0; c < n; ++c) {
        if (modes[c] > LOOPKV_CELL_SHARE)
            return LOOPKV_ERR_PLAN;
        if (modes[c] == LOOPKV_CELL_SHARE && c / cfg->n_layers == cfg->n_loops - 1)
            return LOOPKV_ERR_PLAN; // the final loop stores its own pages
    }
    loopkv_plan *p = new (std::nothrow) loopkv_plan;
    if (!p)
        return LOOPKV_ERR_INVALID_ARG;
    p->cfg = *cfg;
    p->modes.assign(modes, modes + n);
    p->layer_window.assign(cfg->n_layers, 0);
    p->tau = tau;
    p->tau_mode = tau_mode;
    *out = p;
    return LOOPKV_OK;
}

void loopkv_plan_free(loopkv_plan *plan) { delete plan; }

int loopkv_plan_set_window(loopkv_plan *plan, int layer, int window_tokens)
{
    if (!plan || layer < 0 || layer >= plan->cfg.n_layers || window_tokens < 0)
        return LOOPKV_ERR_INVALID_ARG;
    plan->layer_window[layer] = window_tokens;
    return LOOPKV_OK;
}

int loopkv_plan_bytes(const loopkv_plan *plan, const float *hot_fraction, loopkv_byte_report *out)
{
    if (!plan || !out)
        return LOOPKV_ERR_INVALID_ARG;
    const int H = plan->cfg.n_heads, D = plan->cfg.head_dim;
    // per (token, head): 4-bit stored = main + lo; read = main + hot * lo; 2-bit = main
    const double m4 = LKV_HEAD_MAIN_4B(D) / 16.0, lo4 = LKV_HEAD_LO_4B(D) / 16.0, m2 = LKV_HEAD_MAIN_2B(D) / 16.0;
    loopkv_byte_report r = {};
    for (int c = 0; c < plan->n_cells(); ++c) {
        const int mode = plan->modes[c];
        const int src_mode = plan->modes[plan->src_cell(c)];
        double h = hot_fraction ? hot_fraction[c] : 1.0;
        if (!(h >= 0.0 && h <= 1.0))
            return LOOPKV_ERR_INVALID_ARG;
        if (mode == LOOPKV_CELL_4B)
            r.stored_bytes_per_token += H * (m4 + lo4);
        else if (mode == LOOPKV_CELL_2B)
            r.stored_bytes_per_token += H * m2;
        if (src_mode == LOOPKV_CELL_4B) {
            r.read_bytes_per_token += H * (m4 + h * lo4);
            r.read_bytes_all_hot += H * (m4 + lo4);
            r.read_bytes_all_cold += H * m4;
        } else {
            r.read_bytes_per_token += H * m2;
            r.read_bytes_all_hot += H * m2;
            r.read_bytes_all_cold += H * m2;
        }
        r.bf16_bytes_per_token += 2.0 * H * D * 2;
    }
    *out = r;
    return LOOPKV_OK;
}

int loopkv_required_bytes(const loopkv_plan *plan, size_t *bytes)
{
    if (!plan || !bytes)
        return LOOPKV_ERR_INVALID_ARG;
    int64_t n4, n2;
    full_pools(*plan, n4, n2);
    *bytes = layout(*plan, n4, n2).end;
    return LOOPKV_OK;
}

int loopkv_alloc(const loopkv_plan *plan, void *dev_buf, size_t dev_bytes, void *stream, loopkv_cache **out)
{
    if (!plan || !dev_buf || !out)
        return LOOPKV_ERR_INVALID_ARG;
    *out = nullptr;
    int rc = check_device();
    if (rc)
        return rc;
    if (reinterpret_cast<uintptr_t>(dev_buf) % kAlign)
        return LOOPKV_ERR_INVALID_ARG;
    int64_t n4, n2;
    full_pools(*plan, n4, n2);
    Layout L = layout(*plan, n4, n2);
    if (L.end > dev_bytes) {
        // shrink both pools in proportion to what is left after the fixed regions
        Layout L0 = layout(*plan, 0, 0);
        if (L0.end >= dev_bytes)
            return LOOPKV_ERR_POOL_EXHAUSTED;
        const int H = plan->cfg.n_heads, D = plan->cfg.head_dim;
        const double per4 = (double)H * (LKV_HEAD_MAIN_4B(D) + LKV_HEAD_LO_4B(D)) + 4;
        const double per2 = (double)H * LKV_HEAD_MAIN_2B(D) + 4;
        const double need = n4 * per4 + n2 * per2;
        double f = (double)(dev_bytes - L0.end - 8 * kAlign) / need;
        n4 = (int64_t)(n4 * f);
        n2 = (int64_t)(n2 * f);
        L = layout(*plan, n4, n2);
        while (L.end > dev_bytes && (n4 > 0 || n2 > 0)) {
            n4 = n4 * 99 / 100;
            n2 = n2 * 99 / 100;
            L = layout(*plan, n4, n2);
        }
        if (L.end > dev_bytes)
            return LOOPKV_ERR_POOL_EXHAUSTED;
    }
    if (n4 > INT32_MAX || n2 > INT32_MAX)
        return LOOPKV_ERR_SHAPE;
    loopkv_cache *c = new (std::nothrow) loopkv_cache;
    if (!c)
        return LOOPKV_ERR_INVALID_ARG;
    uint8_t *b = static_cast<uint8_t *>(dev_buf);
    c->plan = *plan;
    c->base = b;
    c->bytes = dev_bytes;
    c->esz = dtype_size(plan->cfg.in_dtype);
    lkv::DevState &st = c->st;
    st.status = reinterpret_cast<uint32_t *>(b + L.status);
    st.ctrl = reinterpret_cast<int32_t *>(b + L.ctrl);
    st.hist_len = reinterpret_cast<int32_t *>(b + L.hist);
    st.tail_len = reinterpret_cast<int32_t *>(b + L.tail_len);
    st.win_start = reinterpret_cast<int32_t *>(b + L.win_start);
    st.sink = plan->cfg.sink_tokens;
    st.wring = plan->cfg.window_tokens + 32;
    st.near_cap = near_cap(plan->cfg);
    st.block_table = reinterpret_cast<int32_t *>(b + L.table);
    st.free4 = reinterpret_cast<int32_t *>(b + L.free4);
    st.top4 = reinterpret_cast<int32_t *>(b + L.top4);
    st.free2 = reinterpret_cast<int32_t *>(b + L.free2);
    st.top2 = reinterpret_cast<int32_t *>(b + L.top2);
    st.n4 = n4;
    st.n2 = n2;
    st.tail = b + L.tail;
    st.main4 = b + L.main4;
    st.lo4 = b + L.lo4;
    st.main2 = b + L.main2;
    c->modes_dev = b + L.modes;
    c->req_stage = reinterpret_cast<int32_t *>(b + L.reqs);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // zero the control region (status .. block table); the tail and pools need no init
    rc = cuda_err(cudaMemsetAsync(b, 0, L.modes, s));
    if (!rc)
        rc = cuda_err(cudaMemcpyAsync(c->modes_dev, plan->modes.data(), plan->modes.size(), cudaMemcpyHostToDevice, s));
    if (!rc)
        rc = lkv::launch_init_state(st, s);
    if (!rc)
        rc = cuda_err(cudaStreamSynchronize(s)); // the modes copy reads host memory owned by the plan
    if (rc) {
        delete c;
        return rc;
    }
    *out = c;
    return LOOPKV_OK;
}

void loopkv_free(loopkv_cache *cache) { delete cache; }

int loopkv_ingest(loopkv_cache *cache, int loop, int layer, int req, const void *k, const void *v, int T, void *stream)
{
    if (!cache || !k || !v)
        return LOOPKV_ERR_INVALID_ARG;
    const loopkv_plan &p = cache->plan;
    int rc = check_cell(&p, loop, layer);
    if (rc)
        return rc;
    if (req < 0 || req >= p.cfg.max_batch || T < 0)
        return LOOPKV_ERR_INVALID_ARG;
    if (T / LKV_GROUP * 2 > p.cfg.max_blocks_per_seq)
        return LOOPKV_ERR_SHAPE;
    const int cell = p.cell(loop, layer);
    cache->mark_state_written(stream);
    return lkv::launch_ingest(cache->st, cell, p.modes[cell], p.cfg.n_heads, p.cfg.head_dim, p.cfg.in_dtype,
                              p.cfg.max_batch, p.cfg.max_blocks_per_seq, req, k, v, T,
                              static_cast<cudaStream_t>(stream));
}

int loopkv_append(loopkv_cache *cache, int loop, int layer, const void *k, const void *v, const int32_t *req_ids,
                  int B, void *stream)
{
    if (!cache || !k || !v || B < 0)
        return LOOPKV_ERR_INVALID_ARG;
    const loopkv_plan &p = cache->plan;
    int rc = check_cell(&p, loop, layer);
    if (rc)
        return rc;
    if (B > p.cfg.max_batch)
        return LOOPKV_ERR_SHAPE;
    const int32_t *ids_dev = nullptr;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (req_ids) {
        for (int i = 0; i < B; ++i)
            if (req_ids[i] < 0 || req_ids[i] >= p.cfg.max_batch)
                return LOOPKV_ERR_INVALID_ARG;
        rc = cuda_err(cudaMemcpyAsync(cache->req_stage, req_ids, sizeof(int32_t) * B, cudaMemcpyHostToDevice, s));
        if (rc)
            return rc;
        ids_dev = cache->req_stage;
    }
    return lkv::launch_append(cache->st, p.cell(loop, layer), p.cfg.n_heads, p.cfg.head_dim, p.cfg.in_dtype,
                              p.cfg.max_batch, k, v, ids_dev, B, s);
}

int loopkv_flush(loopkv_cache *cache, void *stream)
{
    if (!cache)
        return LOOPKV_ERR_INVALID_ARG;
    const loopkv_plan &p = cache->plan;
    cache->mark_state_written(stream);
    return lkv::launch_flush(cache->st, cache->modes_dev, p.n_cells(), p.cfg.n_heads, p.cfg.head_dim, p.cfg.in_dtype,
                             p.cfg.max_batch, p.cfg.max_blocks_per_seq, static_cast<cudaStream_t>(stream));
}

int loopkv_reset_request(loopkv_cache *cache, int req, void *stream)
{
    if (!cache)
        return LOOPKV_ERR_INVALID_ARG;
    const loopkv_plan &p = cache->plan;
    if (req < 0 || req >= p.cfg.max_batch)
        return LOOPKV_ERR_INVALID_ARG;
    cache->mark_state_written(stream);
    return lkv::launch_reset(cache->st, cache->modes_dev, p.n_cells(), p.cfg.max_batch, p.cfg.max_blocks_per_seq, req,
                             static_cast<cudaStream_t>(stream));
}

int loopkv_decode_debug(const loopkv_plan *plan, int loop, int layer, const void *q, const loopkv_cache *ccache,
                        float *out, int B, void *stream, uint32_t *s_bitmap, float *row_max, float *row_sum)
{
    if (!plan || !ccache || !q || !out)
        return LOOPKV_ERR_INVALID_ARG;
    loopkv_cache *cache = const_cast<loopkv_cache *>(ccache); // only the host bookkeeping changes
    int rc = check_cell(plan, loop, layer);
    if (rc)
        return rc;
    const loopkv_plan &cp = cache->plan;
    if (plan->cfg.n_loops != cp.cfg.n_loops || plan->cfg.n_layers != cp.cfg.n_layers ||
        plan->cfg.n_heads != cp.cfg.n_heads || plan->cfg.head_dim != cp.cfg.head_dim ||
        plan->cfg.in_dtype != cp.cfg.in_dtype || plan->modes != cp.modes)
        return LOOPKV_ERR_PLAN; // the storage of a cache is fixed by the plan it was built with
    if (B <= 0 || B > cp.cfg.max_batch)
        return LOOPKV_ERR_SHAPE;
    const int cell = cp.cell(loop, layer), src = cp.src_cell(cell);
    const int bits = cp.modes[src] == LOOPKV_CELL_4B ? 4 : 2;
    const int H = cp.cfg.n_heads, D = cp.cfg.head_dim, MB = cp.cfg.max_blocks_per_seq;
    lkv::DecodeArgs a = {};
    a.q = q;
    a.out = out;
    a.main = bits == 4 ? cache->st.main4 : cache->st.main2;
    a.lo = cache->st.lo4;
    a.block_table = cache->st.block_table + (int64_t)src * cp.cfg.max_batch * MB;
    a.hist_len = cache->st.hist_len + (int64_t)src * cp.cfg.max_batch;
    a.tail_len = cache->st.tail_len + (int64_t)cell * cp.cfg.max_batch;
    a.win_start = cache->st.win_start + (int64_t)cell * cp.cfg.max_batch;
    a.tail = cache->st.tail + (size_t)cell * cp.cfg.max_batch * 2 * H * cache->st.near_cap * D * cache->esz;
    a.sink = cache->st.sink;
    a.wring = cache->st.wring;
    a.near_cap = cache->st.near_cap;
    a.status = cache->st.status;
    a.s_bitmap = s_bitmap;
    a.row_max = row_max;
    a.row_sum = row_sum;
    a.pool_blocks = bits == 4 ? cache->st.n4 : cache->st.n2;
    a.H = H;
    a.rows = B * H;
    a.max_blocks = MB;
    a.bitmap_words = MB / 2;
    a.qscale = (float)(1.4426950408889634 / std::sqrt((double)D));
    a.tau = plan->tau;
    a.tau_mode = plan->tau_mode;
    a.attn_window = plan->layer_window[layer];
    const lkv::DecodeShape shp = cache->shape(bits, B, single_pass(bits, plan->tau), a.attn_window);
    a.cap_groups = shp.cap;
    {
        std::lock_guard<std::mutex> lock(cache->mu);
        a.wait_ns = cache->wait_ns;
        a.inject = cache->inject;
    }
    // a windowed read sets up its rows from the near counts, which appends write: no overlap
    const bool overlap = cache->decode_may_overlap(stream) && a.attn_window == 0;
    return lkv::launch_decode(a, bits, D, cp.cfg.in_dtype, shp, overlap, static_cast<cudaStream_t>(stream));
}

int loopkv_decode(const loopkv_plan *plan, int loop, int layer, const void *q, const loopkv_cache *cache, float *out,
                  int B, void *stream)
{
    return loopkv_decode_debug(plan, loop, layer, q, cache, out, B, stream, nullptr, nullptr, nullptr);
}

int loopkv_status(loopkv_cache *cache, void *stream, int *device_status)
{
    if (!cache)
        return LOOPKV_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint32_t w = 0;
    int rc = cuda_err(cudaStreamSynchronize(s));
    if (!rc)
        rc = cuda_err(cudaMemcpy(&w, cache->st.status, 4, cudaMemcpyDeviceToHost));
    if (!rc)
        rc = cuda_err(cudaMemset(cache->st.status, 0, 4));
    if (rc)
        return rc;
    if (device_status)
        *device_status = (int)w;
    if (w & LOOPKV_DEV_TIMEOUT)
        return LOOPKV_ERR_TIMEOUT;
    if (w & LOOPKV_DEV_NONFINITE)
        return LOOPKV_ERR_NONFINITE;
    if (w & LOOPKV_DEV_RANGE)
        return LOOPKV_ERR_RANGE;
    if (w & LOOPKV_DEV_POOL_EXHAUSTED)
        return LOOPKV_ERR_POOL_EXHAUSTED;
    if (w & LOOPKV_DEV_TAIL_FULL)
        return LOOPKV_ERR_TAIL_FULL;
    if (w & LOOPKV_DEV_STATE)
        return LOOPKV_ERR_STATE;
    if (w & LOOPKV_DEV_EMPTY_ROW)
        return LOOPKV_ERR_EMPTY_ROW;
    return LOOPKV_OK;
}

int loopkv_set_wait_policy(loopkv_cache *cache, uint64_t wait_limit_ns, int inject)
{
    if (!cache || wait_limit_ns == 0 || (inject != LOOPKV_INJECT_NONE && inject != LOOPKV_INJECT_STALLED_STAGE))
        return LOOPKV_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> lock(cache->mu);
    cache->wait_ns = wait_limit_ns;
    cache->inject = inject;
    return LOOPKV_OK;
}

int loopkv_cell_view_get(const loopkv_cache *cache, int loop, int layer, loopkv_cell_view *out)
{
    if (!cache || !out)
        return LOOPKV_ERR_INVALID_ARG;
    const loopkv_plan &p = cache->plan;
    int rc = check_cell(&p, loop, layer);
    if (rc)
        return rc;
    const int cell = p.cell(loop, layer), src = p.src_cell(cell);
    const int bits = p.modes[src] == LOOPKV_CELL_4B ? 4 : 2;
    const int H = p.cfg.n_heads, D = p.cfg.head_dim, MB = p.cfg.max_blocks_per_seq;
    out->mode = p.modes[cell];
    out->src_cell = src;
    out->src_mode = p.modes[src];
    out->head_main_bytes = head_main_bytes(bits, D);
    out->head_lo_bytes = bits == 4 ? LKV_HEAD_LO_4B(D) : 0;
    out->main_pool = bits == 4 ? cache->st.main4 : cache->st.main2;
    out->lo_pool = bits == 4 ? cache->st.lo4 : nullptr;
    out->block_table = cache->st.block_table + (int64_t)src * p.cfg.max_batch * MB;
    out->hist_len = cache->st.hist_len + (int64_t)src * p.cfg.max_batch;
    out->tail_len = cache->st.tail_len + (int64_t)cell * p.cfg.max_batch;
    out->win_start = cache->st.win_start + (int64_t)cell * p.cfg.max_batch;
    out->tail = cache->st.tail + (size_t)cell * p.cfg.max_batch * 2 * H * cache->st.near_cap * D * cache->esz;
    out->near_cap = cache->st.near_cap;
    out->pool_blocks = bits == 4 ? cache->st.n4 : cache->st.n2;
    return LOOPKV_OK;
}

int loopkv_decode_shape(const loopkv_plan *plan, int B, int *cluster_size, int *ctas, int *smem_bytes)
{
    if (!plan || B <= 0)
        return LOOPKV_ERR_INVALID_ARG;
    if (check_device())
        return LOOPKV_ERR_NO_DEVICE; // the shape comes from an occupancy query of the device
    // the shape of a 4-bit source cell (the larger pipeline stage) under the plan's tau
    lkv::DecodeShape shp = lkv::decode_shape(4, plan->cfg.head_dim, plan->cfg.in_dtype, B * plan->cfg.n_heads,
                                             plan->cfg.max_blocks_per_seq, near_cap(plan->cfg), single_pass(4, plan->tau));
    if (cluster_size)
        *cluster_size = shp.cluster;
    if (ctas)
        *ctas = shp.cluster * shp.clusters;
    if (smem_bytes)
        *smem_bytes = shp.smem;
    return shp.cluster > 0 ? LOOPKV_OK : LOOPKV_ERR_CUDA;
}

}  // extern "C"
