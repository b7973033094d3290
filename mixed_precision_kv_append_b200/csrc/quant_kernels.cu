// quant_kernels.cu -- append, window-exit flush, bulk ingest and request reset.
//
// The quantizer is KIVI-style asymmetric quantization with an fp16 zero point and
// fp16 scale per group of 32 (LoopKV paper, §5.1 "Baselines and ablations": groups
// of 32): keys per channel over the 32 tokens of a page, values per token over 32
// channels (Appendix "History reader": per-channel key scale constant over a page,
// per-token value scale).  A 4-bit value code is stored as a hi plane (code >> 2)
// and a separate lo plane (code & 3) (§3.3 "Bit-plane V layout").  Pages are
// quantized when they leave the unquantized tail (§2.3: "each 32-token page is
// processed by the policy when it leaves the window").  Rounding: zero = largest
// fp16 <= min, scale = smallest fp16 >= (max - zero) / L in fp64, code = nearest
// level of the IEEE fp32 quotient (ties to even); see loopkv_format.h.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "lkv_device.cuh"
#include "lkv_internal.h"

namespace lkv {
namespace {

constexpr int kQThreads = 128;

// Quantize 32 values held by one thread.  Returns the LOOPKV_DEV_* bit of an error (0 if ok).
template <int L>
__device__ __forceinline__ uint32_t quant32(const float (&x)[32], uint16_t &zb, uint16_t &sb, uint8_t (&code)[32])
{
    float mn = x[0], mx = x[0];
    bool finite = true;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
        finite &= isfinite(x[i]);
        mn = fminf(mn, x[i]);
        mx = fmaxf(mx, x[i]);
    }
    uint32_t err = 0;
    float z = 0.f, s = 0.f;
    if (!finite) {
        err = LOOPKV_DEV_NONFINITE;
    } else {
        __half zh = __float2half_rd(mn);
        z = __half2float(zh);
        if (isinf(z)) {
            err = LOOPKV_DEV_RANGE;
        } else {
            double r = __ddiv_rn(__dsub_rn((double)mx, (double)z), (double)L);
            __half sh = __float2half_ru(__double2float_ru(r));
            s = __half2float(sh);
            if (isinf(s)) {
                err = LOOPKV_DEV_RANGE;
            } else {
                zb = __half_as_ushort(zh);
                sb = __half_as_ushort(sh);
            }
        }
    }
    if (err) {
        zb = 0;
        sb = 0;
#pragma unroll
        for (int i = 0; i < 32; ++i)
            code[i] = 0;
        return err;
    }
#pragma unroll
    for (int i = 0; i < 32; ++i) {
        int c = 0;
        if (s != 0.f) {
            c = __float2int_rn(__fdiv_rn(__fsub_rn(x[i], z), s));
            c = c < 0 ? 0 : (c > L ? L : c);
        }
        code[i] = (uint8_t)c;
    }
    return 0;
}

template <int D> struct QGeo {
    static constexpr int KCODES4 = 16 * D / 2;
    static constexpr int KCODES2 = 16 * D / 4;
    static constexpr int KMETA = 2 * D;
    static constexpr int VMETA = 16 * (D / 32) * 4;
};

// Pack the 2-bit codes of 16 consecutive channels into one word: channel 4i+b at
// bit 8b+2i.
__device__ __forceinline__ uint32_t pack2_16(const uint8_t *c, int shift, int mask)
{
    uint32_t w = 0;
#pragma unroll
    for (int r = 0; r < 16; ++r) {
        int b = r & 3, i = r >> 2;
        w |= (uint32_t)((c[r] >> shift) & mask) << (8 * b + 2 * i);
    }
    return w;
}

// Quantize one 32-token group of one head into the head regions of its two blocks.
//   ksrc/vsrc: element (t, c) at src[t * tok_stride + c], t in [0,32), c in [0,D)
//   main0/main1: head main regions of the even / odd block; lo0/lo1: lo regions (4-bit)
//   kc_smem: [32][D] bytes of shared scratch.  All threads of the CTA take part.
template <int BITS, int D, typename DT>
__device__ void quant_group_head(const DT *ksrc, const DT *vsrc, int64_t tok_stride, uint8_t *main0,
                                 uint8_t *main1, uint8_t *lo0, uint8_t *lo1, uint32_t *status, uint8_t *kc_smem)
{
    using G = QGeo<D>;
    constexpr int L = (1 << BITS) - 1;
    constexpr int KCODES = BITS == 4 ? G::KCODES4 : G::KCODES2;
    constexpr int ROWK = KCODES / 16;
    const int tid = threadIdx.x;
    uint32_t err = 0;

    // Keys: one thread per channel, grouped over the 32 tokens.
    for (int c = tid; c < D; c += kQThreads) {
        float x[32];
#pragma unroll
        for (int t = 0; t < 32; ++t)
            x[t] = to_f32(ksrc[(int64_t)t * tok_stride + c]);
        uint16_t zb, sb;
        uint8_t code[32];
        err |= quant32<L>(x, zb, sb, code);
        reinterpret_cast<uint16_t *>(main0 + KCODES)[c] = sb; // even block: scales
        reinterpret_cast<uint16_t *>(main1 + KCODES)[c] = zb; // odd block: zero points
#pragma unroll
        for (int t = 0; t < 32; ++t)
            kc_smem[t * D + c] = code[t];
    }
    __syncthreads();
    // Pack key rows: 4-bit word w = channels 8w..8w+7 (byte b: low nibble 8w+b, high
    // nibble 8w+4+b); 2-bit word w = channels 16w..16w+15 (channel 4i+b at bit 8b+2i).
    constexpr int WPR = ROWK / 4; // words per row
    for (int n = tid; n < 32 * WPR; n += kQThreads) {
        int t = n / WPR, w = n % WPR;
        const uint8_t *cr = kc_smem + t * D;
        uint32_t word = 0;
        if (BITS == 4) {
#pragma unroll
            for (int b = 0; b < 4; ++b)
                word |= (uint32_t)((cr[8 * w + b] & 15) | ((cr[8 * w + 4 + b] & 15) << 4)) << (8 * b);
        } else {
            word = pack2_16(cr + 16 * w, 0, 3);
        }
        uint8_t *m = (t < 16) ? main0 : main1;
        reinterpret_cast<uint32_t *>(m + (t & 15) * ROWK)[w] = word;
    }
    __syncthreads(); // the key rows are packed: the scratch now takes the value codes
    // Values: one thread per (token, 32-channel group); the (scale, zero) pair goes to
    // [group][token] of the block's V meta, the codes to the scratch.
    constexpr int NCG = D / 32;
    for (int u = tid; u < 32 * NCG; u += kQThreads) {
        int t = u / NCG, j = u % NCG;
        const DT *row = vsrc + (int64_t)t * tok_stride + 32 * j;
        float x[32];
#pragma unroll
        for (int i = 0; i < 32; ++i)
            x[i] = to_f32(row[i]);
        uint16_t zb, sb;
        uint8_t code[32];
        err |= quant32<L>(x, zb, sb, code);
        uint8_t *m = (t < 16) ? main0 : main1;
        uint16_t *meta = reinterpret_cast<uint16_t *>(m + KCODES + G::KMETA + (j * 16 + (t & 15)) * 4);
        meta[0] = sb;
        meta[1] = zb;
#pragma unroll
        for (int i = 0; i < 32; ++i)
            kc_smem[t * D + 32 * j + i] = code[i];
    }
    __syncthreads();
    // Planes: one thread per (block, channel quad kappa, token quad tau) word; byte b of a
    // word is token 4tau+b, its bits 2i..2i+1 channel 4kappa+i.  hi words (the 2-bit codes
    // of a 2-bit cell) at index 4kappa+tau, lo words at tau*(D/4)+kappa.
    for (int n = tid; n < 2 * D; n += kQThreads) {
        const int blk = n / D, kappa = (n % D) >> 2, tau = n & 3;
        uint32_t hw = 0, lw = 0;
#pragma unroll
        for (int b = 0; b < 4; ++b)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const uint32_t code = kc_smem[(16 * blk + 4 * tau + b) * D + 4 * kappa + i];
                hw |= (BITS == 4 ? code >> 2 : code) << (8 * b + 2 * i);
                lw |= (code & 3u) << (8 * b + 2 * i);
            }
        uint8_t *m = blk ? main1 : main0;
        reinterpret_cast<uint32_t *>(m + KCODES + G::KMETA + G::VMETA)[4 * kappa + tau] = hw;
        if (BITS == 4)
            reinterpret_cast<uint32_t *>(blk ? lo1 : lo0)[tau * (D / 4) + kappa] = lw;
    }
    if (err)
        atomicOr(status, err);
    __syncthreads();
}

// Pop `k` block ids from a free stack; ids[i] gets the i-th popped id.  One thread.
__device__ bool pop_blocks(int32_t *free_ids, int32_t *top, int k, int32_t *ids)
{
    int old = atomicSub(top, k);
    if (old < k) {
        atomicAdd(top, k);
        return false;
    }
    for (int i = 0; i < k; ++i)
        ids[i] = free_ids[old - 1 - i];
    return true;
}

struct PoolPtrs {
    uint8_t *main;
    uint8_t *lo;
    int head_main, head_lo;
    int32_t *free_ids;
    int32_t *top;
};

__device__ PoolPtrs pool_ptrs(const DevState &st, int bits, int D)
{
    PoolPtrs p;
    if (bits == 4) {
        p.main = st.main4;
        p.lo = st.lo4;
        p.head_main = LKV_HEAD_MAIN_4B(D);
        p.head_lo = LKV_HEAD_LO_4B(D);
        p.free_ids = st.free4;
        p.top = st.top4;
    } else {
        p.main = st.main2;
        p.lo = nullptr;
        p.head_main = LKV_HEAD_MAIN_2B(D);
        p.head_lo = 0;
        p.free_ids = st.free2;
        p.top = st.top2;
    }
    return p;
}

// Quantize one group of one head whose two blocks are ids[0], ids[1].
template <int D, typename DT>
__device__ void quant_into_blocks(const DevState &st, int bits, int H, int h, const int32_t *ids, const DT *ksrc,
                                  const DT *vsrc, int64_t tok_stride, uint8_t *kc_smem)
{
    PoolPtrs p = pool_ptrs(st, bits, D);
    uint8_t *m0 = p.main + ((int64_t)ids[0] * H + h) * p.head_main;
    uint8_t *m1 = p.main + ((int64_t)ids[1] * H + h) * p.head_main;
    if (bits == 4) {
        uint8_t *l0 = p.lo + ((int64_t)ids[0] * H + h) * p.head_lo;
        uint8_t *l1 = p.lo + ((int64_t)ids[1] * H + h) * p.head_lo;
        quant_group_head<4, D, DT>(ksrc, vsrc, tok_stride, m0, m1, l0, l1, st.status, kc_smem);
    } else {
        quant_group_head<2, D, DT>(ksrc, vsrc, tok_stride, m0, m1, nullptr, nullptr, st.status, kc_smem);
    }
}

// Slot of near token j (arrival order among the tokens held) of a (cell, request): the
// sink slots first, then the window ring of st.wring slots from its oldest token.
__device__ __forceinline__ int near_slot(const DevState &st, int j, int win_start)
{
    return j < st.sink ? j : st.sink + (win_start + (j - st.sink)) % st.wring;
}

__global__ void init_state_kernel(DevState st)
{
    int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t k = i; k < st.n4; k += stride)
        st.free4[k] = (int32_t)(st.n4 - 1 - k);
    for (int64_t k = i; k < st.n2; k += stride)
        st.free2[k] = (int32_t)(st.n2 - 1 - k);
    if (i == 0) {
        *st.top4 = (int32_t)st.n4;
        *st.top2 = (int32_t)st.n2;
    }
}

// One CTA per request: copy this step's K and V of every head into the tail.
template <typename DT>
__global__ void append_kernel(DevState st, int cell, int H, int D, int max_batch, const DT *k, const DT *v,
                              const int32_t *req_ids, int B)
{
    __shared__ int s_pos;
    const int bi = blockIdx.x;
    const int req = req_ids ? req_ids[bi] : bi;
    const bool bad_req = req < 0 || req >= max_batch;
    if (threadIdx.x == 0) {
        int pos = -1;
        if (bad_req) {
            atomicOr(st.status, LOOPKV_DEV_STATE);
        } else {
            pos = st.tail_len[(int64_t)cell * max_batch + req];
            if (pos >= st.sink + st.wring || pos < 0) { // window full: flush first
                atomicOr(st.status, LOOPKV_DEV_TAIL_FULL);
                pos = -1;
            }
        }
        s_pos = pos;
    }
    __syncthreads();
    const int pos = s_pos;
    if (pos < 0)
        return;
    const int slot = near_slot(st, pos, st.win_start[(int64_t)cell * max_batch + req]);
    const int NC = st.near_cap;
    DT *tail = reinterpret_cast<DT *>(st.tail) + ((int64_t)cell * max_batch + req) * 2 * H * NC * D;
    const int64_t HD = (int64_t)H * D;
    for (int64_t e = threadIdx.x; e < HD; e += blockDim.x) {
        int h = (int)(e / D), c = (int)(e % D);
        tail[((int64_t)h * NC + slot) * D + c] = k[(int64_t)bi * HD + e];
        tail[((int64_t)(H + h) * NC + slot) * D + c] = v[(int64_t)bi * HD + e];
    }
    __syncthreads();
    if (threadIdx.x == 0)
        st.tail_len[(int64_t)cell * max_batch + req] = pos + 1;
}

// One CTA per (cell, request): the oldest 32 tokens of a window holding W + 32 become two
// new blocks (the window ring's oldest page, contiguous in the ring).
template <int D, typename DT>
__global__ void __launch_bounds__(kQThreads) flush_kernel(DevState st, const uint8_t *modes, int H, int max_batch,
                                                          int max_blocks)
{
    __shared__ int32_t s_ids[2];
    __shared__ int s_go;
    __shared__ __align__(16) uint8_t kc_smem[32 * D];
    const int cell = blockIdx.x / max_batch, req = blockIdx.x % max_batch;
    int32_t *tl = st.tail_len + (int64_t)cell * max_batch + req;
    int32_t *hl = st.hist_len + (int64_t)cell * max_batch + req;
    int32_t *ws = st.win_start + (int64_t)cell * max_batch + req;
    const int mode = modes[cell];
    if (threadIdx.x == 0) {
        int go = 0;
        if (*tl == st.sink + st.wring) {
            int nb = *hl / LKV_BLOCK_TOKENS;
            if (nb + 2 > max_blocks) {
                atomicOr(st.status, LOOPKV_DEV_STATE);
            } else if (mode == LOOPKV_CELL_SHARE) {
                go = 2; // a share cell only empties its tail; its pages are the final loop's
            } else {
                PoolPtrs p = pool_ptrs(st, mode == LOOPKV_CELL_4B ? 4 : 2, D);
                if (pop_blocks(p.free_ids, p.top, 2, s_ids)) {
                    int32_t *bt = st.block_table + ((int64_t)cell * max_batch + req) * max_blocks;
                    bt[nb] = s_ids[0];
                    bt[nb + 1] = s_ids[1];
                    go = 1;
                } else {
                    atomicOr(st.status, LOOPKV_DEV_POOL_EXHAUSTED);
                }
            }
        }
        s_go = go;
    }
    __syncthreads();
    const int go = s_go;
    if (go == 0)
        return;
    if (go == 1) {
        const int bits = mode == LOOPKV_CELL_4B ? 4 : 2;
        const int NC = st.near_cap, slot0 = st.sink + *ws;
        const DT *tail = reinterpret_cast<const DT *>(st.tail) + ((int64_t)cell * max_batch + req) * 2 * H * NC * D;
        for (int h = 0; h < H; ++h)
            quant_into_blocks<D, DT>(st, bits, H, h, s_ids, tail + ((int64_t)h * NC + slot0) * D,
                                     tail + ((int64_t)(H + h) * NC + slot0) * D, D, kc_smem);
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        *hl = *hl + LKV_GROUP;
        *tl = *tl - LKV_GROUP;
        *ws = (*ws + LKV_GROUP) % st.wring;
    }
}

// Ingest, step 1 (one thread): admit the (cell, request) if empty, take its blocks,
// set its lengths.  ctrl[0] = 1 admits the following ingest kernels.
__global__ void ingest_prep_kernel(DevState st, int cell, int mode, int D, int max_batch, int max_blocks, int req,
                                   int T, int ngroups)
{
    int32_t *tl = st.tail_len + (int64_t)cell * max_batch + req;
    int32_t *hl = st.hist_len + (int64_t)cell * max_batch + req;
    st.ctrl[0] = 0;
    if (*tl != 0 || *hl != 0 || 2 * ngroups > max_blocks) {
        atomicOr(st.status, LOOPKV_DEV_STATE);
        return;
    }
    if (mode != LOOPKV_CELL_SHARE && ngroups > 0) {
        PoolPtrs p = pool_ptrs(st, mode == LOOPKV_CELL_4B ? 4 : 2, D);
        int k = 2 * ngroups;
        int old = atomicSub(p.top, k);
        if (old < k) {
            atomicAdd(p.top, k);
            atomicOr(st.status, LOOPKV_DEV_POOL_EXHAUSTED);
            return;
        }
        int32_t *bt = st.block_table + ((int64_t)cell * max_batch + req) * max_blocks;
        for (int i = 0; i < k; ++i)
            bt[i] = p.free_ids[old - 1 - i];
    }
    *hl = ngroups * LKV_GROUP;
    *tl = T - ngroups * LKV_GROUP; // sink fill + window length
    st.win_start[(int64_t)cell * max_batch + req] = 0;
    st.ctrl[0] = 1;
}

// Ingest, step 2: one CTA per (group, head).
template <int D, typename DT>
__global__ void __launch_bounds__(kQThreads) ingest_quant_kernel(DevState st, int cell, int mode, int H,
                                                                 int max_batch, int max_blocks, int req,
                                                                 const DT *k, const DT *v, int t0)
{
    __shared__ __align__(16) uint8_t kc_smem[32 * D];
    if (st.ctrl[0] != 1)
        return;
    const int g = blockIdx.x, h = blockIdx.y;
    const int32_t *bt = st.block_table + ((int64_t)cell * max_batch + req) * max_blocks;
    int32_t ids[2] = {bt[2 * g], bt[2 * g + 1]};
    const int64_t tok = (int64_t)H * D;
    const int64_t off = ((int64_t)t0 + (int64_t)g * LKV_GROUP) * tok + (int64_t)h * D; // pages start after the sink
    quant_into_blocks<D, DT>(st, mode == LOOPKV_CELL_4B ? 4 : 2, H, h, ids, k + off, v + off, tok, kc_smem);
}

// Ingest, step 3: the unquantized tokens go to the near region: the first sf (sink) to
// slots 0..sf-1, the last nw (window) to the ring from its slot 0.
template <typename DT>
__global__ void ingest_tail_kernel(DevState st, int cell, int H, int D, int max_batch, int req, const DT *k,
                                   const DT *v, int T, int sf, int nw)
{
    if (st.ctrl[0] != 1)
        return;
    const int NC = st.near_cap;
    DT *tail = reinterpret_cast<DT *>(st.tail) + ((int64_t)cell * max_batch + req) * 2 * H * NC * D;
    const int64_t HD = (int64_t)H * D;
    for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < (int64_t)(sf + nw) * HD;
         e += (int64_t)gridDim.x * blockDim.x) {
        const int j = (int)(e / HD); // near token j: sink token j, or window token j - sf
        const int64_t r = e % HD;
        const int h = (int)(r / D), c = (int)(r % D);
        const int t = j < sf ? j : T - nw + (j - sf);
        const int slot = j < sf ? j : st.sink + (j - sf);
        tail[((int64_t)h * NC + slot) * D + c] = k[(int64_t)t * HD + r];
        tail[((int64_t)(H + h) * NC + slot) * D + c] = v[(int64_t)t * HD + r];
    }
}

// Release a request slot in every cell.  One thread per cell.
__global__ void reset_kernel(DevState st, const uint8_t *modes, int n_cells, int max_batch, int max_blocks, int req,
                             int D)
{
    int cell = blockIdx.x * blockDim.x + threadIdx.x;
    if (cell >= n_cells)
        return;
    int32_t *tl = st.tail_len + (int64_t)cell * max_batch + req;
    int32_t *hl = st.hist_len + (int64_t)cell * max_batch + req;
    const int mode = modes[cell];
    if (mode != LOOPKV_CELL_SHARE) {
        int nb = *hl / LKV_BLOCK_TOKENS;
        if (nb > max_blocks)
            nb = max_blocks;
        if (nb > 0) {
            PoolPtrs p = pool_ptrs(st, mode == LOOPKV_CELL_4B ? 4 : 2, D);
            const int32_t *bt = st.block_table + ((int64_t)cell * max_batch + req) * max_blocks;
            int old = atomicAdd(p.top, nb);
            for (int i = 0; i < nb; ++i)
                p.free_ids[old + i] = bt[nb - 1 - i];
        }
    }
    *hl = 0;
    *tl = 0;
    st.win_start[(int64_t)cell * max_batch + req] = 0;
}

}  // namespace

static int cuda_status(cudaError_t e) { return e == cudaSuccess ? LOOPKV_OK : LOOPKV_ERR_CUDA; }

int launch_init_state(const DevState &st, cudaStream_t s)
{
    init_state_kernel<<<1184, 256, 0, s>>>(st);
    return cuda_status(cudaGetLastError());
}

int launch_append(const DevState &st, int cell, int H, int D, int dtype, int max_batch, const void *k,
                  const void *v, const int32_t *req_ids_dev, int B, cudaStream_t s)
{
    if (B <= 0)
        return LOOPKV_OK;
    if (dtype == LOOPKV_DTYPE_BF16)
        append_kernel<__nv_bfloat16><<<B, 256, 0, s>>>(st, cell, H, D, max_batch, (const __nv_bfloat16 *)k,
                                                       (const __nv_bfloat16 *)v, req_ids_dev, B);
    else
        append_kernel<float><<<B, 256, 0, s>>>(st, cell, H, D, max_batch, (const float *)k, (const float *)v,
                                               req_ids_dev, B);
    return cuda_status(cudaGetLastError());
}

template <int D>
static void flush_dispatch(const DevState &st, const uint8_t *modes, int n_cells, int H, int dtype, int max_batch,
                           int max_blocks, cudaStream_t s)
{
    dim3 grid(n_cells * max_batch);
    if (dtype == LOOPKV_DTYPE_BF16)
        flush_kernel<D, __nv_bfloat16><<<grid, kQThreads, 0, s>>>(st, modes, H, max_batch, max_blocks);
    else
        flush_kernel<D, float><<<grid, kQThreads, 0, s>>>(st, modes, H, max_batch, max_blocks);
}

int launch_flush(const DevState &st, const uint8_t *cell_modes_dev, int n_cells, int H, int D, int dtype,
                 int max_batch, int max_blocks, cudaStream_t s)
{
    if (D == 128)
        flush_dispatch<128>(st, cell_modes_dev, n_cells, H, dtype, max_batch, max_blocks, s);
    else
        flush_dispatch<64>(st, cell_modes_dev, n_cells, H, dtype, max_batch, max_blocks, s);
    return cuda_status(cudaGetLastError());
}

template <int D, typename DT>
static void ingest_dispatch(const DevState &st, int cell, int mode, int H, int max_batch, int max_blocks, int req,
                            const void *k, const void *v, int T, cudaStream_t s)
{
    // sink sf = min(T, sink); of the rest R, 32 * floor((R - W) / 32) pages (none if R < W),
    // then the window
    const int W = st.wring - LKV_GROUP;
    const int sf = T < st.sink ? T : st.sink, R = T - sf;
    const int ngroups = R >= W ? (R - W) / LKV_GROUP : 0;
    const int nw = R - ngroups * LKV_GROUP;
    ingest_prep_kernel<<<1, 1, 0, s>>>(st, cell, mode, D, max_batch, max_blocks, req, T, ngroups);
    if (mode != LOOPKV_CELL_SHARE && ngroups > 0)
        ingest_quant_kernel<D, DT><<<dim3(ngroups, H), kQThreads, 0, s>>>(st, cell, mode, H, max_batch, max_blocks,
                                                                         req, (const DT *)k, (const DT *)v, sf);
    if (sf + nw > 0)
        ingest_tail_kernel<DT><<<64, 256, 0, s>>>(st, cell, H, D, max_batch, req, (const DT *)k, (const DT *)v, T,
                                                  sf, nw);
}

int launch_ingest(const DevState &st, int cell, int mode, int H, int D, int dtype, int max_batch, int max_blocks,
                  int req, const void *k, const void *v, int T, cudaStream_t s)
{
    if (D == 128) {
        if (dtype == LOOPKV_DTYPE_BF16)
            ingest_dispatch<128, __nv_bfloat16>(st, cell, mode, H, max_batch, max_blocks, req, k, v, T, s);
        else
            ingest_dispatch<128, float>(st, cell, mode, H, max_batch, max_blocks, req, k, v, T, s);
    } else {
        if (dtype == LOOPKV_DTYPE_BF16)
            ingest_dispatch<64, __nv_bfloat16>(st, cell, mode, H, max_batch, max_blocks, req, k, v, T, s);
        else
            ingest_dispatch<64, float>(st, cell, mode, H, max_batch, max_blocks, req, k, v, T, s);
    }
    return cuda_status(cudaGetLastError());
}

int launch_reset(const DevState &st, const uint8_t *cell_modes_dev, int n_cells, int max_batch, int max_blocks,
                 int req, cudaStream_t s)
{
    // D only matters for pool selection arithmetic that does not depend on it here.
    reset_kernel<<<(n_cells + 127) / 128, 128, 0, s>>>(st, cell_modes_dev, n_cells, max_batch, max_blocks, req, 128);
    return cuda_status(cudaGetLastError());
}

}  // namespace lkv
