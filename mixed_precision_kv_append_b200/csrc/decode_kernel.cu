// decode_kernel.cu -- fused, plan-driven decode attention over the LoopKV cache.
//
// One launch per cell (LoopKV paper, §3.4 "One launch per cell").  A thread-block
// cluster of C CTAs serves one (request, head) row; CTA r of the cluster owns the
// 32-token groups r, r+C, r+2C, ... of the row's history, and CTA C-1 also the
// unquantized tail.  Each CTA:
//   1. K pass: streams the key codes and per-channel key scale/zero of its groups
//      into shared memory with bulk asynchronous copies (a producer warp, an
//      mbarrier ring), and computes every score from the full 4-bit (or 2-bit) keys
//      with the key scale folded into q once per group (Appendix "History reader").
//      Scores stay in shared memory.
//   2. Exact row maximum: the CTAs exchange their maxima through distributed shared
//      memory across a cluster barrier, so every CTA knows the exact m -- the
//      "ideal" rule of §3.3 (a token is cold if its weight is below tau times the
//      largest in its row), not a streaming seed.  With the normalised-weight rule
//      a second exchange gives sum_t exp(s_t - m).
//   3. V pass: streams V scale/zero and the hi plane of every token; the producer
//      fetches a token's lo plane only if its weight passes the threshold (§3.3
//      "Read-time V precision").  Hot tokens decode to z + s(4h+l), cold ones to the
//      middle of their bucket z + s(4h+1.5), 2-bit cells to z + s*code; the per-token
//      scale and zero are folded into the weight and a running sum.
//   4. Merge: since all CTAs used the same m, their partial sums add directly; the
//      CTAs reduce them through distributed shared memory and write out = o / l.
//
// Code extraction: a field masked out of a packed word, read as an fp32 bit pattern
// x < 2^24, has the value x * 2^-149 exactly (subnormal or smallest-exponent normal
// numbers).  Multiplying it by a factor pre-scaled with 2^(149 - p) (p = the field's
// bit position) gives code * factor with one AND and one FMA per code and no int->
// float conversion; fp32 FMA on sm_100a keeps subnormal inputs (no flush to zero).
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "lkv_device.cuh"
#include "lkv_internal.h"

namespace lkv {
namespace {

constexpr int kConsumerWarps = 4;
constexpr int kThreads = (kConsumerWarps + 1) * 32;
constexpr int kVScaleExp = 40; // V accumulators hold code * w * s * 2^(p - 40)

template <int BITS, int D> struct Geo {
    static constexpr int KCODES = BITS == 4 ? 16 * D / 2 : 16 * D / 4;
    static constexpr int KMETA = 2 * D;
    static constexpr int VMETA = 16 * (D / 32) * 4;
    static constexpr int VPLANE = 16 * D / 4;
    static constexpr int HM = KCODES + KMETA + VMETA + VPLANE; // head main bytes
    static constexpr int LOB = BITS == 4 ? VPLANE : 0;          // head lo bytes
    static constexpr int KB = KCODES + KMETA;                   // K part of a block-head
    static constexpr int VB = VMETA + VPLANE;                   // V meta + hi part
    static constexpr int KSTAGE = 2 * KB;
    static constexpr int VSTAGE = 2 * VB + 2 * LOB;
    static constexpr int STAGE = ((KSTAGE > VSTAGE ? KSTAGE : VSTAGE) + 127) / 128 * 128;
    static constexpr int ROWK = KCODES / 16;  // key bytes per token
    static constexpr int WORDSK = ROWK / 4;
    static constexpr int ROWV = D / 4;        // value plane bytes per token
    static constexpr int NCG = D / 32;        // 32-channel value groups per token
    static constexpr int TPI = 32 / NCG;      // tokens per V iteration of a warp
};

// Slot of channel c in the per-word factor table, and the bit position its field is
// read from (fields above bit 23 are read from the word shifted right by 16).
template <int BITS> __device__ __forceinline__ void key_slot(int c, int &slot, int &pos)
{
    if (BITS == 4) {
        int w = c >> 3, r = c & 7;
        int j = r < 4 ? 2 * r : 2 * (r - 4) + 1; // nibble index in the word
        slot = 8 * w + j;
        pos = j < 6 ? 4 * j : (j == 6 ? 8 : 12);
    } else {
        int w = c >> 4, r = c & 15;
        int b = r & 3, i = r >> 2; // field at bit 8b + 2i
        slot = 16 * w + 4 * b + i;
        pos = b < 3 ? 8 * b + 2 * i : 8 + 2 * i;
    }
}

__device__ __forceinline__ float fbits(uint32_t x) { return __uint_as_float(x); }

__device__ __forceinline__ void ffma2(float2 &acc, float a, float b, float2 f)
{
    acc = __ffma2_rn(make_float2(a, b), f, acc);
}

// acc += sum over the 8 nibbles of w of nibble * A[slot]
__device__ __forceinline__ void key_word4(uint32_t w, const float *A, float2 &acc)
{
    const float4 a0 = reinterpret_cast<const float4 *>(A)[0];
    const float4 a1 = reinterpret_cast<const float4 *>(A)[1];
    const uint32_t h = w >> 16;
    ffma2(acc, fbits(w & 0xFu), fbits(w & 0xF0u), make_float2(a0.x, a0.y));
    ffma2(acc, fbits(w & 0xF00u), fbits(w & 0xF000u), make_float2(a0.z, a0.w));
    ffma2(acc, fbits(w & 0xF0000u), fbits(w & 0xF00000u), make_float2(a1.x, a1.y));
    ffma2(acc, fbits(h & 0xF00u), fbits(h & 0xF000u), make_float2(a1.z, a1.w));
}

// acc += sum over the 16 two-bit fields of w of field * A[slot]
__device__ __forceinline__ void key_word2(uint32_t w, const float *A, float2 &acc)
{
    const float4 a0 = reinterpret_cast<const float4 *>(A)[0];
    const float4 a1 = reinterpret_cast<const float4 *>(A)[1];
    const float4 a2 = reinterpret_cast<const float4 *>(A)[2];
    const float4 a3 = reinterpret_cast<const float4 *>(A)[3];
    const uint32_t h = w >> 16;
    ffma2(acc, fbits(w & 0x3u), fbits(w & 0xCu), make_float2(a0.x, a0.y));
    ffma2(acc, fbits(w & 0x30u), fbits(w & 0xC0u), make_float2(a0.z, a0.w));
    ffma2(acc, fbits(w & 0x300u), fbits(w & 0xC00u), make_float2(a1.x, a1.y));
    ffma2(acc, fbits(w & 0x3000u), fbits(w & 0xC000u), make_float2(a1.z, a1.w));
    ffma2(acc, fbits(w & 0x30000u), fbits(w & 0xC0000u), make_float2(a2.x, a2.y));
    ffma2(acc, fbits(w & 0x300000u), fbits(w & 0xC00000u), make_float2(a2.z, a2.w));
    ffma2(acc, fbits(h & 0x300u), fbits(h & 0xC00u), make_float2(a3.x, a3.y));
    ffma2(acc, fbits(h & 0x3000u), fbits(h & 0xC000u), make_float2(a3.z, a3.w));
}

// Value word pair (hi, lo) of 16 channels -> 4-bit codes 4h+l in two nibble words.
// Field of channel 4i+b sits at bit 8b+2i in both planes.  E holds the channels with
// even i (nibble at 8b+4m is channel 8m+b), O those with odd i (channel 8m+4+b).
// With lo = 0 the nibbles are 4h: the cold / 2-bit decode in the same scale domain.
__device__ __forceinline__ void value_word(uint32_t hi, uint32_t lo, float W, float2 (&acc)[2][4])
{
    const uint32_t E = ((hi << 2) & 0xCCCCCCCCu) | (lo & 0x33333333u);
    const uint32_t O = (hi & 0xCCCCCCCCu) | ((lo >> 2) & 0x33333333u);
    const uint32_t Eh = E >> 16, Oh = O >> 16;
    const float2 w2 = make_float2(W, W);
    ffma2(acc[0][0], fbits(E & 0xFu), fbits(E & 0xF0u), w2);
    ffma2(acc[0][1], fbits(E & 0xF00u), fbits(E & 0xF000u), w2);
    ffma2(acc[0][2], fbits(E & 0xF0000u), fbits(E & 0xF00000u), w2);
    ffma2(acc[0][3], fbits(Eh & 0xF00u), fbits(Eh & 0xF000u), w2);
    ffma2(acc[1][0], fbits(O & 0xFu), fbits(O & 0xF0u), w2);
    ffma2(acc[1][1], fbits(O & 0xF00u), fbits(O & 0xF000u), w2);
    ffma2(acc[1][2], fbits(O & 0xF0000u), fbits(O & 0xF00000u), w2);
    ffma2(acc[1][3], fbits(Oh & 0xF00u), fbits(Oh & 0xF000u), w2);
}

// Channel offset (within 16) and bit position of accumulator (e, n): e = 0 for E,
// 1 for O; n = nibble index 0..7.
__device__ __forceinline__ int value_channel(int e, int n) { return 8 * (n & 1) + (n >> 1) + 4 * e; }
__device__ __forceinline__ int value_pos(int n) { return n < 6 ? 4 * n : (n == 6 ? 8 : 12); }

struct Smem {
    uint8_t *ring;
    uint64_t *full;
    uint64_t *empty;
    float *scores; // [cap * 32] history scores, then [32] tail scores
    float *aw;     // [kConsumerWarps][D] key factors
    float *qs;     // [D] pre-scaled query (tail scoring)
    float *wmax;   // [kConsumerWarps]
    float *wsum;   // [kConsumerWarps]
    float *red;    // [kConsumerWarps][D + 1]
    float *po;     // [D + 1] CTA partial o and l, read by the other CTAs
};

template <int BITS, int D> __host__ __device__ constexpr int smem_bytes(int stages, int cap)
{
    using G = Geo<BITS, D>;
    return stages * G::STAGE + 2 * stages * 8 + (cap * 32 + 32) * 4 + kConsumerWarps * D * 4 + D * 4 +
           2 * kConsumerWarps * 4 + kConsumerWarps * (D + 1) * 4 + (D + 1) * 4 + 128;
}

template <int BITS, int D> __device__ Smem carve(uint8_t *base, int stages, int cap)
{
    using G = Geo<BITS, D>;
    Smem s;
    uint8_t *p = base;
    s.ring = p;
    p += stages * G::STAGE;
    s.full = reinterpret_cast<uint64_t *>(p);
    p += stages * 8;
    s.empty = reinterpret_cast<uint64_t *>(p);
    p += stages * 8;
    s.scores = reinterpret_cast<float *>(p);
    p += (cap * 32 + 32) * 4;
    s.aw = reinterpret_cast<float *>(p);
    p += kConsumerWarps * D * 4;
    s.qs = reinterpret_cast<float *>(p);
    p += D * 4;
    s.wmax = reinterpret_cast<float *>(p);
    p += kConsumerWarps * 4;
    s.wsum = reinterpret_cast<float *>(p);
    p += kConsumerWarps * 4;
    s.red = reinterpret_cast<float *>(p);
    p += kConsumerWarps * (D + 1) * 4;
    s.po = reinterpret_cast<float *>(p);
    return s;
}

// Maximum over all CTAs of the cluster of the per-warp values v[kConsumerWarps].
__device__ __forceinline__ float cluster_max(const float *v, uint32_t C, int lane)
{
    float m = -INFINITY;
    for (uint32_t k = lane; k < C * kConsumerWarps; k += 32)
        m = fmaxf(m, ld_dsmem_f32(v + (k % kConsumerWarps), k / kConsumerWarps));
    return warp_max(m);
}

// Sum over all CTAs in a fixed order (rank-major, then warp), identical in every warp.
__device__ __forceinline__ float cluster_sum_fixed(const float *v, uint32_t C)
{
    float s = 0.f;
    for (uint32_t r = 0; r < C; ++r)
        for (int w = 0; w < kConsumerWarps; ++w)
            s += ld_dsmem_f32(v + w, r);
    return s;
}

template <int BITS, int D, typename DT>
__global__ void __launch_bounds__(kThreads) decode_kernel(const DecodeArgs a, const int stages)
{
    using G = Geo<BITS, D>;
    extern __shared__ __align__(128) uint8_t smem_raw[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int row = blockIdx.y;
    const int b = row / a.H, h = row % a.H;
    const uint32_t crank = cluster_ctarank(), C = cluster_nctarank();
    Smem sm = carve<BITS, D>(smem_raw, stages, a.cap_groups);

    // Row lengths (history of the source cell, tail of this cell), validated.
    int hist = a.hist_len[b], tail = a.tail_len[b];
    bool bad = false;
    if (hist < 0 || hist > a.max_blocks * 16 || (hist & 31)) {
        bad = true;
        hist = 0;
    }
    if (tail < 0 || tail > 32) {
        bad = true;
        tail = 0;
    }
    const int ngroups = hist >> 5;
    int nmy = ngroups > (int)crank ? (ngroups - (int)crank + (int)C - 1) / (int)C : 0;
    if (nmy > a.cap_groups) {
        bad = true;
        nmy = a.cap_groups;
    }
    const bool tail_cta = (crank == C - 1) && tail > 0;
    if (bad && threadIdx.x == 0)
        atomicOr(a.status, LOOPKV_DEV_STATE);

    const bool all_hot = (BITS == 4) && !(a.tau > 0.f);
    const bool decide = (BITS == 4) && (a.tau > 0.f); // lo planes depend on the row max
    const int32_t *bt = a.block_table + (int64_t)b * a.max_blocks;
    const DT *tailk = reinterpret_cast<const DT *>(a.tail) + ((int64_t)b * 2 * a.H + h) * 32 * D;
    const DT *tailv = reinterpret_cast<const DT *>(a.tail) + ((int64_t)(b * 2 + 1) * a.H + h) * 32 * D;

    if (threadIdx.x == 0) {
        for (int i = 0; i < stages; ++i) {
            mbar_init(&sm.full[i], 1);
            mbar_init(&sm.empty[i], 1);
        }
        fence_mbar_init();
    }
    // pre-scaled query (log2(e)/sqrt(D) folded in) for the tail
    const DT *qrow = reinterpret_cast<const DT *>(a.q) + (int64_t)row * D;
    for (int c = threadIdx.x; c < D; c += kThreads)
        sm.qs[c] = to_f32(qrow[c]) * a.qscale;
    __syncthreads();

    float m2 = -INFINITY, thr2 = -INFINITY;

    if (warp == kConsumerWarps) {
        // ------------------------------------------------------------ producer
        auto block_id = [&](int idx) -> int64_t {
            int64_t id = bt[idx];
            if (id < 0 || id >= a.pool_blocks) {
                atomicOr(a.status, LOOPKV_DEV_STATE);
                id = 0;
            }
            return id;
        };
        auto wait_empty = [&](int i) {
            if (i >= stages)
                mbar_wait(&sm.empty[i % stages], ((i / stages) - 1) & 1, a.status);
        };
        for (int i = 0; i < nmy; ++i) { // K stages
            wait_empty(i);
            if (lane == 0) {
                const int g = (int)crank + i * (int)C;
                uint8_t *st = sm.ring + (i % stages) * G::STAGE;
                uint64_t *fb = &sm.full[i % stages];
                mbar_arrive_expect_tx(fb, 2 * G::KB);
                bulk_g2s(st, a.main + (block_id(2 * g) * a.H + h) * G::HM, G::KB, fb);
                bulk_g2s(st + G::KB, a.main + (block_id(2 * g + 1) * a.H + h) * G::HM, G::KB, fb);
            }
            __syncwarp();
        }
        cluster_arrive(); // barrier 1: the producer contributes no score

        auto issue_main = [&](int j) { // V meta + hi of group j, without arriving
            const int i = nmy + j;
            wait_empty(i);
            if (lane == 0) {
                const int g = (int)crank + j * (int)C;
                uint8_t *st = sm.ring + (i % stages) * G::STAGE;
                uint64_t *fb = &sm.full[i % stages];
                mbar_expect_tx(fb, 2 * G::VB);
                bulk_g2s(st, a.main + (block_id(2 * g) * a.H + h) * G::HM + G::KB, G::VB, fb);
                bulk_g2s(st + G::VB, a.main + (block_id(2 * g + 1) * a.H + h) * G::HM + G::KB, G::VB, fb);
            }
            __syncwarp();
        };
        auto issue_lo = [&](int j) { // lo planes of the hot tokens of group j, then arrive
            const int i = nmy + j;
            const int g = (int)crank + j * (int)C;
            uint8_t *st = sm.ring + (i % stages) * G::STAGE;
            uint64_t *fb = &sm.full[i % stages];
            uint32_t mask = 0;
            if (BITS == 4)
                mask = all_hot ? 0xFFFFFFFFu : __ballot_sync(0xFFFFFFFFu, sm.scores[j * 32 + lane] >= thr2);
            if (a.s_bitmap && lane == 0)
                a.s_bitmap[(int64_t)row * a.bitmap_words + g] = mask;
            if (BITS == 4 && mask == 0xFFFFFFFFu) {
                if (lane == 0) {
                    mbar_arrive_expect_tx(fb, 2 * G::LOB);
                    bulk_g2s(st + 2 * G::VB, a.lo + (block_id(2 * g) * a.H + h) * G::LOB, G::LOB, fb);
                    bulk_g2s(st + 2 * G::VB + G::LOB, a.lo + (block_id(2 * g + 1) * a.H + h) * G::LOB, G::LOB, fb);
                }
            } else {
                if (lane == 0)
                    mbar_arrive_expect_tx(fb, (uint32_t)__popc(mask) * G::ROWV);
                __syncwarp();
                if (BITS == 4 && ((mask >> lane) & 1u)) {
                    const int blk = lane >> 4, r = lane & 15;
                    bulk_g2s(st + 2 * G::VB + blk * G::LOB + r * G::ROWV,
                             a.lo + (block_id(2 * g + blk) * a.H + h) * G::LOB + r * G::ROWV, G::ROWV, fb);
                }
            }
            __syncwarp();
        };

        if (decide) {
            const int npre = nmy < stages ? nmy : stages;
            for (int j = 0; j < npre; ++j)
                issue_main(j);
            cluster_wait();
            m2 = cluster_max(sm.wmax, C, lane);
            float lt = 1.f;
            if (a.tau_mode == LOOPKV_TAU_ABS_PROB) {
                cluster_arrive();
                cluster_wait();
                lt = cluster_sum_fixed(sm.wsum, C);
            }
            thr2 = m2 + log2f(a.tau * lt);
            for (int j = 0; j < npre; ++j)
                issue_lo(j);
            for (int j = npre; j < nmy; ++j) {
                issue_main(j);
                issue_lo(j);
            }
        } else {
            for (int j = 0; j < nmy; ++j) {
                issue_main(j);
                issue_lo(j);
            }
            cluster_wait();
            if (a.tau_mode == LOOPKV_TAU_ABS_PROB) {
                cluster_arrive();
                cluster_wait();
            }
        }
        cluster_arrive(); // barrier 3: partial sums ready
        cluster_wait();
        cluster_arrive(); // barrier 4: remote reads done
        cluster_wait();
        return;
    }

    // ---------------------------------------------------------------- consumers
    float qreg[D / 32];
#pragma unroll
    for (int i = 0; i < D / 32; ++i)
        qreg[i] = sm.qs[lane + 32 * i];
    float *aw = sm.aw + warp * D;
    float mx = -INFINITY;

    for (int i = warp; i < nmy; i += kConsumerWarps) { // K pass
        const int slot = i % stages;
        mbar_wait(&sm.full[slot], (i / stages) & 1, a.status);
        const uint8_t *st = sm.ring + slot * G::STAGE;
        const __half *ksc = reinterpret_cast<const __half *>(st + G::KCODES);        // even block: scales
        const __half *kzp = reinterpret_cast<const __half *>(st + G::KB + G::KCODES); // odd block: zeros
        float av[D / 32];
        float zs = 0.f, amax = 0.f;
#pragma unroll
        for (int k = 0; k < D / 32; ++k) {
            const int c = lane + 32 * k;
            av[k] = qreg[k] * __half2float(ksc[c]);
            zs = fmaf(qreg[k], __half2float(kzp[c]), zs);
            amax = fmaxf(amax, fabsf(av[k]));
        }
        zs = warp_sum(zs);
        amax = warp_max(amax);
        const int E = amax > 0.f ? ilogbf(amax) : 0;
#pragma unroll
        for (int k = 0; k < D / 32; ++k) {
            int slot_c, pos;
            key_slot<BITS>(lane + 32 * k, slot_c, pos);
            aw[slot_c] = mul_pow2(av[k], 126 - E - pos);
        }
        __syncwarp();
        const uint32_t *kr = reinterpret_cast<const uint32_t *>(st + (lane >> 4) * G::KB + (lane & 15) * G::ROWK);
        float2 acc = make_float2(0.f, 0.f);
#pragma unroll
        for (int w4 = 0; w4 < G::WORDSK / 4; ++w4) {
            const uint4 cw = reinterpret_cast<const uint4 *>(kr)[w4];
            if (BITS == 4) {
                key_word4(cw.x, aw + 8 * (4 * w4 + 0), acc);
                key_word4(cw.y, aw + 8 * (4 * w4 + 1), acc);
                key_word4(cw.z, aw + 8 * (4 * w4 + 2), acc);
                key_word4(cw.w, aw + 8 * (4 * w4 + 3), acc);
            } else {
                key_word2(cw.x, aw + 16 * (4 * w4 + 0), acc);
                key_word2(cw.y, aw + 16 * (4 * w4 + 1), acc);
                key_word2(cw.z, aw + 16 * (4 * w4 + 2), acc);
                key_word2(cw.w, aw + 16 * (4 * w4 + 3), acc);
            }
        }
        const float s2 = mul_pow2(acc.x + acc.y, E + 23) + zs;
        sm.scores[i * 32 + lane] = s2;
        mx = fmaxf(mx, s2);
        __syncwarp();
        if (lane == 0)
            mbar_arrive(&sm.empty[slot]);
    }
    float *tsc = sm.scores + a.cap_groups * 32;
    if (tail_cta && warp == kConsumerWarps - 1 && lane < tail) { // tail keys, exact
        const DT *kt = tailk + (int64_t)lane * D;
        float s2 = 0.f;
        for (int c = 0; c < D; ++c)
            s2 = fmaf(sm.qs[c], to_f32(kt[c]), s2);
        tsc[lane] = s2;
        mx = fmaxf(mx, s2);
    }
    mx = warp_max(mx);
    if (lane == 0)
        sm.wmax[warp] = mx;
    cluster_arrive(); // barrier 1
    cluster_wait();
    m2 = cluster_max(sm.wmax, C, lane);

    float lt = 1.f;
    if (a.tau_mode == LOOPKV_TAU_ABS_PROB) {
        float ps = 0.f;
        for (int i = warp; i < nmy; i += kConsumerWarps)
            ps += exp2f(sm.scores[i * 32 + lane] - m2);
        if (tail_cta && warp == kConsumerWarps - 1 && lane < tail)
            ps += exp2f(tsc[lane] - m2);
        ps = warp_sum(ps);
        if (lane == 0)
            sm.wsum[warp] = ps;
        cluster_arrive(); // barrier 2
        cluster_wait();
        lt = cluster_sum_fixed(sm.wsum, C);
    }
    thr2 = decide ? m2 + log2f(a.tau * lt) : -INFINITY;

    // V pass: lane = (token slot ts, 32-channel group cg)
    const int cg = lane % G::NCG, ts = lane / G::NCG;
    float2 acc[2][2][4];
#pragma unroll
    for (int k = 0; k < 2; ++k)
#pragma unroll
        for (int e = 0; e < 2; ++e)
#pragma unroll
            for (int n = 0; n < 4; ++n)
                acc[k][e][n] = make_float2(0.f, 0.f);
    float zacc = 0.f, lsum = 0.f;
    const float vscale = 6.490371073168535e32f; // 2^(149 - kVScaleExp) = 2^109
    const int first_v = ((warp - nmy) % kConsumerWarps + kConsumerWarps) % kConsumerWarps;
    for (int j = first_v; j < nmy; j += kConsumerWarps) {
        const int i = nmy + j;
        const int slot = i % stages;
        mbar_wait(&sm.full[slot], (i / stages) & 1, a.status);
        const uint8_t *st = sm.ring + slot * G::STAGE;
#pragma unroll
        for (int u = 0; u < 32 / G::TPI; ++u) {
            const int t = u * G::TPI + ts;
            const float s2 = sm.scores[j * 32 + t];
            const float w = exp2f(s2 - m2);
            const bool hot = all_hot || (BITS == 4 && s2 >= thr2);
            const int blk = t >> 4, r = t & 15;
            const uint8_t *vb = st + blk * G::VB;
            const __half2 meta = *reinterpret_cast<const __half2 *>(vb + r * G::NCG * 4 + cg * 4);
            const float vs = __low2float(meta), vz = __high2float(meta);
            const uint2 hw = *reinterpret_cast<const uint2 *>(vb + G::VMETA + r * G::ROWV + cg * 8);
            uint2 lw = make_uint2(0u, 0u);
            float W;
            if (BITS == 4) {
                if (hot)
                    lw = *reinterpret_cast<const uint2 *>(st + 2 * G::VB + blk * G::LOB + r * G::ROWV + cg * 8);
                W = w * vs;
                zacc = fmaf(w, hot ? vz : fmaf(1.5f, vs, vz), zacc);
            } else {
                W = w * vs * 0.25f;
                zacc = fmaf(w, vz, zacc);
            }
            if (cg == 0)
                lsum += w;
            const float Wp = W * vscale;
            value_word(hw.x, lw.x, Wp, acc[0]);
            value_word(hw.y, lw.y, Wp, acc[1]);
        }
        __syncwarp();
        if (lane == 0)
            mbar_arrive(&sm.empty[slot]);
    }

    // Reduce over the token slots of the warp (lanes with the same cg).
#pragma unroll
    for (int off = G::NCG; off < 32; off <<= 1) {
#pragma unroll
        for (int k = 0; k < 2; ++k)
#pragma unroll
            for (int e = 0; e < 2; ++e)
#pragma unroll
                for (int n = 0; n < 4; ++n) {
                    acc[k][e][n].x += __shfl_xor_sync(0xFFFFFFFFu, acc[k][e][n].x, off);
                    acc[k][e][n].y += __shfl_xor_sync(0xFFFFFFFFu, acc[k][e][n].y, off);
                }
        zacc += __shfl_xor_sync(0xFFFFFFFFu, zacc, off);
    }
    lsum = warp_sum(lsum);
    float *red = sm.red + warp * (D + 1);
    if (lane < G::NCG) {
#pragma unroll
        for (int k = 0; k < 2; ++k)
#pragma unroll
            for (int e = 0; e < 2; ++e)
#pragma unroll
                for (int n = 0; n < 8; ++n) {
                    const float v = (n & 1) ? acc[k][e][n >> 1].y : acc[k][e][n >> 1].x;
                    const int ch = 32 * cg + 16 * k + value_channel(e, n);
                    red[ch] = mul_pow2(v, kVScaleExp - value_pos(n)) + zacc;
                }
    }
    if (lane == 0)
        red[D] = lsum;
    __syncwarp();
    if (tail_cta && warp == kConsumerWarps - 1) { // tail values, exact
        float tl = 0.f;
        for (int t = 0; t < tail; ++t) {
            const float w = exp2f(tsc[t] - m2);
            tl += w;
            const DT *vt = tailv + (int64_t)t * D;
#pragma unroll
            for (int k = 0; k < D / 32; ++k)
                red[lane + 32 * k] = fmaf(w, to_f32(vt[lane + 32 * k]), red[lane + 32 * k]);
        }
        __syncwarp();
        if (lane == 0)
            red[D] += tl;
    }
    named_sync(1, kConsumerWarps * 32);
    for (int c = threadIdx.x; c <= D; c += kConsumerWarps * 32) {
        float s = 0.f;
#pragma unroll
        for (int w = 0; w < kConsumerWarps; ++w)
            s += sm.red[w * (D + 1) + c];
        sm.po[c] = s;
    }
    cluster_arrive(); // barrier 3
    cluster_wait();
    // CTA `crank` reduces channels [crank*D/C, (crank+1)*D/C) over the cluster.
    const int per = D / (int)C;
    if ((int)threadIdx.x < per) {
        const int c = (int)crank * per + (int)threadIdx.x;
        float s = 0.f, l = 0.f;
        for (uint32_t r = 0; r < C; ++r) {
            s += ld_dsmem_f32(sm.po + c, r);
            l += ld_dsmem_f32(sm.po + D, r);
        }
        float o = 0.f;
        if (l > 0.f)
            o = s / l;
        else if (c == 0)
            atomicOr(a.status, LOOPKV_DEV_EMPTY_ROW);
        a.out[(int64_t)row * D + c] = o;
        if (c == 0) {
            if (a.row_max)
                a.row_max[row] = m2 * 0.6931471805599453f;
            if (a.row_sum)
                a.row_sum[row] = l;
        }
    }
    cluster_arrive(); // barrier 4
    cluster_wait();
}

template <int BITS, int D, typename DT>
int launch_t(const DecodeArgs &a, int B, const DecodeShape &shp, cudaStream_t s)
{
    auto kern = decode_kernel<BITS, D, DT>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, shp.smem);
    if (e != cudaSuccess)
        return LOOPKV_ERR_CUDA;
    if (shp.cluster > 8) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        if (e != cudaSuccess)
            return LOOPKV_ERR_CUDA;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(shp.cluster, B * a.H, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = shp.smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = shp.cluster;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, kern, a, shp.stages);
    return e == cudaSuccess ? LOOPKV_OK : LOOPKV_ERR_CUDA;
}

}  // namespace

DecodeShape decode_shape(int bits, int D, int rows, int max_blocks)
{
    DecodeShape shp;
    shp.threads = kThreads;
    shp.stages = 8;
    const int max_groups = max_blocks / 2;
    // Cluster size: enough CTAs to cover the GPU several times, at most 8 (portable).
    int C = 1;
    while (C < 8 && rows * C < 4 * 148)
        C *= 2;
    while (C > 1 && (max_groups + C - 1) / C < 1)
        C /= 2;
    shp.cluster = C;
    const int cap = (max_groups + C - 1) / C;
    if (bits == 4)
        shp.smem = D == 128 ? smem_bytes<4, 128>(shp.stages, cap) : smem_bytes<4, 64>(shp.stages, cap);
    else
        shp.smem = D == 128 ? smem_bytes<2, 128>(shp.stages, cap) : smem_bytes<2, 64>(shp.stages, cap);
    return shp;
}

int launch_decode(const DecodeArgs &a, int bits, int D, int dtype, int B, const DecodeShape &shp, cudaStream_t s)
{
    const bool bf = dtype == LOOPKV_DTYPE_BF16;
    if (bits == 4) {
        if (D == 128)
            return bf ? launch_t<4, 128, __nv_bfloat16>(a, B, shp, s) : launch_t<4, 128, float>(a, B, shp, s);
        return bf ? launch_t<4, 64, __nv_bfloat16>(a, B, shp, s) : launch_t<4, 64, float>(a, B, shp, s);
    }
    if (D == 128)
        return bf ? launch_t<2, 128, __nv_bfloat16>(a, B, shp, s) : launch_t<2, 128, float>(a, B, shp, s);
    return bf ? launch_t<2, 64, __nv_bfloat16>(a, B, shp, s) : launch_t<2, 64, float>(a, B, shp, s);
}

}  // namespace lkv
