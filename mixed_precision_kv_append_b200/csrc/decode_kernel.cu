// decode_kernel.cu -- fused, plan-driven decode attention over the LoopKV cache.
//
// One launch per cell (LoopKV paper, §3.4 "One launch per cell").  The grid is a set
// of persistent thread-block clusters of C CTAs; cluster c serves the (request, head)
// rows c, c + NC, c + 2NC, ... one after another.  Inside a row, CTA k of the cluster
// owns the 32-token groups k, k+C, k+2C, ... of the history, and CTA C-1 also the
// unquantized tail.  For each row a CTA:
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
// Rows are software-pipelined: while the cluster barrier that publishes row r's
// maxima completes, the CTA already streams and scores the keys of row r+1, so the
// memory pipe never drains at a row boundary.  One cluster barrier per row carries
// both the per-warp maxima (with their partial exponential sums, for the normalised
// rule) of row r and the partial outputs of row r-1.
//
// Keys: the dot product of a 32-token group is computed exactly in integers.  The
// group's per-channel factor q_c * s_c (key scale folded into the query once per group,
// as the paper's reader does) is rounded to a 22-bit fixed-point integer and split into
// three signed 8-bit digits; the 4-bit (or 2-bit) codes are unpacked four at a time into
// bytes with one AND, and dp4a accumulates code * digit in int32 with no rounding.
// Values: a field masked out of a packed word, read as an fp32 bit pattern x < 2^24, has
// the value x * 2^-149 exactly (subnormal or smallest-exponent normal numbers);
// multiplied by a weight pre-scaled with 2^(149 - p) (p = the field's bit position) it
// gives code * weight with one AND and half a packed FMA per code; fp32 FMA on sm_100a
// keeps subnormal inputs (no flush to zero).
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "lkv_device.cuh"
#include "lkv_internal.h"

#include <algorithm>
#include <cstdlib>

namespace lkv {
namespace {

constexpr int kWarps = 4; // every warp both issues the copies of its stages and computes on them
constexpr int kThreads = kWarps * 32;
constexpr int kMinCtasPerSm = 4; // default register bound: 4 CTAs of 128 threads per SM (<= 128 registers)
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

__device__ __forceinline__ float fbits(uint32_t x) { return __uint_as_float(x); }

__device__ __forceinline__ void ffma2(float2 &acc, float a, float b, float2 f)
{
    acc = __ffma2_rn(make_float2(a, b), f, acc);
}

// acc += sum of the four unsigned bytes of `u` times the four signed bytes of `d`
__device__ __forceinline__ void dp4a_us(int &acc, uint32_t u, int d)
{
    asm("dp4a.u32.s32 %0, %1, %2, %0;" : "+r"(acc) : "r"(u), "r"(d));
}

// Quad q of a key row = channels 4q..4q+3 as four bytes.  4-bit word w holds quads 2w
// (low nibbles) and 2w+1 (high nibbles); 2-bit word w holds quads 4w+i at bit 2i.
template <int BITS>
__device__ __forceinline__ void key_word(uint32_t w, const int4 *dig, int (&acc)[2][3])
{
    if (BITS == 4) {
        const uint32_t u0 = w & 0x0F0F0F0Fu, u1 = (w >> 4) & 0x0F0F0F0Fu;
        const int4 d0 = dig[0], d1 = dig[1];
        dp4a_us(acc[0][0], u0, d0.x);
        dp4a_us(acc[0][1], u0, d0.y);
        dp4a_us(acc[0][2], u0, d0.z);
        dp4a_us(acc[1][0], u1, d1.x);
        dp4a_us(acc[1][1], u1, d1.y);
        dp4a_us(acc[1][2], u1, d1.z);
    } else {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint32_t u = (w >> (2 * i)) & 0x03030303u;
            const int4 d = dig[i];
            dp4a_us(acc[i & 1][0], u, d.x);
            dp4a_us(acc[i & 1][1], u, d.y);
            dp4a_us(acc[i & 1][2], u, d.z);
        }
    }
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
    uint8_t *ring;     // [kWarps][spw][STAGE] stage slots, a private slice per warp
    uint64_t *full;    // [kWarps][spw] completion barriers of the slots
    float *scores;     // [2][kWarps][capw * 32] scores of a warp's groups, by row parity
    float *tscores;    // [2][32] tail scores, by row parity
    uint8_t *scr;      // [kWarps][SCR] per-warp scratch, used in turn as: key-factor digits
                       // [D/4][4] during a K stage, value weights [32][D/32] during a V
                       // stage, the warp's partial o and l [D + 1] at the end of a V pass
    float *stat;       // [3][kWarps][2] per-warp (max, sum exp(s - max)), by row index mod 3
    float *part;       // [2][D + 1] CTA partial o and l of a row, by row parity
    int32_t *ids;      // [3][kWarps][2 * capw] block ids of a warp's groups, by row index mod 3
    int32_t *irow;     // [3][kWarps][8] issuer state of a row, by row index mod 3
};

// Issuer state of one row (int fields of Smem::irow).
enum { IR_ROW = 0, IR_H, IR_OWN, IR_VFIRST, IR_VISSUED, IR_THR, IR_N = 8 };

// Byte offsets of the shared-memory regions; every region starts on a 16-byte boundary
// (the key factors and the stage data are read with 16-byte vector loads).
struct SmemLayout {
    int full, scores, tscores, scr, stat, part, ids, irow, total;
};

__host__ __device__ constexpr int align16(int x) { return (x + 15) & ~15; }

// Bytes of a warp's scratch: the largest of its three uses.
template <int D> __host__ __device__ constexpr int scratch_bytes()
{
    return align16((D * 4 > (D + 1) * 4 ? D * 4 : (D + 1) * 4) > 32 * (D / 32) * 4
                       ? (D * 4 > (D + 1) * 4 ? D * 4 : (D + 1) * 4)
                       : 32 * (D / 32) * 4);
}

// nbuf: score buffers (2 when a cluster reads more than one row, so that the next row's
// keys can be scored while the current row's values are read).
template <int BITS, int D> __host__ __device__ constexpr SmemLayout smem_layout(int spw, int capw, int nbuf)
{
    SmemLayout L{};
    int o = kWarps * spw * Geo<BITS, D>::STAGE; // ring, 128-byte aligned slots
    L.full = o;
    o = align16(o + kWarps * spw * 8);
    L.scores = o;
    o = align16(o + nbuf * kWarps * capw * 32 * 4);
    L.tscores = o;
    o = align16(o + 2 * 32 * 4);
    L.scr = o;
    o = align16(o + kWarps * scratch_bytes<D>());
    L.stat = o;
    o = align16(o + 3 * kWarps * 2 * 4);
    L.part = o;
    o = align16(o + 2 * (D + 1) * 4);
    L.ids = o;
    o = align16(o + 3 * kWarps * 2 * capw * 4);
    L.irow = o;
    o = align16(o + 3 * kWarps * IR_N * 4);
    L.total = o;
    return L;
}

template <int BITS, int D> __host__ __device__ constexpr int smem_bytes(int spw, int capw, int nbuf)
{
    return smem_layout<BITS, D>(spw, capw, nbuf).total;
}

template <int BITS, int D> __device__ Smem carve(uint8_t *base, int spw, int capw, int nbuf)
{
    const SmemLayout L = smem_layout<BITS, D>(spw, capw, nbuf);
    Smem s;
    s.ring = base;
    s.full = reinterpret_cast<uint64_t *>(base + L.full);
    s.scores = reinterpret_cast<float *>(base + L.scores);
    s.tscores = reinterpret_cast<float *>(base + L.tscores);
    s.scr = base + L.scr;
    s.stat = reinterpret_cast<float *>(base + L.stat);
    s.part = reinterpret_cast<float *>(base + L.part);
    s.ids = reinterpret_cast<int32_t *>(base + L.ids);
    s.irow = reinterpret_cast<int32_t *>(base + L.irow);
    return s;
}

// Host check of a layout: every region 16-byte aligned, in order, inside the allocation.
template <int BITS, int D> bool layout_ok(int spw, int capw, int nbuf)
{
    const SmemLayout L = smem_layout<BITS, D>(spw, capw, nbuf);
    const int offs[] = {L.full, L.scores, L.tscores, L.scr, L.stat, L.part, L.ids, L.irow};
    int prev = kWarps * spw * Geo<BITS, D>::STAGE;
    for (int o : offs) {
        if (o % 16 || o < prev)
            return false;
        prev = o;
    }
    return (Geo<BITS, D>::STAGE % 128) == 0 && L.total >= prev && (spw & (spw - 1)) == 0 &&
           scratch_bytes<D>() >= D * 4 && scratch_bytes<D>() >= (D + 1) * 4 && scratch_bytes<D>() >= 32 * (D / 32) * 4;
}

// One (request, head) row as seen by one CTA of its cluster.
struct RowCtx {
    int row, b, h;
    int tail;       // validated tail length
    int nmy;        // 32-token groups of the history owned by this CTA
    bool tail_cta;  // this CTA also reads the tail
};

__device__ __forceinline__ RowCtx row_ctx(const DecodeArgs &a, int row, uint32_t crank, uint32_t C, bool report)
{
    RowCtx r;
    r.row = row;
    r.b = row / a.H;
    r.h = row - r.b * a.H;
    int hist = a.hist_len[r.b], tail = a.tail_len[r.b];
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
    if (bad && report)
        atomicOr(a.status, LOOPKV_DEV_STATE);
    r.tail = tail;
    r.nmy = nmy;
    r.tail_cta = (crank == C - 1) && tail > 0;
    return r;
}

// Groups of a row owned by warp w of the CTA: local groups w, w + kWarps, ...
__device__ __forceinline__ int owned(int nmy, int w) { return nmy > w ? (nmy - w + kWarps - 1) / kWarps : 0; }

// Row max m (log2 units) and, for the normalised rule, l = sum_t 2^(s_t - m), from the
// per-warp pairs of every CTA of the cluster (fixed order: every caller gets the same).
__device__ __forceinline__ void cluster_row_stats(const float *stat, uint32_t C, float &m, float &l)
{
    m = -INFINITY;
    for (uint32_t r = 0; r < C; ++r)
        for (int w = 0; w < kWarps; ++w)
            m = fmaxf(m, ld_dsmem_f32(stat + 2 * w, r));
    l = 0.f;
    if (m == -INFINITY)
        return;
    for (uint32_t r = 0; r < C; ++r)
        for (int w = 0; w < kWarps; ++w) {
            const float mw = ld_dsmem_f32(stat + 2 * w, r);
            if (mw != -INFINITY)
                l += ld_dsmem_f32(stat + 2 * w + 1, r) * exp2f(mw - m);
        }
}

__device__ __forceinline__ float row_threshold(const DecodeArgs &a, float m, float l, bool decide)
{
    if (!decide)
        return -INFINITY;
    return a.tau_mode == LOOPKV_TAU_ABS_PROB ? m + log2f(a.tau * l) : m + log2f(a.tau);
}

// Segment sig of a warp's stage sequence K(0), K(1), V(0), K(2), V(1), ..., V(n-1):
// returns whether it is a V segment and its row index.
__device__ __forceinline__ void segment(int sig, int nrows, bool &is_v, int &ri)
{
    if (sig == 0) {
        is_v = false;
        ri = 0;
    } else if (sig == 2 * nrows - 1) {
        is_v = true;
        ri = nrows - 1;
    } else {
        const int i = (sig + 1) >> 1;
        is_v = !(sig & 1);
        ri = (sig & 1) ? i : i - 1;
    }
}

// MINCTA: CTAs per SM the registers are budgeted for (4: <= 128 registers, 5: <= 96).
template <int BITS, int D, typename DT, int MINCTA>
__global__ void __launch_bounds__(kThreads, MINCTA) decode_kernel(const DecodeArgs a, const int spw_log2, const int nbuf)
{
    using G = Geo<BITS, D>;
    extern __shared__ __align__(128) uint8_t smem_raw[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int spw = 1 << spw_log2, smask = spw - 1;
    const uint32_t crank = cluster_ctarank(), C = cluster_nctarank();
    const int cid = blockIdx.x / (int)C, ncl = gridDim.x / (int)C;
    const int nrows = cid < a.rows ? (a.rows - 1 - cid) / ncl + 1 : 0; // rows cid, cid + ncl, ...
    const int capw = (a.cap_groups + kWarps - 1) / kWarps;
    Smem sm = carve<BITS, D>(smem_raw, spw, capw, nbuf);
    const bool all_hot = (BITS == 4) && !(a.tau > 0.f);
    const bool decide = (BITS == 4) && (a.tau > 0.f); // lo planes depend on the row max

    if (lane == 0)
        for (int i = 0; i < spw; ++i)
            mbar_init(&sm.full[warp * spw + i], 1);
    fence_mbar_init();
    __syncwarp();

    uint8_t *ring = sm.ring + warp * spw * G::STAGE;
    uint64_t *full = sm.full + warp * spw;
    auto scores_of = [&](int ri) { return sm.scores + (((nbuf == 2) ? (ri & 1) : 0) * kWarps + warp) * capw * 32; };
    auto ids_of = [&](int ri) { return sm.ids + ((ri % 3) * kWarps + warp) * 2 * capw; };
    auto irow_of = [&](int ri) { return sm.irow + ((ri % 3) * kWarps + warp) * IR_N; };

    // ---------------------------------------------------------------- issuing
    // A warp issues the bulk copies of its own stages, `spw` stages ahead of its compute.
    int iss_sig = 0, iss_k = 0, iss_n = 0;
    int seg_len = 0, seg_ri = 0;   // current segment: own stages and row index
    bool seg_v = false;
    int released = 0;              // rows whose threshold the issuer has received

    auto setup_row = [&](int ri) {
        const RowCtx rc = row_ctx(a, cid + ri * ncl, crank, C, false);
        const int n = owned(rc.nmy, warp);
        int32_t *st = irow_of(ri);
        const int32_t *bt = a.block_table + (int64_t)rc.b * a.max_blocks;
        int32_t *ids = ids_of(ri);
        for (int k = lane; k < 2 * n; k += 32) {
            const int g = (int)crank + (warp + (k >> 1) * kWarps) * (int)C;
            int id = bt[2 * g + (k & 1)];
            if (id < 0 || id >= a.pool_blocks) {
                atomicOr(a.status, LOOPKV_DEV_STATE);
                id = 0;
            }
            ids[k] = id;
        }
        if (lane == 0) {
            st[IR_ROW] = rc.row;
            st[IR_H] = rc.h;
            st[IR_OWN] = n;
            st[IR_VFIRST] = 0;
            st[IR_VISSUED] = 0;
            st[IR_THR] = __float_as_int(NAN);
        }
        __syncwarp();
    };
    auto load_segment = [&]() {
        segment(iss_sig, nrows, seg_v, seg_ri);
        seg_len = irow_of(seg_ri)[IR_OWN];
    };
    // lo planes (4-bit sources) of the hot tokens of V stage k of row ri, then arrive
    auto issue_lo = [&](int ri, int k, int n, float thr2) {
        const int32_t *st_row = irow_of(ri);
        const int h = st_row[IR_H];
        const int32_t *ids = ids_of(ri);
        uint8_t *st = ring + (n & smask) * G::STAGE;
        uint64_t *fb = &full[n & smask];
        uint32_t mask = 0;
        if (BITS == 4)
            mask = all_hot ? 0xFFFFFFFFu : __ballot_sync(0xFFFFFFFFu, scores_of(ri)[k * 32 + lane] >= thr2);
        if (a.s_bitmap && lane == 0) {
            const int g = (int)crank + (warp + k * kWarps) * (int)C;
            a.s_bitmap[(int64_t)st_row[IR_ROW] * a.bitmap_words + g] = mask;
        }
        const int64_t b0 = ids[2 * k], b1 = ids[2 * k + 1];
        const bool full_lo = BITS == 4 && mask == 0xFFFFFFFFu;
        if (lane == 0) {
            const uint32_t lo_bytes = full_lo ? 2 * G::LOB : (uint32_t)__popc(mask) * G::ROWV;
            mbar_arrive_expect_tx(fb, lo_bytes);
            if (full_lo) {
                bulk_g2s(st + 2 * G::VB, a.lo + (b0 * a.H + h) * G::LOB, G::LOB, fb);
                bulk_g2s(st + 2 * G::VB + G::LOB, a.lo + (b1 * a.H + h) * G::LOB, G::LOB, fb);
            }
        }
        __syncwarp();
        if (BITS == 4 && !full_lo && ((mask >> lane) & 1u)) {
            const int blk = lane >> 4, r = lane & 15;
            const int64_t bb = blk ? b1 : b0;
            bulk_g2s(st + 2 * G::VB + blk * G::LOB + r * G::ROWV, a.lo + (bb * a.H + h) * G::LOB + r * G::ROWV,
                     G::ROWV, fb);
        }
        __syncwarp();
    };
    auto issue_stage = [&](int n) {
        const int k = iss_k, ri = seg_ri;
        int32_t *st_row = irow_of(ri);
        const int h = st_row[IR_H];
        const int32_t *ids = ids_of(ri);
        uint8_t *st = ring + (n & smask) * G::STAGE;
        uint64_t *fb = &full[n & smask];
        const int64_t b0 = ids[2 * k], b1 = ids[2 * k + 1];
        if (!seg_v) {
            if (lane == 0) {
                mbar_arrive_expect_tx(fb, 2 * G::KB);
                bulk_g2s(st, a.main + (b0 * a.H + h) * G::HM, G::KB, fb);
                bulk_g2s(st + G::KB, a.main + (b1 * a.H + h) * G::HM, G::KB, fb);
            }
            __syncwarp();
            return;
        }
        if (lane == 0) {
            if (k == 0)
                st_row[IR_VFIRST] = n;
            st_row[IR_VISSUED] = k + 1;
            mbar_expect_tx(fb, 2 * G::VB);
            bulk_g2s(st, a.main + (b0 * a.H + h) * G::HM + G::KB, G::VB, fb);
            bulk_g2s(st + G::VB, a.main + (b1 * a.H + h) * G::HM + G::KB, G::VB, fb);
        }
        __syncwarp();
        const float thr2 = __int_as_float(st_row[IR_THR]);
        if (!decide || !isnan(thr2)) // the lo part needs the row threshold when tau > 0
            issue_lo(ri, k, n, thr2);
    };
    // Issue every stage numbered below `limit` that the sequence allows.  The issuer
    // state of a row lives in slot (row mod 3), so row r is set up only after row r - 3
    // has been released (all of its lo copies issued).
    auto pump = [&](int limit) {
        while (iss_n < limit && iss_sig < 2 * nrows) {
            if (iss_k < seg_len) {
                issue_stage(iss_n);
                ++iss_k;
                ++iss_n;
                continue;
            }
            const int nsig = iss_sig + 1;
            if (nsig < 2 * nrows) {
                bool nv;
                int nri;
                segment(nsig, nrows, nv, nri);
                if (!nv) {
                    if (nri - 3 >= released)
                        break;
                    setup_row(nri);
                }
            }
            iss_sig = nsig;
            iss_k = 0;
            if (iss_sig < 2 * nrows)
                load_segment();
        }
    };
    // the threshold of row ri is known: finish the V stages issued without their lo part
    auto release_row = [&](int ri, float thr2) {
        int32_t *st_row = irow_of(ri);
        const int vfirst = st_row[IR_VFIRST], vissued = st_row[IR_VISSUED];
        __syncwarp();
        if (lane == 0)
            st_row[IR_THR] = __float_as_int(thr2);
        __syncwarp();
        if (decide)
            for (int k = 0; k < vissued; ++k)
                issue_lo(ri, k, vfirst + k, thr2);
        released = ri + 1;
    };

    // ---------------------------------------------------------------- compute
    constexpr int SCR = scratch_bytes<D>();
    uint8_t *scr = sm.scr + warp * SCR;
    uint8_t *awb = scr;                                    // K stage: digit table, 16 bytes per quad
    const int4 *aw4 = reinterpret_cast<const int4 *>(scr);
    float4 *wv4 = reinterpret_cast<float4 *>(scr);         // V stage: weights per token and group
    const float *wvf = reinterpret_cast<const float *>(scr);
    // a lane owns the channel pairs (2*lane + 64j, 2*lane + 1 + 64j), j < D/64
    const float vscale = 6.490371073168535e32f; // 2^(149 - kVScaleExp) = 2^109
    int prc_n = 0;
    bool timed_out = false; // after one bounded wait gives up, later waits are skipped
    auto wait_stage = [&](int n) {
        if (!timed_out)
            timed_out = !mbar_wait(&full[n & smask], (n >> spw_log2) & 1, a.status);
    };

    // K pass of the warp's groups of row ri; per-warp (max, sum) into stat.
    auto consume_k = [&](int ri) {
        const RowCtx rc = row_ctx(a, cid + ri * ncl, crank, C, warp == 0 && lane == 0);
        float *sc = scores_of(ri);
        const DT *qrow = reinterpret_cast<const DT *>(a.q) + (int64_t)rc.row * D;
        float qreg[D / 32];
#pragma unroll
        for (int k = 0; k < D / 32; ++k)
            qreg[k] = to_f32(qrow[2 * lane + 64 * (k >> 1) + (k & 1)]) * a.qscale;
        float mx = -INFINITY;
        const int nown = owned(rc.nmy, warp);
        for (int k = 0; k < nown; ++k) {
            const int n = prc_n++;
            if (iss_n < n + spw)
                pump(n + spw);
            wait_stage(n);
            const uint8_t *st = ring + (n & smask) * G::STAGE;
            const __half2 *ksc = reinterpret_cast<const __half2 *>(st + G::KCODES);        // even: scales
            const __half2 *kzp = reinterpret_cast<const __half2 *>(st + G::KB + G::KCODES); // odd: zeros
            float av[D / 32];
            float zs = 0.f, amax = 0.f;
#pragma unroll
            for (int j = 0; j < D / 64; ++j) {
                const float2 sv = __half22float2(ksc[lane + 32 * j]);
                const float2 zv = __half22float2(kzp[lane + 32 * j]);
                av[2 * j] = qreg[2 * j] * sv.x;
                av[2 * j + 1] = qreg[2 * j + 1] * sv.y;
                zs = fmaf(qreg[2 * j], zv.x, zs);
                zs = fmaf(qreg[2 * j + 1], zv.y, zs);
                amax = fmaxf(amax, fmaxf(fabsf(av[2 * j]), fabsf(av[2 * j + 1])));
            }
            zs = warp_sum(zs);
            amax = warp_max(amax);
            // Fixed point: I_c = round(a_c * 2^F) with F = 21 - E (E = exponent of max |a|),
            // so |I_c| <= 2^22; balanced base-256 digits d0 + 256 d1 + 65536 d2, |d2| <= 65.
            const uint32_t abits = __float_as_uint(amax);
            const int E = abits >= 0x00800000u ? (int)(abits >> 23) - 127 : -126;
            const int F = 21 - E;
            const bool fast = F >= -126 && F <= 127 && E - 21 >= -126;
            const float fs = fast ? __int_as_float((F + 127) << 23) : 0.f;
#pragma unroll
            for (int c4 = 0; c4 < D / 32; ++c4) {
                const int c = 2 * lane + 64 * (c4 >> 1) + (c4 & 1);
                const float x = fast ? av[c4] * fs : mul_pow2(av[c4], F);
                const int I = __float2int_rn(x);
                const int d0 = (I << 24) >> 24;
                const int I1 = (I - d0) >> 8;
                const int d1 = (I1 << 24) >> 24;
                const int d2 = (I1 - d1) >> 8;
                uint8_t *q = awb + (c >> 2) * 16 + (c & 3);
                q[0] = (uint8_t)d0;
                q[4] = (uint8_t)d1;
                q[8] = (uint8_t)d2;
            }
            __syncwarp();
            const uint32_t *kr =
                reinterpret_cast<const uint32_t *>(st + (lane >> 4) * G::KB + (lane & 15) * G::ROWK);
            int acc[2][3] = {{0, 0, 0}, {0, 0, 0}};
            constexpr int QPW = BITS == 4 ? 2 : 4; // quads per code word
#pragma unroll
            for (int w4 = 0; w4 < G::WORDSK / 4; ++w4) {
                const uint4 cw = reinterpret_cast<const uint4 *>(kr)[w4];
                key_word<BITS>(cw.x, aw4 + QPW * (4 * w4 + 0), acc);
                key_word<BITS>(cw.y, aw4 + QPW * (4 * w4 + 1), acc);
                key_word<BITS>(cw.z, aw4 + QPW * (4 * w4 + 2), acc);
                key_word<BITS>(cw.w, aw4 + QPW * (4 * w4 + 3), acc);
            }
            const float dot = fmaf((float)(acc[0][2] + acc[1][2]), 65536.f,
                                   fmaf((float)(acc[0][1] + acc[1][1]), 256.f, (float)(acc[0][0] + acc[1][0])));
            const float s2 = (fast ? dot * __int_as_float((127 - F) << 23) : mul_pow2(dot, -F)) + zs;
            sc[k * 32 + lane] = s2;
            mx = fmaxf(mx, s2);
            __syncwarp();
        }
        float *tsc = sm.tscores + (ri & 1) * 32;
        if (rc.tail_cta && warp == kWarps - 1) { // tail keys, exact; lane = tail token
            const DT *kt = reinterpret_cast<const DT *>(a.tail) + ((int64_t)rc.b * 2 * a.H + rc.h) * 32 * D;
            float s2 = 0.f;
#pragma unroll
            for (int c4 = 0; c4 < D / 32; ++c4)
                for (int l = 0; l < 32; ++l) {
                    const float qc = __shfl_sync(0xFFFFFFFFu, qreg[c4], l);
                    const int c = 2 * l + 64 * (c4 >> 1) + (c4 & 1);
                    if (lane < rc.tail)
                        s2 = fmaf(qc, to_f32(kt[(int64_t)lane * D + c]), s2);
                }
            if (lane < rc.tail) {
                tsc[lane] = s2;
                mx = fmaxf(mx, s2);
            }
        }
        mx = warp_max(mx);
        float ls = 0.f;
        if (a.tau_mode == LOOPKV_TAU_ABS_PROB && mx != -INFINITY) {
            for (int k = 0; k < nown; ++k)
                ls += exp2f(sc[k * 32 + lane] - mx);
            if (rc.tail_cta && warp == kWarps - 1 && lane < rc.tail)
                ls += exp2f(tsc[lane] - mx);
            ls = warp_sum(ls);
        }
        if (lane == 0) {
            float *stw = sm.stat + (ri % 3) * kWarps * 2;
            stw[2 * warp] = mx;
            stw[2 * warp + 1] = ls;
        }
    };

    // V pass of the warp's groups of row ri, then the CTA partial (o, l) into part.
    auto consume_v = [&](int ri, float m2, float thr2) {
        const RowCtx rc = row_ctx(a, cid + ri * ncl, crank, C, false);
        const float *sc = scores_of(ri);
        const int cg = lane % G::NCG, ts = lane / G::NCG;
        float2 acc[2][2][4];
#pragma unroll
        for (int k = 0; k < 2; ++k)
#pragma unroll
            for (int e = 0; e < 2; ++e)
#pragma unroll
                for (int n = 0; n < 4; ++n)
                    acc[k][e][n] = make_float2(0.f, 0.f);
        float zl[G::NCG];
#pragma unroll
        for (int j = 0; j < G::NCG; ++j)
            zl[j] = 0.f;
        float lsum = 0.f;
        const int nown = owned(rc.nmy, warp);
        for (int k = 0; k < nown; ++k) {
            const int n = prc_n++;
            if (iss_n < n + spw)
                pump(n + spw);
            const float s2l = sc[k * 32 + lane];
            const float wl = exp2f(s2l - m2);
            const bool hotl = all_hot || (BITS == 4 && s2l >= thr2);
            const uint32_t hotmask = __ballot_sync(0xFFFFFFFFu, hotl);
            lsum += wl;
            wait_stage(n);
            const uint8_t *st = ring + (n & smask) * G::STAGE;
            {   // token `lane`: fold its value scales and zeros into the weight and a running sum
                const uint8_t *mrow = st + (lane >> 4) * G::VB + (lane & 15) * G::NCG * 4;
                float wsc[4];
#pragma unroll
                for (int j = 0; j < G::NCG; ++j) {
                    const float2 m = __half22float2(reinterpret_cast<const __half2 *>(mrow)[j]); // (scale, zero)
                    if (BITS == 4) {
                        zl[j] = fmaf(wl, hotl ? m.y : fmaf(1.5f, m.x, m.y), zl[j]);
                        wsc[j] = wl * m.x * vscale;
                    } else {
                        zl[j] = fmaf(wl, m.y, zl[j]);
                        wsc[j] = wl * m.x * (0.25f * vscale);
                    }
                }
                if (G::NCG == 4)
                    wv4[lane] = make_float4(wsc[0], wsc[1], wsc[2], wsc[3]);
                else
                    reinterpret_cast<float2 *>(wv4)[lane] = make_float2(wsc[0], wsc[1]);
            }
            __syncwarp();
#pragma unroll
            for (int u = 0; u < 32 / G::TPI; ++u) {
                const int t = u * G::TPI + ts;
                const float Wp = wvf[t * G::NCG + cg];
                const bool hot = (hotmask >> t) & 1u;
                const int blk = t >> 4, r = t & 15;
                const uint2 hw =
                    *reinterpret_cast<const uint2 *>(st + blk * G::VB + G::VMETA + r * G::ROWV + cg * 8);
                uint2 lw = make_uint2(0u, 0u);
                if (BITS == 4 && hot)
                    lw = *reinterpret_cast<const uint2 *>(st + 2 * G::VB + blk * G::LOB + r * G::ROWV + cg * 8);
                value_word(hw.x, lw.x, Wp, acc[0]);
                value_word(hw.y, lw.y, Wp, acc[1]);
            }
            __syncwarp();
        }
        // reduce over the token slots of the warp (lanes with the same cg)
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
        }
        float zacc = 0.f;
#pragma unroll
        for (int j = 0; j < G::NCG; ++j) {
            const float z = warp_sum(zl[j]);
            if (cg == j)
                zacc = z;
        }
        lsum = warp_sum(lsum);
        __syncwarp();
        float *red = reinterpret_cast<float *>(scr); // end of the V pass: the warp's partial o, l
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
        if (rc.tail_cta && warp == kWarps - 1) { // tail values, exact
            const float *tsc = sm.tscores + (ri & 1) * 32;
            const DT *vt0 = reinterpret_cast<const DT *>(a.tail) + ((int64_t)(rc.b * 2 + 1) * a.H + rc.h) * 32 * D;
            float tl = 0.f;
            for (int t = 0; t < rc.tail; ++t) {
                const float w = exp2f(tsc[t] - m2);
                tl += w;
                const DT *vt = vt0 + (int64_t)t * D;
#pragma unroll
                for (int c4 = 0; c4 < D / 32; ++c4)
                    red[lane + 32 * c4] = fmaf(w, to_f32(vt[lane + 32 * c4]), red[lane + 32 * c4]);
            }
            __syncwarp();
            if (lane == 0)
                red[D] += tl;
        }
        named_sync(1, kThreads);
        float *part = sm.part + (ri & 1) * (D + 1);
        for (int c = threadIdx.x; c <= D; c += kThreads) {
            float sum = 0.f;
#pragma unroll
            for (int w = 0; w < kWarps; ++w)
                sum += reinterpret_cast<const float *>(sm.scr + w * SCR)[c];
            part[c] = sum;
        }
        named_sync(1, kThreads); // every warp's scratch is free again
    };

    // CTA `crank` writes channels [crank*D/C, (crank+1)*D/C) of row ri, summing the
    // partials of every CTA of the cluster.
    auto merge = [&](int ri, float m2) {
        const int row = cid + ri * ncl;
        const float *part = sm.part + (ri & 1) * (D + 1);
        const int per = D / (int)C;
        if ((int)threadIdx.x < per) {
            const int c = (int)crank * per + (int)threadIdx.x;
            float o = 0.f, l = 0.f;
            for (uint32_t r = 0; r < C; ++r) {
                o += ld_dsmem_f32(part + c, r);
                l += ld_dsmem_f32(part + D, r);
            }
            float out = 0.f;
            if (l > 0.f)
                out = o / l;
            else if (c == 0)
                atomicOr(a.status, LOOPKV_DEV_EMPTY_ROW);
            a.out[(int64_t)row * D + c] = out;
            if (c == 0) {
                if (a.row_max)
                    a.row_max[row] = m2 * 0.6931471805599453f;
                if (a.row_sum)
                    a.row_sum[row] = l;
            }
        }
    };

    float m_prev = 0.f, m_prev2 = 0.f;
    if (nrows > 0) {
        setup_row(0);
        load_segment();
        pump(spw);
        consume_k(0);
    }
    cluster_arrive(); // row 0
    for (int i = 1; i < nrows; ++i) {
        consume_k(i);
        cluster_wait(); // row i - 1: maxima of row i - 1, partials of row i - 2
        if (i >= 2)
            merge(i - 2, m_prev2);
        float m2, l2;
        cluster_row_stats(sm.stat + ((i - 1) % 3) * kWarps * 2, C, m2, l2);
        const float thr2 = row_threshold(a, m2, l2, decide);
        release_row(i - 1, thr2);
        consume_v(i - 1, m2, thr2);
        m_prev2 = m2;
        cluster_arrive(); // row i
    }
    cluster_wait(); // last row
    if (nrows >= 2)
        merge(nrows - 2, m_prev2);
    if (nrows > 0) {
        float m2, l2;
        cluster_row_stats(sm.stat + ((nrows - 1) % 3) * kWarps * 2, C, m2, l2);
        const float thr2 = row_threshold(a, m2, l2, decide);
        release_row(nrows - 1, thr2);
        consume_v(nrows - 1, m2, thr2);
        m_prev = m2;
    }
    cluster_arrive(); // partials of the last row
    cluster_wait();
    if (nrows > 0)
        merge(nrows - 1, m_prev);
    cluster_arrive(); // remote reads done
    cluster_wait();
}

template <int BITS, int D, typename DT>
int launch_t(const DecodeArgs &a, const DecodeShape &shp, cudaStream_t s)
{
    auto kern = shp.min_ctas == 5 ? decode_kernel<BITS, D, DT, 5> : decode_kernel<BITS, D, DT, 4>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, shp.smem);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    if (e == cudaSuccess && shp.cluster > 8)
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess)
        return LOOPKV_ERR_CUDA;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(shp.cluster * shp.clusters, 1, 1);
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
    e = cudaLaunchKernelEx(&cfg, kern, a, shp.stages_log2, shp.score_bufs);
    return e == cudaSuccess ? LOOPKV_OK : LOOPKV_ERR_CUDA;
}

// Clusters of size C that can be resident at once for this kernel and shared memory.
template <int BITS, int D, typename DT> int max_active_clusters(int C, int smem, int min_ctas)
{
    auto kern = min_ctas == 5 ? decode_kernel<BITS, D, DT, 5> : decode_kernel<BITS, D, DT, 4>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
        return 0;
    cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    if (C > 8)
        cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(C, 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = C;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess) {
        cudaGetLastError();
        return 0;
    }
    return n;
}

template <int BITS, int D, typename DT> DecodeShape shape_t(int rows, int max_blocks)
{
    using G = Geo<BITS, D>;
    DecodeShape best = {};
    double best_eff = -1.0;
    const int max_groups = max_blocks / 2;
    int sm_count = 148;
    {
        int dev = 0;
        cudaGetDevice(&dev);
        if (cudaDeviceGetAttribute(&sm_count, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            sm_count = 148;
    }
    const int smem_per_sm = 228 * 1024;
    const char *env_c = getenv("LOOPKV_DECODE_CLUSTER");
    const char *env_s = getenv("LOOPKV_DECODE_STAGES");
    const char *env_o = getenv("LOOPKV_DECODE_CTAS_PER_SM");
    for (int want_ctas = 4; want_ctas <= 5; ++want_ctas) {
    if (env_o && atoi(env_o) != want_ctas)
        continue;
    for (int C = 1; C <= 16; C *= 2) {
        if (env_c && atoi(env_c) != C)
            continue;
        if (D / C < 4)
            continue;
        const int cap = (max_groups + C - 1) / C;
        const int capw = (cap + kWarps - 1) / kWarps;
        const int budget = smem_per_sm / want_ctas - 1024;
        for (int nbuf = 1; nbuf <= 2; ++nbuf) {
            // slots per warp (a power of two): fill the shared memory of `want_ctas` CTAs per SM
            int spw = 8;
            while (spw > 2 && smem_bytes<BITS, D>(spw, capw, nbuf) > budget)
                spw >>= 1;
            if (env_s)
                spw = atoi(env_s);
            const int smem = smem_bytes<BITS, D>(spw, capw, nbuf);
            if (smem > 227 * 1024 || !layout_ok<BITS, D>(spw, capw, nbuf))
                continue;
            int ncl = max_active_clusters<BITS, D, DT>(C, smem, want_ctas);
            if (ncl <= 0)
                continue;
            if (ncl > rows)
                ncl = rows;
            if (nbuf == 1 && ncl < rows)
                continue; // a cluster would read several rows: it needs two score buffers
            // balance: each cluster takes ceil(rows / ncl) rows; too few CTAs per SM penalised;
            // more resident CTAs (warps to hide latency) and deeper rings (bytes in flight)
            // preferred
            const double rounds = (double)((rows + ncl - 1) / ncl);
            const double eff = ((double)rows / ncl) / rounds *
                               std::min(1.0, (double)(ncl * C) / (3.0 * sm_count)) *
                               (1.0 + 0.3 * std::min(1.0, (double)(ncl * C) / (want_ctas * sm_count))) *
                               (1.0 + 0.01 * spw);
            if (eff > best_eff + 1e-9) {
                best_eff = eff;
                best.cluster = C;
                best.clusters = ncl;
                best.stages = spw;
                best.stages_log2 = __builtin_ctz(spw);
                best.score_bufs = nbuf;
                best.smem = smem;
                best.threads = kThreads;
                best.cap = cap;
                best.min_ctas = want_ctas;
            }
            break;
        }
    }
    }
    return best;
}

}  // namespace

DecodeShape decode_shape(int bits, int D, int dtype, int rows, int max_blocks)
{
    const bool bf = dtype == LOOPKV_DTYPE_BF16;
    if (bits == 4) {
        if (D == 128)
            return bf ? shape_t<4, 128, __nv_bfloat16>(rows, max_blocks) : shape_t<4, 128, float>(rows, max_blocks);
        return bf ? shape_t<4, 64, __nv_bfloat16>(rows, max_blocks) : shape_t<4, 64, float>(rows, max_blocks);
    }
    if (D == 128)
        return bf ? shape_t<2, 128, __nv_bfloat16>(rows, max_blocks) : shape_t<2, 128, float>(rows, max_blocks);
    return bf ? shape_t<2, 64, __nv_bfloat16>(rows, max_blocks) : shape_t<2, 64, float>(rows, max_blocks);
}

int launch_decode(const DecodeArgs &a, int bits, int D, int dtype, const DecodeShape &shp, cudaStream_t s)
{
    if (shp.cluster <= 0 || shp.clusters <= 0)
        return LOOPKV_ERR_CUDA;
    const bool bf = dtype == LOOPKV_DTYPE_BF16;
    if (bits == 4) {
        if (D == 128)
            return bf ? launch_t<4, 128, __nv_bfloat16>(a, shp, s) : launch_t<4, 128, float>(a, shp, s);
        return bf ? launch_t<4, 64, __nv_bfloat16>(a, shp, s) : launch_t<4, 64, float>(a, shp, s);
    }
    if (D == 128)
        return bf ? launch_t<2, 128, __nv_bfloat16>(a, shp, s) : launch_t<2, 128, float>(a, shp, s);
    return bf ? launch_t<2, 64, __nv_bfloat16>(a, shp, s) : launch_t<2, 64, float>(a, shp, s);
}

}  // namespace lkv
