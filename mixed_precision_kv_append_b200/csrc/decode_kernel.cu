// decode_kernel.cu -- fused, plan-driven decode attention over the LoopKV cache.
//
// Two kernels.  decode_kernel (below) serves reads whose refine set depends on the row
// maximum (4-bit sources, tau > 0) and takes the exact maximum in two phases;
// decode_kernel_1p (further down) serves reads whose refine set is fixed in advance
// (2-bit sources, tau <= 0) in a single pass with a running maximum.
//
// One launch per cell (LoopKV paper, §3.4 "One launch per cell").  The grid is a set
// of persistent thread-block clusters of C CTAs; cluster c serves the (request, head)
// rows c, c + NC, c + 2NC, ... one after another.  Inside a row, CTA k of the cluster
// owns the 32-token groups k, k+C, k+2C, ... of the history; the unquantized near tokens
// (sink and window) are dealt over every warp of the cluster.  Warp w of a CTA owns the
// CTA's groups w, w+4, ...  For each row a warp:
//   1. K pass: streams the key codes and the per-channel key scale/zero of its groups
//      into shared memory with bulk asynchronous copies that it issues itself (one
//      elected lane, a private mbarrier ring), and computes every score from the full
//      4-bit (or 2-bit) keys with the key scale folded into q once per group (Appendix
//      "History reader").  Scores stay in shared memory.
//   2. Exact row maximum: the CTAs exchange their per-warp maxima through distributed
//      shared memory across a cluster barrier, so every CTA knows the exact m -- the
//      "ideal" rule of §3.3 (a token is cold if its weight is below tau times the
//      largest in its row), not a streaming seed.  With the normalised-weight rule the
//      same exchange carries the partial sums of exp(s_t - m_w).
//   3. V pass: streams V scale/zero and the hi plane of every token; the lo plane of a
//      token is fetched only if its weight passes the threshold (§3.3 "Read-time V
//      precision").  Hot tokens decode to z + s(4h+l), cold ones to the middle of their
//      bucket z + s(4h+1.5), 2-bit cells to z + s*code; the per-token scale and zero
//      are folded into the weight and a running sum.
//   4. Merge: since all CTAs used the same m, their partial sums add directly; the CTAs
//      reduce them through distributed shared memory and write out = o / l.
// With two score buffers rows are software-pipelined: while the cluster barrier that
// publishes row r's maxima completes, the warp already streams and scores the keys of row
// r+1, so the memory pipe never drains at a row boundary, and one cluster barrier per row
// carries both the per-warp maxima of row r and the partial outputs of row r-1.  Long
// rows, whose scores fill the shared memory, take one score buffer and run in sequence.
//
// Keys: the dot products of a 32-token group run in integers on the tensor cores
// (group_scores): the per-channel factors a_c = q_c * s_c are rounded to 30-bit fixed point
// and split into four signed byte digits, the [32 tokens x D] code matrix times the [D x 4]
// digit matrix runs as m16n8k32 u8 x s8 products with exact int32 accumulation, and the
// digit sums meet in fp32 with the zero term.
// Values: a value-plane word holds 4 tokens x 4 channels (token in the byte).  The hi and
// lo words merge into 4-bit codes (lo bits of cold tokens masked off), one AND unpacks the
// codes of one channel for 4 tokens, and dp4a against the two 8-bit digits of the tokens'
// 15-bit fixed-point weights w * scale (relative step 2^-15 of the group's largest) sums
// code * weight over tokens exactly in int32; each 32-token group's sum (< 2^24) converts
// to fp32 exactly.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "lkv_device.cuh"
#include "lkv_internal.h"

#include <algorithm>
#include <cstdio>
#include <cstdlib>

namespace lkv {
namespace {

constexpr int kWarps = 4; // every warp both issues the copies of its stages and computes on them
constexpr int kThreads = kWarps * 32;
constexpr int kGPS = 2;        // 32-token groups per pipeline stage (one barrier, one slot)

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
    static constexpr int GSLOT = ((KSTAGE > VSTAGE ? KSTAGE : VSTAGE) + 127) / 128 * 128; // one group
    static constexpr int STAGE = kGPS * GSLOT;
    static constexpr int ROWK = KCODES / 16;  // key bytes per token
    static constexpr int NCG = D / 32;        // 32-channel value groups per token
    static constexpr int NQ = D / 4;          // channel quads
};

// acc += sum of the four unsigned bytes of `u` times the four unsigned bytes of `d`
__device__ __forceinline__ void dp4a_uu(uint32_t &acc, uint32_t u, uint32_t d)
{
    asm("dp4a.u32.u32 %0, %1, %2, %0;" : "+r"(acc) : "r"(u), "r"(d));
}

// 2^x by the hardware approximation (relative error about 2^-22; tiny results flush to 0)
__device__ __forceinline__ float ex2(float x)
{
    float r;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}

// Byte b of the result = 0xFF if bit 8b+7 of x is set, else 0 (prmt's sign-replicating
// selector values 8..11).
__device__ __forceinline__ uint32_t byte_signs(uint32_t x)
{
    uint32_t r;
    asm("prmt.b32 %0, %1, 0, 0xBA98;" : "=r"(r) : "r"(x));
    return r;
}

// max over the warp of v
__device__ __forceinline__ float warp_max_f(float v)
{
    float r;
    asm volatile("redux.sync.max.f32 %0, %1, 0xffffffff;" : "=f"(r) : "f"(v));
    return r;
}

// max over the warp of |v|
__device__ __forceinline__ float warp_max_abs(float v)
{
    float r;
    asm volatile("redux.sync.max.abs.f32 %0, %1, 0xffffffff;" : "=f"(r) : "f"(v));
    return r;
}


// d += A (16 x 32, u8) * B (32 x 8, s8) with s32 accumulation: one warp-level tensor-core
// product.  Fragments (per lane, groupID g = lane / 4, t = lane % 4): a0 = row g, k 4t..4t+3;
// a1 = row g + 8, same k; a2 = row g, k 16 + 4t..; a3 = row g + 8, k 16 + 4t..; b0 = k 4t..4t+3
// of column g; b1 = k 16 + 4t.. of column g; d0, d1 = row g, columns 2t, 2t + 1; d2, d3 = row
// g + 8.  Element i of a register is its byte i.
__device__ __forceinline__ void mma_u8s8(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1)
{
    asm("mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Bytes of the per-warp digit table of group_scores: 4 rows (one per digit) of D bytes, each
// padded by 16 so that the B-fragment loads of two digit rows fall in different banks.
template <int D> __host__ __device__ constexpr int digit_table_bytes() { return 4 * (D + 16); }

// Scores (log2 units) of the 32 tokens of a group, exact up to one fp32 rounding of each
// partial sum: token j of block A is token j, token j of block B is token 16 + j; blkA and
// blkB point at the blocks' key regions (codes, then the per-channel scales in block A and
// zeros in block B).  Returns the score of token `lane`.  qreg: the query of the lane's channel
// quad as read (bf16 widens exactly); qscale = log2(e) / sqrt(D).  scr: the warp's scratch.
//
// The group's score is a dense integer contraction.  The factors a_c = q_c s_c are products of
// an 8-bit and an 11-bit significand, exact in fp32; they are rounded to 30-bit fixed point
// I_c = round(a_c 2^F), F = 29 - E (E = exponent of max |a|), which is exact for every channel
// within 2^11 of the largest, and I_c is split into four signed base-256 digits (balanced:
// I = d0 + 2^8 d1 + 2^16 d2 + 2^24 d3, each in [-128, 127]).  The codes of 32 tokens x D channels
// times the D x 4 digit matrix is then a [32 x D] x [D x 4] integer product, which the tensor
// cores take as m16n8k32 tiles (u8 codes, s8 digits, digits in columns 0..3 of the 8): tokens
// are the 16 rows of a tile (one tile per block), channels the k dimension.  Since the sum runs
// over channels in any order, each lane takes one 4-byte code word per k half as it lies in the
// row: 4-bit codes unpack with one mask into the low nibbles (channels 8W..8W+3 of word W) and
// one into the high nibbles (16 x channels 8W+4..8W+7, accumulated apart and divided by 16
// exactly); 2-bit codes unpack field by field (channels 16W+4i..16W+4i+3).  The B fragment of a
// lane is the digits of exactly the channels its A words hold, loaded from a table that the
// factor lanes fill.  Per token, sum_c I_c code_c = P0 + 2^8 P1 + 2^16 P2 + 2^24 P3 with P_k the
// exact int32 column sums; the pairs (P0, P1) and (P2, P3) combine exactly in int32 and meet in
// fp32, scaled by 2^-F, with the zero term sum_c q_c z_c.
template <int BITS, int D>
__device__ __forceinline__ float group_scores(const uint8_t *blkA, const uint8_t *blkB, uint8_t *scr,
                                              const float (&qreg)[4], const float qscale, const int lane)
{
    using G = Geo<BITS, D>;
    constexpr int DROW = D + 16;
    const bool ownq = lane < G::NQ;
    // factors a_c = q_c s_c of the lane's quad (exact) and the zero term sum_c q_c z_c
    float av[4], zs = 0.f;
    {
        uint2 sr = make_uint2(0u, 0u), zr = make_uint2(0u, 0u);
        if (ownq) {
            sr = *reinterpret_cast<const uint2 *>(blkA + G::KCODES + 8 * lane); // scales
            zr = *reinterpret_cast<const uint2 *>(blkB + G::KCODES + 8 * lane); // zeros
        }
        const float2 s01 = __half22float2(*reinterpret_cast<const __half2 *>(&sr.x));
        const float2 s23 = __half22float2(*reinterpret_cast<const __half2 *>(&sr.y));
        const float2 z01 = __half22float2(*reinterpret_cast<const __half2 *>(&zr.x));
        const float2 z23 = __half22float2(*reinterpret_cast<const __half2 *>(&zr.y));
        av[0] = qreg[0] * s01.x;
        av[1] = qreg[1] * s01.y;
        av[2] = qreg[2] * s23.x;
        av[3] = qreg[3] * s23.y;
        zs = fmaf(qreg[0], z01.x, fmaf(qreg[1], z01.y, fmaf(qreg[2], z23.x, qreg[3] * z23.y)));
    }
    const float amax = warp_max_abs(fmaxf(fmaxf(fabsf(av[0]), fabsf(av[1])), fmaxf(fabsf(av[2]), fabsf(av[3]))));
    zs = warp_sum(zs);
    // F = 29 - E keeps |I| < 2^30 (capped so that 2^F and 2^-F stay normal)
    int F = 29 - ((int)(__float_as_uint(amax) >> 23) - 127);
    F = F > 126 ? 126 : F;
    const float fs = __int_as_float((F + 127) << 23);
    if (ownq) {
        int I[4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
            I[i] = __float2int_rn(av[i] * fs);
        // byte k of I + (0x80 in each byte below k) is digit k as a signed byte.  Quad L goes to
        // word NB t + pos(j) of each row (t = L / NB, j = L % NB), ordered so that the two words
        // of every B fragment are adjacent in the lane's loaded registers (see the mma calls)
        constexpr int NBW = D / 16;
        const int jq = lane % NBW;
        const int pos = NBW == 8 ? (BITS == 4 ? (jq & 1) * 4 + (jq >> 1) : (jq & 3) * 2 + (jq >> 2))
                                 : (BITS == 4 ? (jq & 1) * 2 + (jq >> 1) : jq);
        uint32_t *tab = reinterpret_cast<uint32_t *>(scr) + (lane - jq) + pos;
        tab[0] = __byte_perm(__byte_perm(I[0], I[1], 0x0040), __byte_perm(I[2], I[3], 0x0040), 0x5410);
#pragma unroll
        for (int k = 1; k < 4; ++k) {
            const int off = (int)(0x808080u >> (8 * (3 - k)));
            const uint32_t sel = (uint32_t)(((4 + k) << 4) | k);
            tab[k * DROW / 4] = __byte_perm(__byte_perm(I[0] + off, I[1] + off, sel),
                                            __byte_perm(I[2] + off, I[3] + off, sel), 0x5410);
        }
    }
    __syncwarp();
    const int g = lane >> 2, t = lane & 3;
    constexpr int NB = D / 16; // digit words (channel quads) of a lane's B fragment
    uint32_t b[NB];
    if (g < 4) {
        const uint8_t *row = scr + g * DROW + t * (4 * NB);
#pragma unroll
        for (int j = 0; j < NB / 4; ++j) {
            const uint4 v = *reinterpret_cast<const uint4 *>(row + 16 * j);
            b[4 * j] = v.x, b[4 * j + 1] = v.y, b[4 * j + 2] = v.z, b[4 * j + 3] = v.w;
        }
    } else {
#pragma unroll
        for (int j = 0; j < NB; ++j)
            b[j] = 0u;
    }
    constexpr uint32_t M2 = 0x03030303u, M4 = 0x0F0F0F0Fu, H4 = 0xF0F0F0F0u;
    float sv[2][2]; // scores of tokens g, g + 8 of each block (valid in lanes with t = 0)
    const float k1 = qscale * __int_as_float((127 - F) << 23), zq = zs * qscale;
#pragma unroll
    for (int mt = 0; mt < 2; ++mt) {
        const uint8_t *rows = (mt ? blkB : blkA);
        int c[4] = {0, 0, 0, 0};
        if (BITS == 4) {
            int ch[4] = {0, 0, 0, 0};
            if (D == 128) { // words 4t..4t+3: quads 8t + 2w (low nibbles) and 8t + 2w + 1 (high)
                const uint4 r0 = *reinterpret_cast<const uint4 *>(rows + g * G::ROWK + 16 * t);
                const uint4 r1 = *reinterpret_cast<const uint4 *>(rows + (g + 8) * G::ROWK + 16 * t);
                // b = digits of quads 8t + {0, 2, 4, 6, 1, 3, 5, 7}
                mma_u8s8(c, r0.x & M4, r1.x & M4, r0.y & M4, r1.y & M4, b[0], b[1]);
                mma_u8s8(c, r0.z & M4, r1.z & M4, r0.w & M4, r1.w & M4, b[2], b[3]);
                mma_u8s8(ch, r0.x & H4, r1.x & H4, r0.y & H4, r1.y & H4, b[4], b[5]);
                mma_u8s8(ch, r0.z & H4, r1.z & H4, r0.w & H4, r1.w & H4, b[6], b[7]);
            } else { // D = 64: words 2t, 2t+1: quads 4t, 4t+2 (low), 4t+1, 4t+3 (high)
                const uint2 r0 = *reinterpret_cast<const uint2 *>(rows + g * G::ROWK + 8 * t);
                const uint2 r1 = *reinterpret_cast<const uint2 *>(rows + (g + 8) * G::ROWK + 8 * t);
                // b = digits of quads 4t + {0, 2, 1, 3}
                mma_u8s8(c, r0.x & M4, r1.x & M4, r0.y & M4, r1.y & M4, b[0], b[1]);
                mma_u8s8(ch, r0.x & H4, r1.x & H4, r0.y & H4, r1.y & H4, b[2], b[3]);
            }
#pragma unroll
            for (int r = 0; r < 4; ++r)
                c[r] += ch[r] >> 4; // a multiple of 16: exact
        } else if (D == 128) { // words 2t, 2t+1: field i is quad 8t + i, resp. 8t + 4 + i
            const uint2 r0 = *reinterpret_cast<const uint2 *>(rows + g * G::ROWK + 8 * t);
            const uint2 r1 = *reinterpret_cast<const uint2 *>(rows + (g + 8) * G::ROWK + 8 * t);
#pragma unroll
            for (int i = 0; i < 4; ++i) // b = digits of quads 8t + {0, 4, 1, 5, 2, 6, 3, 7}
                mma_u8s8(c, (r0.x >> (2 * i)) & M2, (r1.x >> (2 * i)) & M2, (r0.y >> (2 * i)) & M2,
                         (r1.y >> (2 * i)) & M2, b[2 * i], b[2 * i + 1]);
        } else { // D = 64, 2-bit: word t, field i is quad 4t + i
            const uint32_t r0 = *reinterpret_cast<const uint32_t *>(rows + g * G::ROWK + 4 * t);
            const uint32_t r1 = *reinterpret_cast<const uint32_t *>(rows + (g + 8) * G::ROWK + 4 * t);
#pragma unroll
            for (int i = 0; i < 4; i += 2)
                mma_u8s8(c, (r0 >> (2 * i)) & M2, (r1 >> (2 * i)) & M2, (r0 >> (2 * i + 2)) & M2,
                         (r1 >> (2 * i + 2)) & M2, b[i], b[i + 1]);
        }
        // lane t = 0 holds digits 0, 1 of tokens g, g + 8; lane t = 1 digits 2, 3 (|P_k| < 2^18)
        const float e0 = (float)(c[0] + (c[1] << 8)), e1 = (float)(c[2] + (c[3] << 8));
        const float h0 = __shfl_down_sync(0xFFFFFFFFu, e0, 1), h1 = __shfl_down_sync(0xFFFFFFFFu, e1, 1);
        sv[mt][0] = fmaf(h0, k1 * 65536.f, fmaf(e0, k1, zq));
        sv[mt][1] = fmaf(h1, k1 * 65536.f, fmaf(e1, k1, zq));
    }
    // token L sits in lane 4 (L % 8): block L / 16, row half (L / 8) % 2
    const int src = (lane & 7) << 2, j = lane >> 3;
    const float v0 = __shfl_sync(0xFFFFFFFFu, sv[0][0], src), v1 = __shfl_sync(0xFFFFFFFFu, sv[0][1], src);
    const float v2 = __shfl_sync(0xFFFFFFFFu, sv[1][0], src), v3 = __shfl_sync(0xFFFFFFFFu, sv[1][1], src);
    return j == 0 ? v0 : (j == 1 ? v1 : (j == 2 ? v2 : v3));
}

// Value sums of one 32-token group for a lane's channel quad (channels 0..3 of the quad).  A
// plane word holds 4 tokens x 4 channels (token in the byte).  E packs the codes of channels 0
// and 2 of each token into one byte (c0 + 16 c2), O those of channels 1 and 3; dp4a of E and of
// E with its low nibbles masked (16 c2) against a weight digit gives sum c0 d + 16 sum c2 d and
// 16 sum c2 d, from which both sums follow exactly, so no nibble is shifted down.  Two weight
// digits (d0, d1: the token weights' 15-bit fixed point) per word.
struct VSums {
    uint32_t a0[4] = {0u, 0u, 0u, 0u}, a1[4] = {0u, 0u, 0u, 0u}; // E, E & 0xF0.., O, O & 0xF0..

    // 4-bit: hi word hw (2-bit fields h) and lo word lw (fields l, zero for cold tokens) give
    // codes 4h + l; 2-bit: hw holds the codes themselves.
    template <int BITS> __device__ __forceinline__ void add(uint32_t hw, uint32_t lw, uint32_t d0, uint32_t d1)
    {
        uint32_t E, O;
        if (BITS == 4) {
            E = ((hw << 2) & 0xCCCCCCCCu) | (lw & 0x33333333u);
            O = (hw & 0xCCCCCCCCu) | ((lw >> 2) & 0x33333333u);
        } else {
            E = hw & 0x33333333u;
            O = (hw >> 2) & 0x33333333u;
        }
        const uint32_t EH = E & 0xF0F0F0F0u, OH = O & 0xF0F0F0F0u;
        dp4a_uu(a0[0], E, d0);
        dp4a_uu(a1[0], E, d1);
        dp4a_uu(a0[1], EH, d0);
        dp4a_uu(a1[1], EH, d1);
        dp4a_uu(a0[2], O, d0);
        dp4a_uu(a1[2], O, d1);
        dp4a_uu(a0[3], OH, d0);
        dp4a_uu(a1[3], OH, d1);
    }

    // o[i] += (sum over tokens of code_i * weight) * fsi.  Per channel sum_t code I < 15 * 2^15 * 32
    // < 2^24, exact in fp32; the sums of E bytes stay below 2^30.
    __device__ __forceinline__ void finish(float fsi, float (&o)[4]) const
    {
        const uint32_t vE = a0[0] + (a1[0] << 8), vEH = a0[1] + (a1[1] << 8);
        const uint32_t vO = a0[2] + (a1[2] << 8), vOH = a0[3] + (a1[3] << 8);
        o[0] = fmaf((float)(vE - vEH), fsi, o[0]);
        o[1] = fmaf((float)(vO - vOH), fsi, o[1]);
        o[2] = fmaf((float)(vEH >> 4), fsi, o[2]);
        o[3] = fmaf((float)(vOH >> 4), fsi, o[3]);
    }
};

// Four consecutive elements of a near-region row as floats (bf16 widens exactly); p is
// 8-byte (bf16) or 16-byte (fp32) aligned.
__device__ __forceinline__ void load4f(const __nv_bfloat16 *p, float (&f)[4])
{
    const uint2 u = *reinterpret_cast<const uint2 *>(p);
    f[0] = __uint_as_float(u.x << 16);
    f[1] = __uint_as_float(u.x & 0xFFFF0000u);
    f[2] = __uint_as_float(u.y << 16);
    f[3] = __uint_as_float(u.y & 0xFFFF0000u);
}
__device__ __forceinline__ void load4f(const float *p, float (&f)[4])
{
    const float4 v = *reinterpret_cast<const float4 *>(p);
    f[0] = v.x, f[1] = v.y, f[2] = v.z, f[3] = v.w;
}

// Near tokens a warp takes per round of loads.
constexpr int kNearBatch = 4;

// q . k of up to kNearBatch unquantized (near) tokens, in log2 units: key rows krow[u] (nullptr:
// no token, score 0); the lane holds channels 4 lane .. 4 lane + 3 of the exact query.  Every
// load is issued before the first product, so that one memory latency covers the batch.
// Warp-uniform results.
template <int D, typename DT>
__device__ __forceinline__ void near_scores(const DT *const (&krow)[kNearBatch], const float (&qreg)[4],
                                            const float qscale, const int lane, float (&s)[kNearBatch])
{
    float k[kNearBatch][4];
#pragma unroll
    for (int u = 0; u < kNearBatch; ++u) {
        k[u][0] = k[u][1] = k[u][2] = k[u][3] = 0.f;
        if (lane < D / 4 && krow[u] != nullptr)
            load4f(krow[u] + 4 * lane, k[u]);
    }
    float p[kNearBatch];
#pragma unroll
    for (int u = 0; u < kNearBatch; ++u)
        p[u] = lane < D / 4 ? fmaf(qreg[0], k[u][0], fmaf(qreg[1], k[u][1], fmaf(qreg[2], k[u][2], qreg[3] * k[u][3])))
                            : 0.f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
#pragma unroll
        for (int u = 0; u < kNearBatch; ++u)
            p[u] += __shfl_xor_sync(0xFFFFFFFFu, p[u], o);
#pragma unroll
    for (int u = 0; u < kNearBatch; ++u)
        s[u] = p[u] * qscale;
}

// Slot of near token j (0 .. near tokens - 1) in a (cell, request)'s near region: the sink
// slots first, then the window ring from its oldest token (ws).  The order of the tokens
// does not matter to attention, only that each is read once.
__device__ __forceinline__ int near_slot(const DecodeArgs &a, int j, int ws)
{
    return j < a.sink ? j : a.sink + (ws + (j - a.sink)) % a.wring;
}

// Near rows per chunk of the two-phase reader's ring (one sub-slot: 16 D bytes, 2 KiB at D = 128).
template <typename DT> __host__ __device__ constexpr int near_chunk_rows() { return 16 / (int)sizeof(DT); }

// Logical near index (sink first, then the window from its oldest token, as near_slot orders
// them) of physical slot s of a near region holding nnear tokens, or -1 when the slot is empty.
__device__ __forceinline__ int near_index(const DecodeArgs &a, const int s, const int ws, const int nnear)
{
    int j = s;
    if (s >= a.sink) {
        int r = s - a.sink - ws;
        if (r < 0)
            r += a.wring;
        j = a.sink + r;
    }
    return j < nnear ? j : -1;
}

// Warm L2 with the rows of near tokens j0, j0 + stride, ... < n of one (cell, request, K or V,
// head) near region `base` (rows of D elements in near_slot order), a 128-byte line per lane and
// step: the rows are read after the row's history groups, long after this call.
template <int D, typename DT>
__device__ __forceinline__ void prefetch_near(const DecodeArgs &a, const DT *base, const int ws, const int j0,
                                              const int stride, const int n, const int lane)
{
    constexpr int LPR = D * (int)sizeof(DT) / 128; // lines per row
    const int cnt = n > j0 ? (n - j0 + stride - 1) / stride : 0;
    for (int i = lane; i < cnt * LPR; i += 32) {
        const int j = j0 + (i / LPR) * stride;
        prefetch_l2_keep(reinterpret_cast<const char *>(base + (int64_t)near_slot(a, j, ws) * D) + 128 * (i % LPR));
    }
}

struct Smem {
    uint8_t *ring;     // [kWarps][spw][STAGE] stage slots (kGPS groups each), a private slice per warp
    uint64_t *full;    // [kWarps][spw] completion barriers of the slots
    float *scores;     // [nbuf][kWarps][capw * 32] scores of a warp's groups, by row parity
    float *tscores;    // [2][32] tail scores, by row parity
    uint8_t *scr;      // [kWarps][SCR] per-warp scratch, used in turn as: key digit records
                       // [D/4 + D/32][16 B] (padded) during a K stage, the fixed-point weight transpose
                       // [D/32][40 words] (overwritten in place by the value digit records)
                       // and 2^-F during a V stage, the warp's partial o and l [D + 1] at
                       // the end of a V pass
    float *stat;       // [3][kWarps][4] per-warp (max, sum exp(s - max), sink max, -), by row index mod 3
    float *part;       // [2][D + 1] CTA partial o and l of a row, by row parity
    int32_t *ids;      // [3][kWarps][2 * capw] block ids of a warp's groups, by row index mod 3
    int32_t *irow;     // [3][kWarps][IR_N] row parameters and issuer state, by row index mod 3
    int32_t *order;    // [kMaxOrder] requests by decreasing history length, then index
};

// Fields of a row slot (Smem::irow).
enum {
    IR_ROW = 0, IR_B, IR_H, IR_N, IR_TAIL, IR_WS,
    IR_G0,   // first history group inside the attention window
    IR_M0,   // tokens of group IR_G0 before the window
    IR_HIST, // history tokens of the row
    IR_NC,   // near-region chunks read by this warp (streamed near regions)
    IR_N_FIELDS = 16
};

// First history token inside a sliding attention window of `win` tokens (0: full attention)
// for a row of `hist` history and `nnear` near tokens: positions are the sink (0 .. sink-1),
// the history (sink .. sink+hist-1), then the window; the last `win` positions are attended.
__host__ __device__ __forceinline__ int window_first(int win, int sink, int hist, int nnear)
{
    if (win <= 0)
        return 0;
    int h0 = hist + nnear - win - sink;
    return h0 < 0 ? 0 : (h0 > hist ? hist : h0);
}

// Whether near token j (sink first, then the window) is inside the attention window.
__device__ __forceinline__ bool near_attended(const DecodeArgs &a, int j, int hist, int nnear)
{
    if (a.attn_window <= 0)
        return true;
    const int pos = j < a.sink ? j : hist + j;
    return pos >= hist + nnear - a.attn_window;
}

// Byte offsets of the shared-memory regions; every region starts on a 16-byte boundary
// (digit records, weights and stage data are read with 16-byte vector loads).
struct SmemLayout {
    int full, scores, tscores, scr, stat, part, ids, irow, order, total;
};

constexpr int kMaxOrder = 64; // batches up to this size are ordered longest request first

__host__ __device__ constexpr int align16(int x) { return (x + 15) & ~15; }
__host__ __device__ constexpr int imax(int a, int b) { return a > b ? a : b; }

// Bytes of a warp's scratch: the largest of its three uses.
template <int D> __host__ __device__ constexpr int scratch_bytes()
{
    return align16(imax(digit_table_bytes<D>(), imax((D + 2) * 4, (D / 32) * 40 * 4 + 4)));
}

// nbuf: score buffers (2: the next row's keys are scored while the current row's values are
// read; 1: a cluster's rows run one after another, for long rows whose scores fill the
// shared memory).
template <int BITS, int D>
__host__ __device__ constexpr SmemLayout smem_layout(int spw, int capw, int nbuf, int near_cap)
{
    SmemLayout L{};
    int o = kWarps * spw * Geo<BITS, D>::STAGE; // ring, 128-byte aligned slots
    L.full = o;
    o = align16(o + kWarps * spw * 8);
    L.scores = o;
    o = align16(o + nbuf * kWarps * capw * 32 * 4);
    L.tscores = o;
    o = align16(o + 2 * near_cap * 4);
    L.scr = o;
    o = align16(o + kWarps * scratch_bytes<D>());
    L.stat = o;
    o = align16(o + 3 * kWarps * 4 * 4);
    L.part = o;
    o = align16(o + 2 * (D + 1) * 4);
    L.ids = o;
    o = align16(o + 3 * kWarps * 2 * capw * 4);
    L.irow = o;
    o = align16(o + 3 * kWarps * IR_N_FIELDS * 4);
    L.order = o;
    o = align16(o + 2 * kMaxOrder * 4);
    L.total = o;
    return L;
}

template <int BITS, int D> __host__ __device__ constexpr int smem_bytes(int spw, int capw, int nbuf, int near_cap)
{
    return smem_layout<BITS, D>(spw, capw, nbuf, near_cap).total;
}

template <int BITS, int D> __device__ Smem carve(uint8_t *base, int spw, int capw, int nbuf, int near_cap)
{
    const SmemLayout L = smem_layout<BITS, D>(spw, capw, nbuf, near_cap);
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
    s.order = reinterpret_cast<int32_t *>(base + L.order);
    return s;
}

// Host check of a layout: every region 16-byte aligned, in order, inside the allocation;
// the per-warp id lists 8-byte aligned (read as pairs).
template <int BITS, int D> bool layout_ok(int spw, int capw, int nbuf, int near_cap)
{
    const SmemLayout L = smem_layout<BITS, D>(spw, capw, nbuf, near_cap);
    const int offs[] = {L.full, L.scores, L.tscores, L.scr, L.stat, L.part, L.ids, L.irow, L.order};
    int prev = kWarps * spw * Geo<BITS, D>::STAGE;
    for (int o : offs) {
        if (o % 16 || o < prev)
            return false;
        prev = o;
    }
    return (Geo<BITS, D>::GSLOT % 128) == 0 && L.total >= prev && (spw & (spw - 1)) == 0 &&
           scratch_bytes<D>() >= digit_table_bytes<D>() && scratch_bytes<D>() >= (D + 1) * 4 &&
           scratch_bytes<D>() >= (D / 32) * 40 * 4 + 4 && (2 * capw * 4) % 8 == 0;
}

// Groups of a row owned by warp w of the CTA: local groups w, w + kWarps, ...
__device__ __forceinline__ int owned(int nmy, int w) { return nmy > w ? (nmy - w + kWarps - 1) / kWarps : 0; }

// Segment sig of a warp's stage sequence: returns whether it is a V segment and its row
// index.  Overlapped order (two score buffers) K(0), K(1), V(0), K(2), V(1), ..., V(n-1);
// sequential order (one score buffer) K(0), V(0), K(1), V(1), ...
__device__ __forceinline__ void segment(int sig, int nrows, bool seq, bool &is_v, int &ri)
{
    if (seq) {
        is_v = sig & 1;
        ri = sig >> 1;
    } else if (sig == 0) {
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

// Row max m (log2 units), for the normalised rule l = sum_t 2^(s_t - m), and the largest
// sink score m0 (the streaming rule's seed), from the per-warp records of every CTA of the
// cluster.  Lane j < C * kWarps fetches record j; the warp reductions give every lane the
// same values.
__device__ __forceinline__ void cluster_row_stats(const float *stat, uint32_t C, int lane, float &m, float &l,
                                                  float &m0)
{
    float mw = -INFINITY, lw = 0.f, sw = -INFINITY;
    for (int j = lane; j < (int)C * kWarps; j += 32) {
        const float mj = ld_dsmem_f32(stat + 4 * (j % kWarps), (uint32_t)(j / kWarps));
        const float lj = ld_dsmem_f32(stat + 4 * (j % kWarps) + 1, (uint32_t)(j / kWarps));
        sw = fmaxf(sw, ld_dsmem_f32(stat + 4 * (j % kWarps) + 2, (uint32_t)(j / kWarps)));
        if (mj == -INFINITY)
            continue;
        if (mw == -INFINITY) {
            mw = mj;
            lw = lj;
        } else {
            const float mn = fmaxf(mw, mj);
            lw = lw * exp2f(mw - mn) + lj * exp2f(mj - mn);
            mw = mn;
        }
    }
    m = warp_max(mw);
    m0 = warp_max(sw);
    l = 0.f;
    if (m == -INFINITY)
        return;
    l = __shfl_sync(0xFFFFFFFFu, warp_sum(mw == -INFINITY ? 0.f : lw * exp2f(mw - m)), 0); // one value for all lanes
}

// MINCTA: CTAs per SM the registers are budgeted for (4: <= 128 registers, 5: <= 96).  VAR: the
// build.  2 (general) serves everything: the streaming rule, sliding windows, the refine-set bitmap
// of the debug entry point, the wait test hook and streamed near regions.  Launches that use none
// of the first four take a lean build, whose per-group path carries no tests for them: 1 when the
// near region is streamed (a sink or a window), else 0.
template <int BITS, int D, typename DT, int MINCTA, int VAR>
__global__ void __launch_bounds__(kThreads, MINCTA) decode_kernel(const DecodeArgs a, const int spw_log2, const int nbuf)
{
    constexpr bool GEN = VAR == 2;
    constexpr bool NSC = VAR >= 1; // the streamed near path is compiled in
    using G = Geo<BITS, D>;
    extern __shared__ __align__(128) uint8_t smem_raw[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int spw = 1 << spw_log2, smask = spw - 1;
    const uint32_t crank = cluster_ctarank(), C = cluster_nctarank();
    const int cid = blockIdx.x / (int)C, ncl = gridDim.x / (int)C;

    const int capw = (a.cap_groups + kWarps - 1) / kWarps;
    Smem sm = carve<BITS, D>(smem_raw, spw, capw, nbuf, a.near_cap);
    static_assert(BITS == 4, "the exact-maximum reader serves 4-bit sources read with tau > 0");
    // streaming refine rule (LOOPKV_TAU_STREAM): per warp, tokens are tested against a running
    // maximum seeded with the row's largest sink score, in the warp's group order
    const bool stream = GEN && a.tau_mode == LOOPKV_TAU_STREAM;
    const float ltau = log2f(a.tau);
    const bool seq = nbuf == 1; // one score buffer: rows one after another (see the main loop)
    // A near region beyond a 32-token tail (a sink or a window) streams through the ring in chunks
    // of NR physical rows, dealt over the cluster's warps like history groups: chunk c to warp
    // c mod 4C.  Slots without a token are read too and get score -inf.
    const bool nstream = NSC && a.near_cap > 32;
    constexpr int NR = near_chunk_rows<DT>();
    constexpr uint32_t NRB = (uint32_t)(NR * D * sizeof(DT)); // bytes of a chunk
    static_assert(NR * D * (int)sizeof(DT) <= G::GSLOT, "a near chunk fills at most one sub-slot");
    // warp rank in the cluster and warps of the cluster, recomputed where used (cheaper than
    // holding them in registers through the whole kernel)
    auto wgl = [&]() { return (int)crank * kWarps + warp; };
    auto nwl = [&]() { return (int)C * kWarps; };
    bool dep_ok = false; // the previous grid of the stream has finished (near rows are final)
    // byte distance between consecutive block ids in the pools (one block = H heads)
    const uint32_t bstride = (uint32_t)a.H * G::HM, lstride = (uint32_t)a.H * G::LOB;

    // Programmatic dependent launch: the next kernel of the stream may start its CTAs once
    // every CTA of this grid has run this (so it never takes resources this grid still
    // needs); they wait in griddepcontrol.wait for this grid to finish before reading q.
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    if (lane == 0)
        for (int i = 0; i < spw; ++i)
            mbar_init(&sm.full[warp * spw + i], 1);
    fence_mbar_init();
    // Row schedule.  Requests of equal history length: cluster c takes rows c, c + ncl, ...
    // Otherwise (batches up to kMaxOrder) a pass-by-pass deal of the rows ordered longest
    // request first: pass j gives positions j*ncl .. j*ncl + ncl - 1 to clusters 0..ncl-1
    // (even j) or ncl-1..0 (odd j), position p being head p % H of the (p / H)-th longest
    // request, so that a cluster drawing a long row early draws a short one next.
    const int nreq = a.rows / a.H;
    bool ordered = false;
    if (nreq <= kMaxOrder) { // rank the requests by history length (every CTA derives the same order)
        int32_t *lens = sm.order + kMaxOrder;
        for (int b = threadIdx.x; b < nreq; b += kThreads)
            lens[b] = a.hist_len[b];
        __syncthreads();
        for (int b = threadIdx.x; b < nreq; b += kThreads) {
            const int lb = lens[b];
            int rank = 0;
            for (int b2 = 0; b2 < nreq; ++b2) {
                const int l2 = lens[b2];
                rank += (l2 > lb) || (l2 == lb && b2 < b);
            }
            sm.order[rank] = b;
        }
        for (int b = 1; b < nreq; ++b)
            ordered |= lens[b] != lens[0];
    }
    __syncthreads();
    const int full_passes = a.rows / ncl, rem = a.rows % ncl;
    const int nrows = !ordered ? (cid < a.rows ? (a.rows - 1 - cid) / ncl + 1 : 0)
                               : full_passes + ((full_passes & 1) ? (cid >= ncl - rem) : (cid < rem));
    auto row_of = [&](int ri) {
        if (!ordered)
            return cid + ri * ncl;
        const int p = ri * ncl + ((ri & 1) ? ncl - 1 - cid : cid);
        const int q = p / a.H;
        return sm.order[q] * a.H + (p - q * a.H);
    };

    uint8_t *ring = sm.ring + warp * spw * G::STAGE;
    uint64_t *full = sm.full + warp * spw;
    auto scores_of = [&](int ri) { return sm.scores + (((nbuf == 2) ? (ri & 1) : 0) * kWarps + warp) * capw * 32; };
    auto ids_of = [&](int ri) { return sm.ids + ((ri % 3) * kWarps + warp) * 2 * capw; };
    auto irow_of = [&](int ri) { return sm.irow + ((ri % 3) * kWarps + warp) * IR_N_FIELDS; };

    // ---------------------------------------------------------------- issuing
    // A warp issues the bulk copies of its own stages, `spw` stages ahead of its compute.
    int iss_sig = -1, iss_k = 0, iss_n = 0; // the sequence starts before its first segment
    int seg_len = 0, seg_ri = 0;   // current segment: own stages and row index
    int seg_n = 0;                 // groups of the segment's row owned by this warp
    bool seg_v = false;
    const uint8_t *seg_src = nullptr; // main pool + head offset (+ K part) of the segment's row
    const uint8_t *seg_near = nullptr; // near region (K or V) of the segment's row
    int seg_gst = 0, seg_nc = 0;      // group stages, then near chunks of this warp
    const int2 *seg_ids = nullptr;
    int setup_upto = -1;           // rows 0..setup_upto have their parameters and ids in place
    // After one bounded wait gives up, later waits are skipped, nothing new is issued, and the
    // stages from drain_from on are waited for (bounded) before the CTA exits.
    bool timed_out = false;
    int drain_from = 0;

    // Row parameters, validation and the warp's block ids of row ri.
    auto setup_row = [&](int ri) {
        const int row = row_of(ri);
        const int b = row / a.H, h = row - b * a.H;
        // history length and block ids come from flush / ingest / reset launches, which the
        // host never overlaps with a decode; the tail length (appends) is read after the grid
        // dependency wait (read_tail)
        int hist = a.hist_len[b];
        bool bad = false;
        if (hist < 0 || hist > a.max_blocks * 16 || (hist & 31)) {
            bad = true;
            hist = 0;
        }
        // sliding attention window: only the groups from the window's first token on (the
        // host launches windowed reads without overlap, so the near count is final here)
        int h0 = 0;
        if (GEN && a.attn_window > 0) {
            const int nn = a.tail_len[b];
            h0 = window_first(a.attn_window, a.sink, hist, nn < 0 ? 0 : nn);
        }
        const int g0 = h0 >> 5;
        const int ngroups = (hist >> 5) - g0;
        int nmy = ngroups > (int)crank ? (ngroups - (int)crank + (int)C - 1) / (int)C : 0;
        if (nmy > a.cap_groups) {
            bad = true;
            nmy = a.cap_groups;
        }
        if (bad && warp == 0 && lane == 0)
            atomicOr(a.status, LOOPKV_DEV_STATE);
        const int n = owned(nmy, warp);
        const int32_t *bt = a.block_table + (int64_t)b * a.max_blocks;
        int32_t *ids = ids_of(ri);
        for (int k = lane; k < 2 * n; k += 32) {
            const int g = g0 + (int)crank + (warp + (k >> 1) * kWarps) * (int)C;
            int id = bt[2 * g + (k & 1)];
            if (id < 0 || id >= a.pool_blocks) {
                atomicOr(a.status, LOOPKV_DEV_STATE);
                id = 0;
            }
            ids[k] = id;
        }
        int32_t *st = irow_of(ri);
        if (lane == 0) {
            st[IR_ROW] = row;
            st[IR_B] = b;
            st[IR_H] = h;
            st[IR_N] = n;
            st[IR_TAIL] = -1; // tail length not read yet (read after the grid dependency wait)
            st[IR_G0] = g0;
            st[IR_M0] = h0 & 31;
            st[IR_HIST] = hist;
            if (NSC) {
                const int nch = nstream ? a.near_cap / NR : 0;
                st[IR_NC] = nch > wgl() ? (nch - wgl() + nwl() - 1) / nwl() : 0;
            }
        }
        __syncwarp();
    };
    auto load_segment = [&]() {
        segment(iss_sig, nrows, seq, seg_v, seg_ri);
        const int32_t *st = irow_of(seg_ri);
        seg_n = st[IR_N];
        seg_gst = (seg_n + kGPS - 1) / kGPS;
        seg_len = seg_gst;
        seg_src = a.main + (size_t)st[IR_H] * G::HM + (seg_v ? G::KB : 0);
        if (NSC) {
            seg_nc = st[IR_NC];
            seg_len += (seg_nc + kGPS - 1) / kGPS;
            seg_near = reinterpret_cast<const uint8_t *>(a.tail) +
                       ((int64_t)(st[IR_B] * 2 + (seg_v ? 1 : 0)) * a.H + st[IR_H]) * a.near_cap * D * sizeof(DT);
        }
        seg_ids = reinterpret_cast<const int2 *>(ids_of(seg_ri));
    };
    // Stage k2 of the current segment: groups kGPS*k2 .. kGPS*k2 + ng - 1 of the row, group
    // j into sub-slot j.
    auto issue_stage = [&](int n) {
        const int k2 = iss_k;
        uint8_t *stg = ring + (n & smask) * G::STAGE;
        uint64_t *fb = &full[n & smask];
        if (NSC && k2 >= seg_gst) { // near stage: this warp's chunks kGPS*(k2 - seg_gst) .. of the row
            const int c0 = kGPS * (k2 - seg_gst), ncs = min(kGPS, seg_nc - c0);
            if (lane == 0) {
                mbar_arrive_expect_tx(fb, (uint32_t)ncs * NRB);
                for (int j = 0; j < ncs; ++j)
                    bulk_g2s(stg + j * G::GSLOT, seg_near + (size_t)(wgl() + (c0 + j) * nwl()) * NRB, NRB, fb);
            }
            return;
        }
        const int ng = min(kGPS, seg_n - kGPS * k2);
        const int2 *ids = seg_ids + kGPS * k2;
        if (!seg_v) {
            if (lane == 0) {
                mbar_arrive_expect_tx(fb, (uint32_t)ng * 2 * G::KB);
                if (GEN && a.inject == LOOPKV_INJECT_STALLED_STAGE && n == 0 && warp == 0 && blockIdx.x == 0)
                    return; // test hook: the stage's bytes never arrive, so its wait runs out
                for (int j = 0; j < ng; ++j) {
                    const int2 id = ids[j];
                    bulk_g2s(stg + j * G::GSLOT, seg_src + (uint64_t)(uint32_t)id.x * bstride, G::KB, fb);
                    bulk_g2s(stg + j * G::GSLOT + G::KB, seg_src + (uint64_t)(uint32_t)id.y * bstride, G::KB, fb);
                }
            }
            return;
        }
        if (lane == 0) { // V stage: value meta and hi planes (the lo planes of hot tokens: consume_v)
            mbar_arrive_expect_tx(fb, (uint32_t)ng * 2 * G::VB);
            for (int j = 0; j < ng; ++j) {
                const int2 id = ids[j];
                bulk_g2s(stg + j * G::GSLOT, seg_src + (uint64_t)(uint32_t)id.x * bstride, G::VB, fb);
                bulk_g2s(stg + j * G::GSLOT + G::VB, seg_src + (uint64_t)(uint32_t)id.y * bstride, G::VB, fb);
            }
        }
    };
    // Issue every stage numbered below `limit` that the sequence allows.  The K segment
    // of a row waits until the row is set up (the compute side sets up row r + 1 when it
    // starts scoring row r, see consume_k).
    auto pump = [&](int limit) {
        if (timed_out)
            return; // after a give-up nothing new is issued
        for (;;) {
            if (iss_k < seg_len) {
                if (iss_n >= limit || (NSC && !dep_ok && iss_k >= seg_gst)) // near rows: after the grid dependency
                    break;
                issue_stage(iss_n);
                ++iss_k;
                ++iss_n;
                continue;
            }
            const int nsig = iss_sig + 1;
            if (nsig >= 2 * nrows)
                break;
            bool nv;
            int nri;
            segment(nsig, nrows, seq, nv, nri);
            if (!nv && nri > setup_upto)
                break;
            iss_sig = nsig;
            iss_k = 0;
            load_segment();
        }
    };
    // ---------------------------------------------------------------- compute
    constexpr int SCR = scratch_bytes<D>();
    uint8_t *scr = sm.scr + warp * SCR;
    int prc_n = 0;
    auto wait_stage = [&](int n) {
        if (!timed_out && !mbar_wait(&full[n & smask], (n >> spw_log2) & 1, a.status, a.wait_ns)) {
            timed_out = true;
            drain_from = n;
        }
    };

    // K pass of the warp's groups of row ri; per-warp (max, sum) into stat.
    auto consume_k = [&](int ri) {
        // Set up row ri + 1 (and row 0 first).  Its slot (ri + 1) mod 3 last held row
        // ri - 2, whose values and lo planes were read in the previous iteration, so nothing
        // reads that slot any more.
        for (int r = ri == 0 ? 0 : ri + 1; r <= ri + 1 && r < nrows; ++r) {
            setup_row(r);
            setup_upto = r;
        }
        int32_t *srow = irow_of(ri);
        const int row = srow[IR_ROW], nown = srow[IR_N];
        float *sc = scores_of(ri);
        if (ri == 0) {
            // Prefetch the first stages, then wait for the previous grid of the stream: it may
            // have written q or the tails (an append), and it may read the outputs this grid
            // writes.  Lengths, block tables and pools were written by flush / ingest / reset
            // launches that the host does not let a decode overlap.
            pump(prc_n + spw);
            asm volatile("griddepcontrol.wait;" ::: "memory");
            dep_ok = true;
        }
        int tail = srow[IR_TAIL];
        if (tail < 0) { // near tokens and ring start (an append may just have written them)
            tail = a.tail_len[srow[IR_B]];
            int ws = a.win_start[srow[IR_B]];
            if (tail < 0 || tail > a.sink + a.wring || ws < 0 || ws >= a.wring) {
                if (lane == 0 && warp == 0)
                    atomicOr(a.status, LOOPKV_DEV_STATE);
                tail = 0;
                ws = 0;
            }
            __syncwarp();
            if (lane == 0) {
                srow[IR_TAIL] = tail;
                srow[IR_WS] = ws;
            }
            __syncwarp();
        }
        const int wg = wgl(), nw = nwl(); // near token j: warp j mod nw
        if (!nstream && tail > wg)
            prefetch_near<D, DT>(a, reinterpret_cast<const DT *>(a.tail) +
                                        ((int64_t)srow[IR_B] * 2 * a.H + srow[IR_H]) * a.near_cap * D,
                                 srow[IR_WS], wg, nw, tail, lane);
        // lane owns the channel quad 4*lane .. 4*lane+3 (lanes >= D/4 own none)
        const bool ownq = lane < G::NQ;
        float qreg[4];
        {
            const DT *qrow = reinterpret_cast<const DT *>(a.q) + (int64_t)row * D + 4 * lane;
#pragma unroll
            for (int i = 0; i < 4; ++i)
                qreg[i] = ownq ? to_f32(qrow[i]) : 0.f;
        }
        float mx = -INFINITY;
        const uint8_t *stg = ring;
        for (int k = 0; k < nown; ++k) {
            if (k % kGPS == 0) { // first group of a stage
                const int n = prc_n++;
                if (iss_n < n + spw)
                    pump(n + spw);
                wait_stage(n);
                stg = ring + (n & smask) * G::STAGE;
            }
            const uint8_t *st = stg + (k % kGPS) * G::GSLOT;
            float s2 = group_scores<BITS, D>(st, st + G::KB, scr, qreg, a.qscale, lane);
            if (GEN && k == 0 && crank == 0 && warp == 0 && lane < srow[IR_M0])
                s2 = -INFINITY; // before the attention window
            sc[k * 32 + lane] = s2;
            mx = fmaxf(mx, s2);
            __syncwarp();
        }
        // tail tokens (exact keys), dealt over every warp of the cluster: token j to warp
        // j mod (C * kWarps) of the cluster, so that no warp carries the whole tail
        float *tsc = sm.tscores + (ri & 1) * a.near_cap; // by near index (register path) or slot (chunks)
        float smx = -INFINITY; // largest sink score of this warp's near tokens
        const int ncw = nstream ? srow[IR_NC] : 0;
        if (nstream) { // this warp's chunks of the streamed near region
            const int ws = srow[IR_WS], hist = srow[IR_HIST];
            for (int c = 0; c < ncw; ++c) {
                if (c % kGPS == 0) {
                    const int n = prc_n++;
                    if (iss_n < n + spw)
                        pump(n + spw);
                    wait_stage(n);
                    stg = ring + (n & smask) * G::STAGE;
                }
                const DT *rows = reinterpret_cast<const DT *>(stg + (c % kGPS) * G::GSLOT);
                float p[NR];
#pragma unroll
                for (int r = 0; r < NR; ++r) { // lane: channels 4 lane .. 4 lane + 3 of every row
                    float k4[4] = {0.f, 0.f, 0.f, 0.f};
                    if (lane < D / 4)
                        load4f(rows + r * D + 4 * lane, k4);
                    p[r] = lane < D / 4 ? fmaf(qreg[0], k4[0], fmaf(qreg[1], k4[1], fmaf(qreg[2], k4[2], qreg[3] * k4[3])))
                                        : 0.f;
                }
#pragma unroll
                for (int o = 16; o > 0; o >>= 1)
#pragma unroll
                    for (int r = 0; r < NR; ++r)
                        p[r] += __shfl_xor_sync(0xFFFFFFFFu, p[r], o);
                const int slot0 = (wg + c * nw) * NR;
#pragma unroll
                for (int r = 0; r < NR; ++r) {
                    const int j = near_index(a, slot0 + r, ws, tail);
                    const float s2 = j >= 0 && (!GEN || near_attended(a, j, hist, tail)) ? p[r] * a.qscale : -INFINITY;
                    if (lane == 0)
                        tsc[slot0 + r] = s2;
                    mx = fmaxf(mx, s2);
                    if (j >= 0 && j < a.sink)
                        smx = fmaxf(smx, s2);
                }
                __syncwarp();
            }
        } else if (tail > wg) {
            const DT *kt = reinterpret_cast<const DT *>(a.tail) + ((int64_t)srow[IR_B] * 2 * a.H + srow[IR_H]) *
                                                                      a.near_cap * D;
            const int ws = srow[IR_WS], hist = srow[IR_HIST];
            for (int j0 = wg; j0 < tail; j0 += kNearBatch * nw) { // a batch of this warp's near tokens
                const DT *rows[kNearBatch];
#pragma unroll
                for (int u = 0; u < kNearBatch; ++u) {
                    const int j = j0 + u * nw;
                    rows[u] = j < tail && (!GEN || near_attended(a, j, hist, tail))
                                  ? kt + (int64_t)near_slot(a, j, ws) * D
                                  : nullptr;
                }
                float sb[kNearBatch];
                near_scores<D, DT>(rows, qreg, a.qscale, lane, sb);
#pragma unroll
                for (int u = 0; u < kNearBatch; ++u) {
                    const int j = j0 + u * nw;
                    if (j < tail) {
                        const float s2 = rows[u] != nullptr ? sb[u] : -INFINITY; // -inf: outside the window
                        if (lane == 0)
                            tsc[j] = s2;
                        mx = fmaxf(mx, s2);
                        if (j < a.sink)
                            smx = fmaxf(smx, s2);
                    }
                }
            }
            __syncwarp();
        }
        mx = warp_max(mx);
        float ls = 0.f;
        if (a.tau_mode == LOOPKV_TAU_ABS_PROB && mx != -INFINITY) {
            for (int k = 0; k < nown; ++k)
                ls += exp2f(sc[k * 32 + lane] - mx);
            if (nstream)
                for (int i = lane; i < ncw * NR; i += 32)
                    ls += exp2f(tsc[(wg + (i / NR) * nw) * NR + i % NR] - mx);
            else
                for (int j = wg + lane * nw; j < tail; j += 32 * nw)
                    ls += exp2f(tsc[j] - mx);
            ls = warp_sum(ls);
        }
        if (lane == 0) {
            float *stw = sm.stat + (ri % 3) * kWarps * 4;
            stw[4 * warp] = mx;
            stw[4 * warp + 1] = ls;
            stw[4 * warp + 2] = smx;
        }
    };

    // V pass of the warp's groups of row ri, then the CTA partial (o, l) into part.
    //
    // Per group, lane t takes token t: weight w = 2^(s - m), the zero terms, W_g = w * scale_g
    // and, with F from the
    // exact maximum of W over the group, the 15-bit fixed-point I_g = round(W_g 2^F) as the
    // low bits of W_g 2^F + 2^23.  Through a padded shared transpose, lane (t8, g) then packs
    // the two byte digits of I_g of the 4 tokens of token quad t8 into a record
    // {d0, d1, hot-byte mask}.  Consumer lane vk owns channel quad vk and, for every token
    // quad, merges its hi and lo plane words into 4-bit codes (lo bits kept for hot tokens
    // only), unpacks the four channels' codes of the four tokens with one AND each and
    // accumulates code * digit over tokens with dp4a, exact in int32; the group's sum goes
    // to fp32 exactly.
    auto consume_v = [&](int ri, float m2, float thr2) {
        const int32_t *srow = irow_of(ri);
        const int nown = srow[IR_N], tail = srow[IR_TAIL];
        if (!nstream && tail > wgl()) // this warp's near values, read after its groups
            prefetch_near<D, DT>(a, reinterpret_cast<const DT *>(a.tail) +
                                        ((int64_t)(srow[IR_B] * 2 + 1) * a.H + srow[IR_H]) * a.near_cap * D,
                                 srow[IR_WS], (int)crank * kWarps + warp, (int)C * kWarps, tail, lane);
        const float *sc = scores_of(ri);
        constexpr int NCG = G::NCG;
        constexpr int YS = 40; // word stride of a group's row in the transpose (conflict-free both ways)
        const int pt8 = lane / NCG, pg = lane % NCG;  // record lane: token quad, channel group
        const bool pv = pt8 < 8;
        constexpr int BPL = G::NQ == 32 ? 2 : 1;      // blocks of a group per consumer lane
        const int vk = lane % G::NQ, vg = vk >> 3;     // consumer lane: channel quad and its group
        const int vb0 = G::NQ == 32 ? 0 : lane / G::NQ;
        // [NCG][YS] fixed-point words of the tokens; record (g, t8) is then written in place
        // over words 4 t8 .. 4 t8 + 3 of row g, the only words its lane reads
        uint32_t *ybuf = reinterpret_cast<uint32_t *>(scr);
        float *fsit = reinterpret_cast<float *>(ybuf + NCG * YS);
        float facc[4] = {0.f, 0.f, 0.f, 0.f};
        float zl[NCG];
#pragma unroll
        for (int g = 0; g < NCG; ++g)
            zl[g] = 0.f;
        float lsum = 0.f;
        float run_v = thr2; // streaming rule: running maximum from the seed
        const uint8_t *lob = a.lo + (size_t)srow[IR_H] * G::LOB;
        const int2 *gids = reinterpret_cast<const int2 *>(ids_of(ri));
        // Hot tokens of group k (bit t: token t).  The streaming rule's running maximum takes
        // each group's largest score before the group's tokens are tested, in group order.
        auto hot_mask = [&](int k) {
            const float s2 = sc[k * 32 + lane];
            float thr_k = thr2;
            if (stream) {
                run_v = fmaxf(run_v, warp_max_f(s2));
                thr_k = run_v + ltau;
            }
            return __ballot_sync(0xFFFFFFFFu, s2 >= thr_k);
        };
        // Lo planes of the hot token quads of group k into the group's slot of ring stage n,
        // one group ahead of its use.  A quad (4 tokens x D channels x 2 bits = D bytes) with a
        // hot token is copied whole in 16-byte pieces, each lane its own; then one commit
        // group per call (empty when nothing is hot).  The slot is free: its previous stage was
        // consumed before the current one.
        auto fetch_lo = [&](int k, int n, uint32_t hm) {
            if (k < nown && hm != 0u) {
                uint8_t *dst = ring + (n & smask) * G::STAGE + (k % kGPS) * G::GSLOT + 2 * G::VB;
                const int2 id = gids[k];
                constexpr int P = D / 16; // 16-byte pieces of a quad
#pragma unroll
                for (int j = 0; j < 8 * P / 32; ++j) {
                    const int idx = lane + 32 * j, q = idx / P, off = (q & 3) * D + 16 * (idx % P);
                    if ((hm >> (4 * q)) & 0xFu) {
                        const int blk = q >> 2;
                        const uint32_t bid = (uint32_t)(blk ? id.y : id.x);
                        cp_async16(dst + blk * G::LOB + off, lob + (uint64_t)bid * lstride + off);
                    }
                }
            }
            cp_async_commit();
        };
        uint32_t hm_next = nown > 0 ? hot_mask(0) : 0u;
        fetch_lo(0, prc_n, hm_next); // group 0 lies in the next stage to be consumed
        const uint8_t *stg = ring;
        for (int k = 0; k < nown; ++k) {
            const bool first = k % kGPS == 0; // first group of a stage
            int n = 0;
            if (first) {
                n = prc_n++;
                if (iss_n < n + spw)
                    pump(n + spw);
            }
            const float s2l = sc[k * 32 + lane];
            const float wl = ex2(s2l - m2);
            const uint32_t hm = hm_next;
            const bool hotl = (hm >> lane) & 1u;
            if (k + 1 < nown)
                hm_next = hot_mask(k + 1);
            // group k + 1 lies in the next stage (prc_n) or in this one (prc_n - 1)
            fetch_lo(k + 1, (k + 1) % kGPS == 0 ? prc_n : prc_n - 1, hm_next);
            if (GEN && a.s_bitmap && lane == 0) // refine set of the debug entry point, one bit per token
                a.s_bitmap[(int64_t)srow[IR_ROW] * a.bitmap_words + srow[IR_G0] + (int)crank +
                           (warp + k * kWarps) * (int)C] = hm;
            lsum += wl;
            if (first) {
                wait_stage(n);
                stg = ring + (n & smask) * G::STAGE;
            }
            const uint8_t *st = stg + (k % kGPS) * G::GSLOT;
            // ---- token lane: zero terms, fixed-point weights
            {
                const uint8_t *vm = st + (lane >> 4) * G::VB + (lane & 15) * 4; // (scale, zero) of group g at + 64 g
                float W[NCG], wmax = 0.f;
#pragma unroll
                for (int g = 0; g < NCG; ++g) {
                    const float2 m = __half22float2(*reinterpret_cast<const __half2 *>(vm + 64 * g));
                    zl[g] = fmaf(wl, hotl ? m.y : fmaf(1.5f, m.x, m.y), zl[g]);
                    W[g] = wl * m.x;
                    wmax = fmaxf(wmax, W[g]);
                }
                wmax = warp_max_f(wmax);
                // I < 2^15 + 1 with F = 14 - E (E = exponent of the maximum), capped so that
                // 2^F and 2^-F stay normal: two byte digits
                int F = 14 - ((int)(__float_as_uint(wmax) >> 23) - 127);
                F = F > 126 ? 126 : F;
                const float fs = __int_as_float((F + 127) << 23);
#pragma unroll
                for (int g = 0; g < NCG; ++g)
                    ybuf[g * YS + lane] = __float_as_uint(fmaf(W[g], fs, 8388608.f));
                if (lane == 0)
                    *fsit = __int_as_float((127 - F) << 23);
            }
            __syncwarp();
            // ---- record lane (t8, g): byte digits of the 4 tokens of quad t8, hot-byte mask
            if (pv) {
                const uint4 y = *reinterpret_cast<const uint4 *>(ybuf + pg * YS + 4 * pt8);
                const uint32_t t01 = __byte_perm(y.x, y.y, 0x5140), t23 = __byte_perm(y.z, y.w, 0x5140);
                // bit b of the quad's 4 hot bits to bit 8b+7, then each byte takes its top bit
                const uint32_t hb = byte_signs(((hm >> (4 * pt8)) & 0xFu) * 0x10204080u);
                reinterpret_cast<uint4 *>(ybuf + pg * YS)[pt8] =
                    make_uint4(__byte_perm(t01, t23, 0x5410), __byte_perm(t01, t23, 0x7632), hb, 0u);
            }
            cp_async_wait<1>(); // this lane's lo copies of group k (those of group k + 1 may fly)
            __syncwarp();       // ... and every other lane's
            // ---- accumulate: channel quad vk, dp4a over the tokens of each token quad
            VSums acc;
#pragma unroll
            for (int bb = 0; bb < BPL; ++bb) {
                const int blk = vb0 + bb;
                const uint4 h4 = *reinterpret_cast<const uint4 *>(st + blk * G::VB + G::VMETA + 16 * vk);
                const uint32_t hwv[4] = {h4.x, h4.y, h4.z, h4.w};
                const uint8_t *lop = st + 2 * G::VB + blk * G::LOB + 4 * vk;
                const uint4 *rq = reinterpret_cast<const uint4 *>(ybuf + vg * YS) + 4 * blk;
#pragma unroll
                for (int tau = 0; tau < 4; ++tau) {
                    const uint4 rc = rq[tau];
                    // lo words exist for quads with a hot token; keep the hot tokens' bits
                    const uint32_t lw = *reinterpret_cast<const uint32_t *>(lop + tau * D) & rc.z;
                    acc.add<BITS>(hwv[tau], lw, rc.x, rc.y);
                }
            }
            acc.finish(*fsit, facc);
            __syncwarp();
        }
        // zero terms: lane ends with the warp's sum of zl[lane % NCG] (reduce-scatter over
        // the group bits, then a sum over the other lanes); lane vk takes its group's from lane vg
#pragma unroll
        for (int s2 = 0; (1 << s2) < NCG; ++s2) {
            const int off = 1 << s2, len = NCG >> (s2 + 1);
            const bool up = (lane & off) != 0;
#pragma unroll
            for (int m = 0; m < len; ++m) {
                const float send = up ? zl[2 * m] : zl[2 * m + 1];
                const float keep = up ? zl[2 * m + 1] : zl[2 * m];
                zl[m] = keep + __shfl_xor_sync(0xFFFFFFFFu, send, off);
            }
        }
        float zsum = zl[0];
#pragma unroll
        for (int off = NCG; off < 32; off <<= 1)
            zsum += __shfl_xor_sync(0xFFFFFFFFu, zsum, off);
        const float zacc = __shfl_sync(0xFFFFFFFFu, zsum, vg);
        lsum = warp_sum(lsum);
        if (BPL == 1) // D = 64: the two halves of the warp read the two blocks
#pragma unroll
            for (int i = 0; i < 4; ++i)
                facc[i] += __shfl_xor_sync(0xFFFFFFFFu, facc[i], 16);
        __syncwarp();
        float *red = reinterpret_cast<float *>(scr); // end of the V pass: the warp's partial o, l
        if (lane < G::NQ)
            *reinterpret_cast<float4 *>(red + 4 * vk) =
                make_float4(facc[0] + zacc, facc[1] + zacc, facc[2] + zacc, facc[3] + zacc);
        if (lane == 0)
            red[D] = lsum;
        __syncwarp();
        const int wg = wgl(), nw = nwl();
        if (nstream) { // this warp's chunks of the streamed near region; scores by slot from the K pass
            const int ncw = srow[IR_NC];
            const float *tsc = sm.tscores + (ri & 1) * a.near_cap;
            float tl = 0.f, acc[4] = {0.f, 0.f, 0.f, 0.f}; // lane: channels 4 lane .. 4 lane + 3
            for (int c = 0; c < ncw; ++c) {
                if (c % kGPS == 0) {
                    const int n = prc_n++;
                    if (iss_n < n + spw)
                        pump(n + spw);
                    wait_stage(n);
                    stg = ring + (n & smask) * G::STAGE;
                }
                const DT *rows = reinterpret_cast<const DT *>(stg + (c % kGPS) * G::GSLOT);
                const int slot0 = (wg + c * nw) * NR;
#pragma unroll
                for (int r = 0; r < NR; ++r) {
                    const float s2 = tsc[slot0 + r];
                    if (s2 != -INFINITY) { // warp-uniform: empty slots and tokens outside a window are -inf
                        const float w = exp2f(s2 - m2);
                        tl += w;
                        if (lane < D / 4) {
                            float v4[4];
                            load4f(rows + r * D + 4 * lane, v4);
#pragma unroll
                            for (int i = 0; i < 4; ++i)
                                acc[i] = fmaf(w, v4[i], acc[i]);
                        }
                    }
                }
                __syncwarp();
            }
            if (lane < D / 4)
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    red[4 * lane + i] += acc[i];
            __syncwarp();
            if (lane == 0)
                red[D] += tl;
        } else if (tail > wg) { // this warp's tail tokens (see consume_k), exact values
            const int b = srow[IR_B], h = srow[IR_H];
            const float *tsc = sm.tscores + (ri & 1) * a.near_cap;
            const DT *vt0 = reinterpret_cast<const DT *>(a.tail) + ((int64_t)(b * 2 + 1) * a.H + h) * a.near_cap * D;
            const int ws = srow[IR_WS];
            float tl = 0.f, acc[D / 32];
#pragma unroll
            for (int c4 = 0; c4 < D / 32; ++c4)
                acc[c4] = 0.f;
            for (int t0 = wg; t0 < tail; t0 += kNearBatch * nw) { // a batch of tokens, loads first
                float w[kNearBatch], v[kNearBatch][D / 32];
#pragma unroll
                for (int u = 0; u < kNearBatch; ++u) {
                    const int t = t0 + u * nw;
                    w[u] = 0.f;
#pragma unroll
                    for (int c4 = 0; c4 < D / 32; ++c4)
                        v[u][c4] = 0.f;
                    if (t < tail) { // tokens outside a sliding window have score -inf: weight 0
                        const DT *vt = vt0 + (int64_t)near_slot(a, t, ws) * D;
                        w[u] = exp2f(tsc[t] - m2);
#pragma unroll
                        for (int c4 = 0; c4 < D / 32; ++c4)
                            v[u][c4] = to_f32(vt[lane + 32 * c4]);
                    }
                }
#pragma unroll
                for (int u = 0; u < kNearBatch; ++u) {
                    tl += w[u];
#pragma unroll
                    for (int c4 = 0; c4 < D / 32; ++c4)
                        acc[c4] = fmaf(w[u], v[u][c4], acc[c4]);
                }
            }
#pragma unroll
            for (int c4 = 0; c4 < D / 32; ++c4)
                red[lane + 32 * c4] += acc[c4];
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

    // CTA `crank` writes channels [crank*per, min(D, (crank+1)*per)) of row ri, per =
    // ceil(D / C), summing the partials of every CTA of the cluster.
    auto merge = [&](int ri, float m2) {
        const int row = row_of(ri);
        const float *part = sm.part + (ri & 1) * (D + 1);
        const int per = (D + (int)C - 1) / (int)C;
        const int c = (int)crank * per + (int)threadIdx.x;
        if ((int)threadIdx.x < per && c < D) {
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

    // exact rules: the row threshold; streaming rule: the seed (the largest sink score)
    auto row_threshold = [&](float m, float l, float m0) {
        if (stream)
            return m0;
        return a.tau_mode == LOOPKV_TAU_ABS_PROB ? m + log2f(a.tau * l) : m + ltau;
    };

    // Overlapped order: iteration i scores row i and reads the values of row i - 1; barrier
    // i (arrived after the iteration) publishes the maxima of row i and the partials of row
    // i - 1.  Sequential order (one score buffer): iteration i scores row i, passes barrier
    // i (maxima of row i, partials of row i - 1), merges row i - 1 and reads the values of
    // row i.  Each phase has a single call site (keeps the kernel's code small).
    float m_prev = 0.f;
    for (int i = 0; i <= nrows; ++i) {
        if (i < nrows)
            consume_k(i);
        if (seq)
            cluster_arrive(); // barrier i
        if (seq || i > 0) {
            cluster_wait(); // barrier i (sequential) or i - 1
            const int mr = seq ? i - 1 : i - 2, vr = seq ? i : i - 1;
            if (mr >= 0)
                merge(mr, m_prev);
            if (vr < nrows) {
                float m2, l2, m0;
                cluster_row_stats(sm.stat + (vr % 3) * kWarps * 4, C, lane, m2, l2, m0);
                const float thr2 = row_threshold(m2, l2, m0);
                consume_v(vr, m2, thr2);
                m_prev = m2;
            }
        }
        if (!seq)
            cluster_arrive(); // barrier i
    }
    if (!seq) {
        cluster_wait(); // partials of the last row
        if (nrows > 0)
            merge(nrows - 1, m_prev);
    }
    if (timed_out) // copies issued before the give-up must land before the shared memory is freed
        for (int n = drain_from; n < iss_n; ++n)
            mbar_wait(&full[n & smask], (n >> spw_log2) & 1, a.status, a.wait_ns);
    cp_async_wait<0>(); // the last (possibly empty) lo commit group of this thread
    cluster_arrive(); // remote reads done
    cluster_wait();
}

// ---------------------------------------------------------------------------------------
// Single-pass reader for rows whose refine set does not depend on the row maximum: 4-bit
// sources read with tau <= 0 (every lo plane is read) and 2-bit sources (no lo plane, S
// empty).  For these, softmax with a running maximum per warp (rescaling the warp's sums
// whenever it grows) gives the result of the exact-maximum reader up to rounding, so a
// group's keys and values are read from one stage and its scores stay in registers: no
// score buffer, no exchange of maxima inside a row, one merge of (m, l, o) per row over
// the warps and CTAs of the cluster.  The smaller shared footprint lets 5 CTAs share an SM.
//
// A stage holds one 32-token group: the whole head region of both of its blocks (key
// codes and meta, value meta, hi plane) and, for 4-bit sources, both lo regions.
template <int BITS, int D> struct Geo1 {
    using G = Geo<BITS, D>;
    static constexpr int STAGE = (2 * G::HM + 2 * G::LOB + 127) / 128 * 128;
    static constexpr int LOFF = 2 * G::HM; // lo regions of the stage
};

struct SmemLayout1 {
    int full, scr, part, ids, irow, order, total;
};

// One row slot (block ids, row fields) per warp: the next row is set up once the current
// row's stages are all issued.  A warp's maximum sits in its scratch after its partial
// (word D + 1).  CTA partials (o[D], l, m) by row parity (see the barrier note in the
// kernel).
constexpr int kFields1 = 9;
constexpr int I1_G0 = 5, I1_M0 = 6, I1_HIST = 7; // fields after IR_ROW .. IR_TAIL (see decode_kernel)
constexpr int I1_NC = 8;                          // near-region chunks read by this warp (streamed)

// Near rows per chunk of the single-pass reader: a chunk's key rows and value rows share one
// ring stage.
template <int BITS, int D, typename DT> __host__ __device__ constexpr int near_chunk_rows1()
{
    return 2 * 8 * D * (int)sizeof(DT) <= Geo1<BITS, D>::STAGE   ? 8
           : 2 * 4 * D * (int)sizeof(DT) <= Geo1<BITS, D>::STAGE ? 4
                                                                  : 2;
}

template <int BITS, int D> __host__ __device__ constexpr SmemLayout1 smem_layout1(int spw, int capw)
{
    SmemLayout1 L{};
    int o = kWarps * spw * Geo1<BITS, D>::STAGE;
    L.full = o;
    o = align16(o + kWarps * spw * 8);
    L.scr = o;
    o = align16(o + kWarps * scratch_bytes<D>());
    L.part = o;
    o = align16(o + 2 * (D + 2) * 4);
    L.ids = o;
    o = align16(o + kWarps * 2 * capw * 4);
    L.irow = o;
    o = align16(o + kWarps * kFields1 * 4);
    L.order = o;
    o = align16(o + kMaxOrder * 4);
    L.total = o;
    return L;
}

template <int BITS, int D> bool layout1_ok(int spw, int capw)
{
    const SmemLayout1 L = smem_layout1<BITS, D>(spw, capw);
    const int offs[] = {L.full, L.scr, L.part, L.ids, L.irow, L.order};
    int prev = kWarps * spw * Geo1<BITS, D>::STAGE;
    for (int o : offs) {
        if (o % 16 || o < prev)
            return false;
        prev = o;
    }
    // the request lengths are ranked in the warps' scratch at kernel start; a warp's
    // partial and maximum take D + 2 words of its scratch; id pairs are read as int2
    return L.total >= prev && (spw & (spw - 1)) == 0 && kWarps * scratch_bytes<D>() >= kMaxOrder * 4 &&
           scratch_bytes<D>() >= (D + 2) * 4 && (2 * capw * 4) % 8 == 0 && (Geo1<BITS, D>::STAGE % 128) == 0 &&
           (Geo<BITS, D>::HM % 16) == 0 && (Geo<BITS, D>::LOB % 16) == 0;
}

// Running state of one warp over its groups of a row (single-pass reader): maximum m
// (log2 units), l = sum of 2^(s - m), the lane's channel-quad sums o of 2^(s - m) * s_v *
// code, and the lane-token's zero terms z per 32-channel group (also relative to 2^m).
template <int D> struct Run1 {
    float m, l;
    float o[4];
    float z[D / 32];
};

template <int D> __device__ __forceinline__ void run1_init(Run1<D> &r)
{
    r.m = -INFINITY;
    r.l = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i)
        r.o[i] = 0.f;
#pragma unroll
    for (int g = 0; g < D / 32; ++g)
        r.z[g] = 0.f;
}

// One 32-token group: head regions of its two blocks at st and st + HM, their lo regions
// at lo (4-bit).  Exact integer key dot products (the key pass of decode_kernel), the
// running-maximum update, then the value pass of decode_kernel with every token refined
// (4-bit source) or plain 2-bit codes.  scr: the warp's scratch.
template <int BITS, int D>
__device__ __forceinline__ void run1_group(const uint8_t *st, const uint8_t *lo, uint8_t *scr, const float (&qreg)[4],
                                           const float qscale, const int lane, Run1<D> &r, const int masked = 0)
{
    using G = Geo<BITS, D>;
    constexpr int NCG = G::NCG;
    constexpr int YS = 40;
    const int pt8 = lane / NCG, pg = lane % NCG;
    const bool pv = pt8 < 8;
    constexpr int BPL = G::NQ == 32 ? 2 : 1;
    const int vk = lane % G::NQ, vg = vk >> 3;
    const int vb0 = G::NQ == 32 ? 0 : lane / G::NQ;
    uint32_t *ybuf = reinterpret_cast<uint32_t *>(scr);
    float *fsit = reinterpret_cast<float *>(ybuf + NCG * YS);
    float s2l = group_scores<BITS, D>(st, st + G::HM, scr, qreg, qscale, lane); // score of token `lane`
    if (lane < masked)
        s2l = -INFINITY; // before a sliding attention window
    // ---- running maximum (warp-uniform): rescale the warp's sums when it grows
    const float mg = warp_max_f(s2l);
    if (mg > r.m) {
        const float f = ex2(r.m - mg); // 0 at the first group
#pragma unroll
        for (int i = 0; i < 4; ++i)
            r.o[i] *= f;
#pragma unroll
        for (int g = 0; g < NCG; ++g)
            r.z[g] *= f;
        r.l *= f;
        r.m = mg;
    }
    const float wl = ex2(s2l - r.m);
    r.l += wl;
    __syncwarp(); // the key digit records are read: the scratch takes the value weights
    // ---- values: decode_kernel's value pass with every token hot
    {
        const uint8_t *vm = st + (lane >> 4) * G::HM + G::KB + (lane & 15) * 4; // (scale, zero) of group g at + 64 g
        float W[NCG], wmax = 0.f;
#pragma unroll
        for (int g = 0; g < NCG; ++g) {
            const float2 m = __half22float2(*reinterpret_cast<const __half2 *>(vm + 64 * g));
            r.z[g] = fmaf(wl, m.y, r.z[g]);
            W[g] = wl * m.x;
            wmax = fmaxf(wmax, W[g]);
        }
        wmax = warp_max_f(wmax);
        // I = round(W 2^F) < 2^15 + 1 with F = 14 - E: two byte digits (the 2^-15 relative
        // step of a weight is far below the fp32 rounding of the sums it enters)
        int Fv = 14 - ((int)(__float_as_uint(wmax) >> 23) - 127);
        Fv = Fv > 126 ? 126 : Fv;
        const float fv = __int_as_float((Fv + 127) << 23);
#pragma unroll
        for (int g = 0; g < NCG; ++g)
            ybuf[g * YS + lane] = __float_as_uint(fmaf(W[g], fv, 8388608.f));
        if (lane == 0)
            *fsit = __int_as_float((127 - Fv) << 23);
    }
    __syncwarp();
    if (pv) { // record lane (t8, g): the two byte digits of the 4 tokens of quad t8
        const uint4 y = *reinterpret_cast<const uint4 *>(ybuf + pg * YS + 4 * pt8);
        const uint32_t t01 = __byte_perm(y.x, y.y, 0x5140), t23 = __byte_perm(y.z, y.w, 0x5140);
        *reinterpret_cast<uint2 *>(ybuf + pg * YS + 4 * pt8) =
            make_uint2(__byte_perm(t01, t23, 0x5410), __byte_perm(t01, t23, 0x7632));
    }
    __syncwarp();
    VSums acc;
#pragma unroll
    for (int bb = 0; bb < BPL; ++bb) {
        const int blk = vb0 + bb;
        const uint4 h4 = *reinterpret_cast<const uint4 *>(st + blk * G::HM + G::KB + G::VMETA + 16 * vk);
        const uint32_t hwv[4] = {h4.x, h4.y, h4.z, h4.w};
        const uint8_t *lop = lo + blk * G::LOB + 4 * vk;
        const uint32_t *rq = ybuf + vg * YS + 16 * blk; // record of token quad 4 blk + tau at + 4 tau
#pragma unroll
        for (int tau = 0; tau < 4; ++tau) {
            const uint2 rc = *reinterpret_cast<const uint2 *>(rq + 4 * tau);
            const uint32_t lw = BITS == 4 ? *reinterpret_cast<const uint32_t *>(lop + tau * D) : 0u;
            acc.add<BITS>(hwv[tau], lw, rc.x, rc.y);
        }
    }
    acc.finish(*fsit, r.o);
    __syncwarp();
}

// End of a row for one warp: its partial o (zero terms added) into red[0 .. D-1] and l into
// red[D], relative to 2^r.m.
template <int BITS, int D> __device__ __forceinline__ void run1_finish(Run1<D> &r, float *red, const int lane)
{
    using G = Geo<BITS, D>;
    constexpr int NCG = G::NCG;
    constexpr int BPL = G::NQ == 32 ? 2 : 1;
    const int vk = lane % G::NQ, vg = vk >> 3;
    // the warp's zero terms (reduce-scatter as in decode_kernel), sums and partial o, l
#pragma unroll
    for (int s2 = 0; (1 << s2) < NCG; ++s2) {
        const int off = 1 << s2, len = NCG >> (s2 + 1);
        const bool up = (lane & off) != 0;
#pragma unroll
        for (int m = 0; m < len; ++m) {
            const float send = up ? r.z[2 * m] : r.z[2 * m + 1];
            const float keep = up ? r.z[2 * m + 1] : r.z[2 * m];
            r.z[m] = keep + __shfl_xor_sync(0xFFFFFFFFu, send, off);
        }
    }
    float zsum = r.z[0];
#pragma unroll
    for (int off = NCG; off < 32; off <<= 1)
        zsum += __shfl_xor_sync(0xFFFFFFFFu, zsum, off);
    const float zacc = __shfl_sync(0xFFFFFFFFu, zsum, vg);
    r.l = warp_sum(r.l);
    if (BPL == 1)
#pragma unroll
        for (int i = 0; i < 4; ++i)
            r.o[i] += __shfl_xor_sync(0xFFFFFFFFu, r.o[i], 16);
    __syncwarp();
    if (lane < G::NQ)
        *reinterpret_cast<float4 *>(red + 4 * vk) =
            make_float4(r.o[0] + zacc, r.o[1] + zacc, r.o[2] + zacc, r.o[3] + zacc);
    if (lane == 0)
        red[D] = r.l;
    __syncwarp();
}

// Tail tokens j0, j0 + stride, ... < n (exact keys kt [*][D], values vt0 [*][D]) folded into the
// warp's partial red (o[D], l relative to 2^r.m), raising r.m (and rescaling red) when a
// tail score exceeds it.
template <int D, typename DT>
__device__ __forceinline__ void run1_tail(Run1<D> &r, float *red, const int lane, const float (&qreg)[4],
                                          const DecodeArgs &a, const DT *kt, const DT *vt0, const int ws,
                                          const int hist, const int j0, const int stride, const int n)
{
    for (int jb = j0; jb < n; jb += kNearBatch * stride) { // a batch of tokens: keys and values loaded first
        const DT *krow[kNearBatch];
        float v[kNearBatch][D / 32];
#pragma unroll
        for (int u = 0; u < kNearBatch; ++u) {
            const int j = jb + u * stride;
            const bool att = j < n && near_attended(a, j, hist, n);
            const int slot = att ? near_slot(a, j, ws) : 0;
            krow[u] = att ? kt + (int64_t)slot * D : nullptr;
#pragma unroll
            for (int c4 = 0; c4 < D / 32; ++c4)
                v[u][c4] = att ? to_f32(vt0[(int64_t)slot * D + lane + 32 * c4]) : 0.f;
        }
        float sb[kNearBatch];
        near_scores<D, DT>(krow, qreg, a.qscale, lane, sb);
#pragma unroll
        for (int u = 0; u < kNearBatch; ++u) {
            if (krow[u] == nullptr)
                continue; // warp-uniform
            const float s2 = sb[u];
            if (s2 > r.m) { // warp-uniform
                const float f = ex2(r.m - s2);
                for (int c = lane; c <= D; c += 32)
                    red[c] *= f;
                r.m = s2;
            }
            const float w = ex2(s2 - r.m);
#pragma unroll
            for (int c4 = 0; c4 < D / 32; ++c4)
                red[lane + 32 * c4] = fmaf(w, v[u][c4], red[lane + 32 * c4]);
            if (lane == 0)
                red[D] += w;
        }
    }
    __syncwarp();
}

// One chunk of NR near rows of a streamed near region (keys at kr, values at vr, physical slots
// slot0 ..): exact scores, the running-maximum update of the single-pass reader, and the rows'
// values added to the warp's sums (lane vk < D/4: channels 4 vk .. 4 vk + 3; l in lane 0).  Empty
// slots and tokens outside a sliding window score -inf and add nothing.
template <int D, typename DT, int NR, bool GEN>
__device__ __forceinline__ void run1_near_chunk(Run1<D> &r, const DT *kr, const DT *vr, const float (&qreg)[4],
                                                const DecodeArgs &a, const int slot0, const int ws, const int nnear,
                                                const int hist, const int lane)
{
    float p[NR];
#pragma unroll
    for (int u = 0; u < NR; ++u) {
        float k4[4] = {0.f, 0.f, 0.f, 0.f};
        if (lane < D / 4)
            load4f(kr + u * D + 4 * lane, k4);
        p[u] = lane < D / 4 ? fmaf(qreg[0], k4[0], fmaf(qreg[1], k4[1], fmaf(qreg[2], k4[2], qreg[3] * k4[3]))) : 0.f;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
#pragma unroll
        for (int u = 0; u < NR; ++u)
            p[u] += __shfl_xor_sync(0xFFFFFFFFu, p[u], o);
    float mc = -INFINITY;
#pragma unroll
    for (int u = 0; u < NR; ++u) {
        const int j = near_index(a, slot0 + u, ws, nnear);
        p[u] = j >= 0 && (!GEN || near_attended(a, j, hist, nnear)) ? p[u] * a.qscale : -INFINITY;
        mc = fmaxf(mc, p[u]);
    }
    if (mc > r.m) { // warp-uniform: rescale the warp's sums to the new maximum
        const float f = ex2(r.m - mc);
#pragma unroll
        for (int i = 0; i < 4; ++i)
            r.o[i] *= f;
#pragma unroll
        for (int g = 0; g < D / 32; ++g)
            r.z[g] *= f;
        r.l *= f;
        r.m = mc;
    }
#pragma unroll
    for (int u = 0; u < NR; ++u) {
        if (p[u] == -INFINITY)
            continue; // warp-uniform
        const float w = ex2(p[u] - r.m);
        if (lane == 0)
            r.l += w;
        if (lane < D / 4) {
            float v4[4];
            load4f(vr + u * D + 4 * lane, v4);
#pragma unroll
            for (int i = 0; i < 4; ++i)
                r.o[i] = fmaf(w, v4[i], r.o[i]);
        }
    }
}

template <int BITS, int D, typename DT, int MINCTA, int VAR> // VAR: as for decode_kernel
__global__ void __launch_bounds__(kThreads, MINCTA) decode_kernel_1p(const DecodeArgs a, const int spw_log2)
{
    constexpr bool GEN = VAR == 2;
    constexpr bool NSC = VAR >= 1; // the streamed near path is compiled in
    constexpr int NR = near_chunk_rows1<BITS, D, DT>();
    constexpr uint32_t NRB = (uint32_t)(NR * D * sizeof(DT)); // bytes of a chunk's keys (and of its values)
    using G = Geo<BITS, D>;
    using G1 = Geo1<BITS, D>;
    extern __shared__ __align__(128) uint8_t smem_raw[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int spw = 1 << spw_log2, smask = spw - 1;
    const uint32_t crank = cluster_ctarank(), C = cluster_nctarank();
    const int cid = blockIdx.x / (int)C, ncl = gridDim.x / (int)C;
    const int capw = (a.cap_groups + kWarps - 1) / kWarps;
    const SmemLayout1 LY = smem_layout1<BITS, D>(spw, capw);
    constexpr int SCR = scratch_bytes<D>();
    uint64_t *fullb = reinterpret_cast<uint64_t *>(smem_raw + LY.full);
    uint8_t *scr_all = smem_raw + LY.scr;
    float *parts = reinterpret_cast<float *>(smem_raw + LY.part);
    int32_t *order = reinterpret_cast<int32_t *>(smem_raw + LY.order);
    const uint32_t bstride = (uint32_t)a.H * G::HM, lstride = (uint32_t)a.H * G::LOB;

    asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); // as in decode_kernel
    if (lane == 0)
        for (int i = 0; i < spw; ++i)
            mbar_init(&fullb[warp * spw + i], 1);
    fence_mbar_init();
    // row schedule of decode_kernel; the lengths are ranked in the scratch
    const int nreq = a.rows / a.H;
    bool ordered = false;
    if (nreq <= kMaxOrder) {
        int32_t *lens = reinterpret_cast<int32_t *>(scr_all);
        for (int b = threadIdx.x; b < nreq; b += kThreads)
            lens[b] = a.hist_len[b];
        __syncthreads();
        for (int b = threadIdx.x; b < nreq; b += kThreads) {
            const int lb = lens[b];
            int rank = 0;
            for (int b2 = 0; b2 < nreq; ++b2) {
                const int l2 = lens[b2];
                rank += (l2 > lb) || (l2 == lb && b2 < b);
            }
            order[rank] = b;
        }
        for (int b = 1; b < nreq; ++b)
            ordered |= lens[b] != lens[0];
    }
    __syncthreads(); // the scratch is free again
    const int full_passes = a.rows / ncl, rem = a.rows % ncl;
    const int nrows = !ordered ? (cid < a.rows ? (a.rows - 1 - cid) / ncl + 1 : 0)
                               : full_passes + ((full_passes & 1) ? (cid >= ncl - rem) : (cid < rem));
    auto row_of = [&](int ri) {
        if (!ordered)
            return cid + ri * ncl;
        const int p = ri * ncl + ((ri & 1) ? ncl - 1 - cid : cid);
        const int q = p / a.H;
        return order[q] * a.H + (p - q * a.H);
    };

    uint8_t *ring = smem_raw + warp * spw * G1::STAGE;
    uint64_t *full = fullb + warp * spw;
    uint8_t *scr = scr_all + warp * SCR;
    int32_t *ids = reinterpret_cast<int32_t *>(smem_raw + LY.ids) + warp * 2 * capw;
    int32_t *irow = reinterpret_cast<int32_t *>(smem_raw + LY.irow) + warp * kFields1;

    // ---------------------------------------------------------------- issuing
    int iss_n = 0, iss_row = -1, iss_k = 0, seg_n = 0, setup_upto = -1;
    int seg_groups = 0;                       // group stages of the issuing row, then its near chunks
    const uint8_t *seg_src = nullptr, *seg_lo = nullptr;
    const uint8_t *seg_near = nullptr;        // near region (keys; values follow H rows on) of the row
    // a near region beyond a 32-token tail streams through the ring (see decode_kernel)
    const bool nstream = NSC && a.near_cap > 32;
    bool dep_ok = false;                      // the previous grid of the stream has finished
    bool timed_out = false; // as in decode_kernel: no waits or copies after a give-up, then a drain
    int drain_from = 0;
    // row parameters, validation and the warp's block ids of row ri (as in decode_kernel)
    auto setup_row = [&](int ri) {
        const int row = row_of(ri);
        const int b = row / a.H, h = row - b * a.H;
        int hist = a.hist_len[b]; // the tail length is read after the grid dependency wait
        bool bad = false;
        if (hist < 0 || hist > a.max_blocks * 16 || (hist & 31)) {
            bad = true;
            hist = 0;
        }
        int h0 = 0; // sliding attention window (see decode_kernel's setup_row)
        if (GEN && a.attn_window > 0) {
            const int nn = a.tail_len[b];
            h0 = window_first(a.attn_window, a.sink, hist, nn < 0 ? 0 : nn);
        }
        const int g0 = h0 >> 5;
        const int ngroups = (hist >> 5) - g0;
        int nmy = ngroups > (int)crank ? (ngroups - (int)crank + (int)C - 1) / (int)C : 0;
        if (nmy > a.cap_groups) {
            bad = true;
            nmy = a.cap_groups;
        }
        if (bad && warp == 0 && lane == 0)
            atomicOr(a.status, LOOPKV_DEV_STATE);
        const int n = owned(nmy, warp);
        const int32_t *bt = a.block_table + (int64_t)b * a.max_blocks;
        for (int k = lane; k < 2 * n; k += 32) {
            const int g = g0 + (int)crank + (warp + (k >> 1) * kWarps) * (int)C;
            int id = bt[2 * g + (k & 1)];
            if (id < 0 || id >= a.pool_blocks) {
                atomicOr(a.status, LOOPKV_DEV_STATE);
                id = 0;
            }
            ids[k] = id;
        }
        if (lane == 0) {
            irow[IR_ROW] = row;
            irow[IR_B] = b;
            irow[IR_H] = h;
            irow[IR_N] = n;
            irow[IR_TAIL] = -1; // tail length read after the grid dependency wait
            irow[I1_G0] = g0;
            irow[I1_M0] = h0 & 31;
            irow[I1_HIST] = hist;
            if (NSC) {
                const int nch = nstream ? a.near_cap / NR : 0, wg = (int)crank * kWarps + warp, nw = (int)C * kWarps;
                irow[I1_NC] = nch > wg ? (nch - wg + nw - 1) / nw : 0;
            }
        }
        __syncwarp();
        setup_upto = ri;
    };
    // stage n = the next group of the issuing row: both head regions (+ both lo regions)
    auto issue_stage = [&](int n) {
        uint8_t *st = ring + (n & smask) * G1::STAGE;
        uint64_t *fb = &full[n & smask];
        if (NSC && iss_k >= seg_groups) { // near chunk: NR key rows, then the same NR value rows
            if (lane == 0) {
                const size_t off = (size_t)((int)crank * kWarps + warp + (iss_k - seg_groups) * (int)C * kWarps) * NRB;
                mbar_arrive_expect_tx(fb, 2 * NRB);
                bulk_g2s(st, seg_near + off, NRB, fb);
                bulk_g2s(st + NRB, seg_near + (size_t)a.H * a.near_cap * D * sizeof(DT) + off, NRB, fb);
            }
            return;
        }
        const int2 id = reinterpret_cast<const int2 *>(ids)[iss_k];
        if (lane == 0) {
            mbar_arrive_expect_tx(fb, 2 * G::HM + 2 * G::LOB);
            if (GEN && a.inject == LOOPKV_INJECT_STALLED_STAGE && n == 0 && warp == 0 && blockIdx.x == 0)
                return; // test hook: the stage's bytes never arrive, so its wait runs out
            bulk_g2s(st, seg_src + (uint64_t)(uint32_t)id.x * bstride, G::HM, fb);
            bulk_g2s(st + G::HM, seg_src + (uint64_t)(uint32_t)id.y * bstride, G::HM, fb);
            if (BITS == 4) {
                bulk_g2s(st + G1::LOFF, seg_lo + (uint64_t)(uint32_t)id.x * lstride, G::LOB, fb);
                bulk_g2s(st + G1::LOFF + G::LOB, seg_lo + (uint64_t)(uint32_t)id.y * lstride, G::LOB, fb);
            }
        }
    };
    // issue every stage numbered below `limit`; a row's stages follow once it is set up
    auto pump = [&](int limit) {
        if (timed_out)
            return;
        for (;;) {
            if (iss_k < seg_n) {
                if (iss_n >= limit || (NSC && !dep_ok && iss_k >= seg_groups)) // near rows: after the dependency
                    break;
                issue_stage(iss_n);
                ++iss_k;
                ++iss_n;
                continue;
            }
            // move to the row in the slot; rows set up and replaced before the issuer got
            // to them had no group for this warp
            if (iss_row >= setup_upto)
                break;
            iss_row = setup_upto;
            iss_k = 0;
            seg_groups = seg_n = irow[IR_N];
            seg_src = a.main + (size_t)irow[IR_H] * G::HM;
            seg_lo = a.lo + (size_t)irow[IR_H] * G::LOB;
            if (NSC) {
                seg_n += irow[I1_NC];
                seg_near = reinterpret_cast<const uint8_t *>(a.tail) +
                           ((int64_t)irow[IR_B] * 2 * a.H + irow[IR_H]) * a.near_cap * D * sizeof(DT);
            }
        }
    };

    // ---------------------------------------------------------------- compute
    int prc_n = 0;
    auto wait_stage = [&](int n) {
        if (!timed_out && !mbar_wait(&full[n & smask], (n >> spw_log2) & 1, a.status, a.wait_ns)) {
            timed_out = true;
            drain_from = n;
        }
    };
    const bool ownq = lane < G::NQ;

    // Row ri of this CTA: the warp's groups and, in the last CTA, the tail; leaves the
    // warp's partial (o, l relative to 2^m) in its scratch, m at word D + 1.
    auto row_pass = [&](int ri) {
        if (ri == 0)
            setup_row(0);
        const int row = irow[IR_ROW], nown = irow[IR_N], rb = irow[IR_B], rh = irow[IR_H];
        const int ncw = NSC ? irow[I1_NC] : 0, nst = nown + ncw; // this warp's stages: groups, near chunks
        const int rg0 = irow[I1_G0], rm0 = (crank == 0 && warp == 0) ? irow[I1_M0] : 0, rhist = irow[I1_HIST];
        int tail = irow[IR_TAIL];
        // the slot takes row ri + 1 once row ri's stages are all issued (after the pump of
        // stage nst - spw, or at once when the warp has no stage)
        const int k_setup = nst > spw ? nst - spw : 0;
        if (nst == 0 && ri + 1 < nrows)
            setup_row(ri + 1);
        if (ri == 0) { // prefetch, then wait for the previous grid of the stream (see decode_kernel)
            pump(prc_n + spw);
            asm volatile("griddepcontrol.wait;" ::: "memory");
            dep_ok = true;
        }
        int ws = 0;
        if (tail < 0) { // near tokens and ring start (an append may have written them)
            tail = a.tail_len[rb];
            ws = a.win_start[rb];
            if (tail < 0 || tail > a.sink + a.wring || ws < 0 || ws >= a.wring) {
                if (lane == 0 && warp == 0)
                    atomicOr(a.status, LOOPKV_DEV_STATE);
                tail = 0;
                ws = 0;
            }
        }
        if (!nstream && tail > (int)crank * kWarps + warp) { // this warp's near keys and values, read after its groups
            const DT *kt = reinterpret_cast<const DT *>(a.tail) + ((int64_t)rb * 2 * a.H + rh) * a.near_cap * D;
            prefetch_near<D, DT>(a, kt, ws, (int)crank * kWarps + warp, (int)C * kWarps, tail, lane);
            prefetch_near<D, DT>(a, kt + (int64_t)a.H * a.near_cap * D, ws, (int)crank * kWarps + warp, (int)C * kWarps,
                                 tail, lane);
        }
        float qreg[4];
        {
            const DT *qrow = reinterpret_cast<const DT *>(a.q) + (int64_t)row * D + 4 * lane;
#pragma unroll
            for (int i = 0; i < 4; ++i)
                qreg[i] = ownq ? to_f32(qrow[i]) : 0.f;
        }
        Run1<D> run;
        run1_init(run);
        for (int k = 0; k < nst; ++k) {
            const int n = prc_n++;
            if (iss_n < n + spw)
                pump(n + spw);
            if (k == k_setup && ri + 1 < nrows) {
                setup_row(ri + 1);
                pump(n + spw);
            }
            wait_stage(n);
            const uint8_t *st = ring + (n & smask) * G1::STAGE;
            if (NSC && k >= nown) { // a chunk of the streamed near region
                const int slot0 = ((int)crank * kWarps + warp + (k - nown) * (int)C * kWarps) * NR;
                run1_near_chunk<D, DT, NR, GEN>(run, reinterpret_cast<const DT *>(st),
                                                reinterpret_cast<const DT *>(st + NRB), qreg, a, slot0, ws, tail, rhist,
                                                lane);
                continue;
            }
            const int masked = GEN && k == 0 ? rm0 : 0; // tokens of the first group before a sliding window
            run1_group<BITS, D>(st, st + G1::LOFF, scr, qreg, a.qscale, lane, run, masked);
            if (GEN && a.s_bitmap && lane == 0) // refine set: every attended token (4-bit, tau <= 0) or none (2-bit)
                a.s_bitmap[(int64_t)row * a.bitmap_words + rg0 + (int)crank + (warp + k * kWarps) * (int)C] =
                    BITS == 4 ? ~((1u << masked) - 1u) : 0u;
        }
        float *red = reinterpret_cast<float *>(scr);
        run1_finish<BITS, D>(run, red, lane);
        const int wg = (int)crank * kWarps + warp; // tail token j to warp j mod (C * kWarps) of the cluster
        if (!nstream && tail > wg) {
            const DT *kt = reinterpret_cast<const DT *>(a.tail) + ((int64_t)rb * 2 * a.H + rh) * a.near_cap * D;
            const DT *vt0 =
                reinterpret_cast<const DT *>(a.tail) + ((int64_t)(rb * 2 + 1) * a.H + rh) * a.near_cap * D;
            run1_tail<D, DT>(run, red, lane, qreg, a, kt, vt0, ws, rhist, wg, (int)C * kWarps, tail);
        }
        if (lane == 0)
            red[D + 1] = run.m;
        named_sync(1, kThreads);
    };

    // The CTA's partial of row ri relative to the CTA's maximum mc, into parts[ri & 1].
    auto cta_partial = [&](int ri) {
        float wmx[kWarps];
#pragma unroll
        for (int w = 0; w < kWarps; ++w)
            wmx[w] = reinterpret_cast<const float *>(scr_all + w * SCR)[D + 1];
        float mc = -INFINITY;
#pragma unroll
        for (int w = 0; w < kWarps; ++w)
            mc = fmaxf(mc, wmx[w]);
        float fw[kWarps];
#pragma unroll
        for (int w = 0; w < kWarps; ++w)
            fw[w] = wmx[w] == -INFINITY ? 0.f : ex2(wmx[w] - mc);
        float *part = parts + (ri & 1) * (D + 2);
        for (int c = threadIdx.x; c <= D; c += kThreads) {
            float sum = 0.f;
#pragma unroll
            for (int w = 0; w < kWarps; ++w)
                sum += fw[w] * reinterpret_cast<const float *>(scr_all + w * SCR)[c];
            part[c] = sum;
        }
        if (threadIdx.x == 0)
            part[D + 1] = mc;
    };

    // CTA `crank` writes channels [crank*per, min(D, (crank+1)*per)) of row ri, per =
    // ceil(D / C), from the partials of every CTA rescaled to the row maximum M.
    auto merge = [&](int ri) {
        const int row = row_of(ri);
        const float *part = parts + (ri & 1) * (D + 2);
        const int per = (D + (int)C - 1) / (int)C;
        const int c = (int)crank * per + (int)threadIdx.x;
        if ((int)threadIdx.x < per && c < D) {
            float M = -INFINITY;
            for (uint32_t r = 0; r < C; ++r)
                M = fmaxf(M, ld_dsmem_f32(part + D + 1, r));
            float o = 0.f, l = 0.f;
            if (M != -INFINITY)
                for (uint32_t r = 0; r < C; ++r) {
                    const float mr = ld_dsmem_f32(part + D + 1, r);
                    const float f = mr == -INFINITY ? 0.f : ex2(mr - M);
                    o = fmaf(f, ld_dsmem_f32(part + c, r), o);
                    l = fmaf(f, ld_dsmem_f32(part + D, r), l);
                }
            float out = 0.f;
            if (l > 0.f)
                out = o / l;
            else if (c == 0)
                atomicOr(a.status, LOOPKV_DEV_EMPTY_ROW);
            a.out[(int64_t)row * D + c] = out;
            if (c == 0) {
                if (a.row_max)
                    a.row_max[row] = M * 0.6931471805599453f;
                if (a.row_sum)
                    a.row_sum[row] = l;
            }
        }
    };

    // One cluster barrier per row: barrier i publishes the CTA partials of row i, merged
    // after the pass of row i + 1.  parts[i & 1] is written once this CTA has passed
    // barrier i - 1, which every CTA reaches only after its merge of row i - 2, the last
    // reader of that buffer.
    for (int i = 0; i <= nrows; ++i) {
        if (i < nrows)
            row_pass(i);
        if (i > 0) {
            cluster_wait(); // barrier i - 1
            merge(i - 1);
        }
        if (i < nrows) {
            cta_partial(i);
            named_sync(1, kThreads); // every warp's scratch is free again
            cluster_arrive();       // barrier i
        }
    }
    if (timed_out) // copies issued before the give-up must land before the shared memory is freed
        for (int n = drain_from; n < iss_n; ++n)
            mbar_wait(&full[n & smask], (n >> spw_log2) & 1, a.status, a.wait_ns);
    cluster_arrive(); // the remote reads of the last merge are done
    cluster_wait();
}

// Launch `kern` with the shape's grid, cluster and shared memory (and programmatic
// stream serialization when the shape asks for it).
template <typename K, typename... Args>
int launch_shape(K kern, const DecodeShape &shp, bool pdl, cudaStream_t s, Args... args)
{
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
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = shp.cluster;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization; // see griddepcontrol in the kernels
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = (shp.pdl && pdl) ? 2 : 1;
    e = cudaLaunchKernelEx(&cfg, kern, args...);
    return e == cudaSuccess ? LOOPKV_OK : LOOPKV_ERR_CUDA;
}

template <int BITS, int D, typename DT>
int launch_t(const DecodeArgs &a, const DecodeShape &shp, bool pdl, cudaStream_t s)
{
    // the general build for the modes that the lean one leaves out
    const bool gen = a.s_bitmap != nullptr || a.tau_mode == LOOPKV_TAU_STREAM || a.attn_window > 0 ||
                     a.inject != LOOPKV_INJECT_NONE;
    if constexpr (BITS == 4) {
        if (!shp.onepass) {
            const int var = gen ? 2 : (a.near_cap > 32 ? 1 : 0);
            auto kern = shp.min_ctas == 5
                            ? (var == 2 ? decode_kernel<BITS, D, DT, 5, 2>
                                        : var == 1 ? decode_kernel<BITS, D, DT, 5, 1> : decode_kernel<BITS, D, DT, 5, 0>)
                            : (var == 2 ? decode_kernel<BITS, D, DT, 4, 2>
                                        : var == 1 ? decode_kernel<BITS, D, DT, 4, 1> : decode_kernel<BITS, D, DT, 4, 0>);
            return launch_shape(kern, shp, pdl, s, a, shp.stages_log2, shp.score_bufs);
        }
    }
    if (!shp.onepass)
        return LOOPKV_ERR_CUDA; // 2-bit sources have no refine set: always the single-pass reader
    const int var = gen ? 2 : (a.near_cap > 32 ? 1 : 0);
    return launch_shape(var == 2   ? decode_kernel_1p<BITS, D, DT, 4, 2>
                        : var == 1 ? decode_kernel_1p<BITS, D, DT, 4, 1>
                                   : decode_kernel_1p<BITS, D, DT, 4, 0>,
                        shp, pdl, s, a, shp.stages_log2);
}

// Clusters of size C that can be resident at once for this kernel and shared memory.
template <typename K> int max_active_clusters(K kern, int C, int smem)
{
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

// Launch shape.  Model: a cluster of C CTAs serves ceil(rows / clusters) rows one after
// another; a CTA's share of one row costs (groups / C + kRowFixed) group-times, and an SM
// running n CTAs gives each 1 / max(n, kSaturate) of its throughput.  Time is then
// rounds * (G / C + kRowFixed) * max(n, kSaturate) with n the CTAs on the busiest SM; rows
// that do not overlap (one score buffer, several rounds) cost kSeqRow more each.  Among
// equal times the deeper ring (more bytes in flight) wins.
constexpr double kRowFixed = 6.0;  // per-CTA cost of a row outside its groups (setup, merge, bubble)
constexpr double kSaturate = 3.5;  // CTAs per SM that keep its issue slots busy
constexpr double kSeqRow = 4.0;    // extra per-row cost when rows do not overlap (one score buffer)

// Overlap with the previous launch of the stream (programmatic dependent launch): on B200
// measured faster for the single-pass reader with clusters of up to 4 CTAs (+9% on the 8K
// KIVI-4 workload) and slower for the exact-maximum reader (-9% on the mixed 8K workload).
inline int pdl_default(int C, bool onepass) { return onepass && C <= 4; }

// Debug override of the launch-shape model, for measurements only: LOOPKV_DECODE_SHAPE =
// "cluster,stages,ctas_per_sm,score_buffers,pdl", each field 0 (or absent) for the model's
// choice; pdl 1 = on, 2 = off.  Read when a cache first computes the shape of a batch size.
struct ShapeOverride {
    int cluster = 0, stages = 0, ctas = 0, bufs = 0, pdl = 0;
};
inline ShapeOverride shape_override()
{
    ShapeOverride o;
    if (const char *env = getenv("LOOPKV_DECODE_SHAPE")) {
        int v[5] = {0, 0, 0, 0, 0};
        sscanf(env, "%d,%d,%d,%d,%d", &v[0], &v[1], &v[2], &v[3], &v[4]);
        o.cluster = v[0], o.stages = v[1], o.ctas = v[2], o.bufs = v[3], o.pdl = v[4];
    }
    return o;
}

// Shared memory of a kernel with `spw` ring slots per warp.
template <int BITS, int D> int kernel_smem(bool onepass, int spw, int capw, int nbuf, int near_cap)
{
    if (onepass)
        return layout1_ok<BITS, D>(spw, capw) ? smem_layout1<BITS, D>(spw, capw).total : -1;
    return layout_ok<BITS, D>(spw, capw, nbuf, near_cap) ? smem_bytes<BITS, D>(spw, capw, nbuf, near_cap) : -1;
}

template <int BITS, int D, typename DT> DecodeShape shape_t(int rows, int max_blocks, int near_cap, bool onepass)
{
    DecodeShape best = {};
    double best_t = 1e300;
    const int max_groups = max_blocks / 2;
    int sm_count = 148;
    {
        int dev = 0;
        cudaGetDevice(&dev);
        if (cudaDeviceGetAttribute(&sm_count, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            sm_count = 148;
    }
    const int smem_per_sm = 228 * 1024;
    const ShapeOverride ov = shape_override();
    if (BITS == 2)
        onepass = true;
    // two-phase builds for 4 and 5 CTAs per SM; the single-pass kernel for 4 (its 96-register
    // build measured 5% slower on the same grid)
    for (int want_ctas = 4; want_ctas <= (onepass ? 4 : 5); ++want_ctas) {
        if (ov.ctas && ov.ctas != want_ctas)
            continue;
        for (int C = 1; C <= 16; C = C < 8 ? C + 1 : 2 * C) { // 1..8, 16
            if (ov.cluster && ov.cluster != C)
                continue;
            const int cap = (max_groups + C - 1) / C;
            const int capw = (cap + kWarps - 1) / kWarps;
            const int budget = smem_per_sm / want_ctas - 1024;
            for (int nbuf = 1; nbuf <= 2; ++nbuf) {
                // slots per warp (a power of two): fill the shared memory of `want_ctas` CTAs per SM
                int spw = 8;
                while (spw > 2 && kernel_smem<BITS, D>(onepass, spw, capw, nbuf, near_cap) > budget)
                    spw >>= 1;
                if (ov.stages) // at least 2: the two-phase reader fills the next stage's slot early
                    spw = std::max(ov.stages, 2);
                const int smem = kernel_smem<BITS, D>(onepass, spw, capw, nbuf, near_cap);
                if (smem <= 0 || smem > 227 * 1024)
                    continue;
                int ncl = 0;
                // occupancy of the general build (the lean one has the same launch bounds)
                if (onepass)
                    ncl = max_active_clusters(decode_kernel_1p<BITS, D, DT, 4, 2>, C, smem);
                else if constexpr (BITS == 4)
                    ncl = want_ctas == 5 ? max_active_clusters(decode_kernel<BITS, D, DT, 5, 2>, C, smem)
                                         : max_active_clusters(decode_kernel<BITS, D, DT, 4, 2>, C, smem);
                if (ncl <= 0)
                    continue;
                if (ncl > rows)
                    ncl = rows;
                if (!onepass && ov.bufs && ov.bufs != nbuf)
                    continue;
                const int rounds = (rows + ncl - 1) / ncl;
                const int per_sm = (ncl * C + sm_count - 1) / sm_count;
                // one score buffer with several rows per cluster: rows run one after another
                const double row_cost = kRowFixed + (!onepass && nbuf == 1 && rounds > 1 ? kSeqRow : 0.0);
                const double t = rounds * ((double)max_groups / C + row_cost) * std::max((double)per_sm, kSaturate) *
                                 (1.0 - 0.01 * spw);
                if (t < best_t * (1.0 - 1e-9)) {
                    best_t = t;
                    best.cluster = C;
                    best.clusters = ncl;
                    best.stages = spw;
                    best.stages_log2 = __builtin_ctz(spw);
                    best.score_bufs = onepass ? 0 : nbuf;
                    best.smem = smem;
                    best.threads = kThreads;
                    best.cap = cap;
                    best.min_ctas = want_ctas;
                    best.pdl = ov.pdl ? ov.pdl == 1 : pdl_default(C, onepass);
                    best.onepass = onepass;
                }
                if (onepass)
                    break; // no score buffers
            }
        }
    }
    return best;
}

}  // namespace

DecodeShape decode_shape(int bits, int D, int dtype, int rows, int max_blocks, int near_cap, bool onepass)
{
    const bool bf = dtype == LOOPKV_DTYPE_BF16;
    const int mb = max_blocks;
    if (bits == 4) {
        if (D == 128)
            return bf ? shape_t<4, 128, __nv_bfloat16>(rows, mb, near_cap, onepass) : shape_t<4, 128, float>(rows, mb, near_cap, onepass);
        return bf ? shape_t<4, 64, __nv_bfloat16>(rows, mb, near_cap, onepass) : shape_t<4, 64, float>(rows, mb, near_cap, onepass);
    }
    if (D == 128)
        return bf ? shape_t<2, 128, __nv_bfloat16>(rows, mb, near_cap, onepass) : shape_t<2, 128, float>(rows, mb, near_cap, onepass);
    return bf ? shape_t<2, 64, __nv_bfloat16>(rows, mb, near_cap, onepass) : shape_t<2, 64, float>(rows, mb, near_cap, onepass);
}

int launch_decode(const DecodeArgs &a, int bits, int D, int dtype, const DecodeShape &shp, bool pdl, cudaStream_t s)
{
    if (shp.cluster <= 0 || shp.clusters <= 0)
        return LOOPKV_ERR_CUDA;
    const bool bf = dtype == LOOPKV_DTYPE_BF16;
    if (bits == 4) {
        if (D == 128)
            return bf ? launch_t<4, 128, __nv_bfloat16>(a, shp, pdl, s) : launch_t<4, 128, float>(a, shp, pdl, s);
        return bf ? launch_t<4, 64, __nv_bfloat16>(a, shp, pdl, s) : launch_t<4, 64, float>(a, shp, pdl, s);
    }
    if (D == 128)
        return bf ? launch_t<2, 128, __nv_bfloat16>(a, shp, pdl, s) : launch_t<2, 128, float>(a, shp, pdl, s);
    return bf ? launch_t<2, 64, __nv_bfloat16>(a, shp, pdl, s) : launch_t<2, 64, float>(a, shp, pdl, s);
}

}  // namespace lkv
