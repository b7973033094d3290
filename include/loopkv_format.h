/*
 * loopkv_format.h -- storage format of the LoopKV history pages (CUDA side).
 *
 * The LoopKV paper (arXiv 2611.04137, §3.3 "Bit-plane V layout" and §3.4 "Layout")
 * fixes what a page holds -- keys as interleaved 4-bit codes, values of a 4-bit cell
 * as two 2-bit planes hi and lo followed by scales and zero points, 2-bit cells with
 * their own 2-bit codes, fp16 scale and zero per group of 32 -- but not the byte
 * order.  This file fixes it.  The CPU oracle restates the same rules in its own
 * code; nothing here is shared with it.
 *
 * Pages.  A block is 16 tokens of one (cell, request) for all H heads; a K group of
 * 32 tokens is two consecutive blocks of the request's block table (the paper's
 * 32-token page).  Inside a block the heads follow one another; per head:
 *
 *   4-bit main region (LKV_HEAD_MAIN_4B(D) bytes; 2048 at D = 128)
 *     [K codes   16 rows x D/2 ]  4-bit row, see below
 *     [K meta    D x fp16      ]  K scale of each channel in the even block of the
 *                                 group, K zero point in the odd block
 *     [V meta    D/32 x 16 x (fp16 scale, fp16 zero)]  ordered [channel group][token]
 *     [V hi      16 x D/4 bytes]  plane of h = code >> 2, words [kappa][tau] (below)
 *   4-bit lo region, a separate pool (LKV_HEAD_LO_4B(D) = 16 x D/4 bytes)
 *     [V lo      16 x D/4 bytes]  plane of l = code & 3, words [tau][kappa]
 *   2-bit main region (LKV_HEAD_MAIN_2B(D); 1536 at D = 128)
 *     [K codes 16 x D/4][K meta D x fp16][V meta D/32 x 16 x 2 fp16][V codes, as V hi]
 *
 * Key rows (little-endian 32-bit words, one row per token):
 *   4-bit row: word w holds channels 8w..8w+7; in byte b of the word the low nibble
 *              is channel 8w+b and the high nibble channel 8w+4+b.  So nibble j of the
 *              word (bits 4j..4j+3) is channel 8w + (j odd ? 4 : 0) + j/2.
 *   2-bit row: word w holds channels 16w..16w+15; in byte b, bits 2i..2i+1 are
 *              channel 16w+4i+b.  So the field at bit 8b+2i is channel 16w+4i+b.
 * Value planes (little-endian 32-bit words, 4 tokens x 4 channels each):
 *   word (kappa, tau) holds tokens 4tau..4tau+3 and channels 4kappa..4kappa+3 of the
 *   block: byte b is token 4tau+b, and in it bits 2i..2i+1 are channel 4kappa+i.  The
 *   hi plane stores word (kappa, tau) at index 4*kappa + tau, the lo plane at index
 *   tau*(D/4) + kappa, so that the lo values of 4 consecutive tokens are D contiguous
 *   bytes.  Four tokens sit in the four bytes of a word, so a dp4a against per-token
 *   weight digits sums over tokens.
 *
 * Quantization rule (per group of 32 values x, L = 15 or 3):
 *   zero = largest fp16 <= min(x); scale = smallest fp16 >= (max(x) - zero) / L in
 *   fp64; code = clamp(round_half_even(fl32(fl32(x - zero) / scale)), 0, L), all 0
 *   when scale = 0.  A non-finite x, or an infinite zero/scale, writes
 *   zero = scale = 0 and all codes 0 and raises the device status bit.
 */
#ifndef LOOPKV_FORMAT_H
#define LOOPKV_FORMAT_H

#define LKV_BLOCK_TOKENS 16
#define LKV_GROUP 32
#define LKV_TAIL_TOKENS 32

#define LKV_HEAD_KCODES_4B(D) (16 * (D) / 2)
#define LKV_HEAD_KCODES_2B(D) (16 * (D) / 4)
#define LKV_HEAD_KMETA(D) (2 * (D))
#define LKV_HEAD_VMETA(D) (16 * ((D) / 32) * 4)
#define LKV_HEAD_VPLANE(D) (16 * (D) / 4)
#define LKV_HEAD_MAIN_4B(D) (LKV_HEAD_KCODES_4B(D) + LKV_HEAD_KMETA(D) + LKV_HEAD_VMETA(D) + LKV_HEAD_VPLANE(D))
#define LKV_HEAD_LO_4B(D) LKV_HEAD_VPLANE(D)
#define LKV_HEAD_MAIN_2B(D) (LKV_HEAD_KCODES_2B(D) + LKV_HEAD_KMETA(D) + LKV_HEAD_VMETA(D) + LKV_HEAD_VPLANE(D))

#endif /* LOOPKV_FORMAT_H */
