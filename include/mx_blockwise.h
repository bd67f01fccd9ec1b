/*
 * mx_blockwise.h -- C ABI of the block-wise bit-width variant of the mixed-
 * precision linear layer (ScaleBITS blog page: section 1.2.2, one bit width per
 * 64 x 128 block of the weight matrix; section 3.2, a block-wise layout with
 * 2-bit metadata giving each block's width; section 4.2, widths from
 * {1, 2, 3, 4, 6, 8}), run on the int8 two-step dequantization of MixLLM
 * (section 3.3).
 *
 * What is computed (readings of the page, which gives no quantizer):
 *  - a block is 64 output rows x 128 input columns; the last row block may be
 *    short; K is a multiple of 128;
 *  - each block's 2-bit code indexes a four-entry width table of the layer
 *    (each width 1..8); codes are four to a byte, block i in bits 2 (i mod 4)
 *    of byte i / 4, row-major over (row block, column block);
 *  - inside a block, each row's 128 weights are one group with an fp16 scale
 *    and a uint8 zero point.  Width b < 8: the asymmetric b-bit quantizer
 *    (levels 0 .. 2^b - 1; the MixLLM 4-bit quantizer when b = 4).  Width 8:
 *    MixLLM's symmetric 8-bit quantizer, stored in offset binary (code
 *    q + 128, zero 128).  Either way q - z fits int8;
 *  - Y[m, n] = s_a[m] * sum_kb s_w[n, kb] * P[m, n, kb] with the exact integer
 *    partial P[m, n, kb] = sum over the block's 128 columns of
 *    Aq[m, k] * (q[n, k] - z[n, kb]); activations as mx_quant_act makes them.
 *
 * Conventions as in mx.h: device pointers unless stated, every call checks its
 * arguments on the host and returns an mx_status before any launch, launches
 * are asynchronous in `stream`, the message of the last error is
 * mx_last_error().
 */
#ifndef MX_BLOCKWISE_H
#define MX_BLOCKWISE_H

#include "mx.h"

#ifdef __cplusplus
extern "C" {
#endif

#define MX_BW_BLOCK_ROWS 64
#define MX_BW_BLOCK_COLS 128

/*
 * Geometry of one block-wise packed layer (all offsets in bytes from the start
 * of the blob, each 16-byte aligned):
 *   header   64 bytes: "MXBW", version 1, N, K, the width table
 *   meta     ceil(NB KB / 4) bytes of 2-bit block codes
 *   offsets  uint32 [NB KB + 1]: start of each block's codes, in 16-byte units
 *            from off_codes; the last entry is the end
 *   scales   fp16 [N][KB]
 *   zeros    uint8 [N][KB]
 *   codes    per block in row-major (row block, column block) order: each of
 *            its rows holds 128 codes of b bits in 16 b bytes, code k in bits
 *            k b .. k b + b - 1 of that little-endian bit string
 */
typedef struct mx_bw_layout {
    int32_t N, K;              /* W is [N, K] */
    int32_t NB, KB;            /* ceil(N / 64) row blocks, K / 128 column blocks */
    uint8_t table[4];          /* the widths the 2-bit codes select */
    int32_t reserved0;
    uint64_t off_meta, off_offsets, off_scales, off_zeros, off_codes;
    uint64_t code_bytes;       /* bytes of all blocks' codes */
    uint64_t total_bytes;
} mx_bw_layout;

/*
 * mx_bw_layout_init -- host only, no device work.  Geometry of a layer whose
 * block codes are `meta` (host, packed as above, ceil(NB KB / 4) bytes).
 * Returns MX_ERR_INVALID_ARG if N < 1, K is not a positive multiple of 128, a
 * width is outside 1..8, or meta is NULL.
 */
mx_status mx_bw_layout_init(int N, int K, const uint8_t table[4], const uint8_t* meta, mx_bw_layout* out);

/*
 * mx_bw_pack -- quantize W block by block into `blob` (L->total_bytes bytes,
 * device, 16-byte aligned).  W is device [N][ldw], fp32 or fp16.  `meta` is the
 * host copy of the block codes L was made from; the header, codes and block
 * offsets are copied into the blob in `stream` before the quantization kernel
 * runs (the host buffers may be reused once the call returns).
 */
mx_status mx_bw_pack(const mx_bw_layout* L, const uint8_t* meta, const void* W, mx_dtype wdtype, int64_t ldw,
                     void* blob, void* stream);

/*
 * mx_bw_gemm -- Y[M, N] = the two-step product above, on CUDA cores (dp4a): one
 * warp per output row, 4 codes per lane per block, an fp32 sum per lane of
 * s_w P, then a warp sum and s_a.  Meant for decode-sized M; any M >= 1 is
 * served (tokens in tiles of 8).
 *   Aq       int8 [M][K], s_a fp16 [M] (mx_quant_act)
 *   Y        fp16 [M][ldy], ldy >= N
 *   partials int32 [M][N][KB] or NULL: every P[m, n, kb] (for testing)
 */
mx_status mx_bw_gemm(const mx_bw_layout* L, const void* blob, const int8_t* Aq, const void* s_a, int M, void* Y,
                     int64_t ldy, int32_t* partials, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* MX_BLOCKWISE_H */
