/*
 * mx.h -- C ABI of the B200 (sm_100a) MixLLM mixed-precision quantized linear layer.
 *
 * The method (MixLLM: "LLM Quantization with Global Mixed-precision between
 * Output-features and Highly-efficient System Design"):
 *   - output features (rows of W [N, K]) are split by saliency into 8-bit
 *     symmetric rows and 4-bit asymmetric rows, each quantized group-wise along
 *     K (group 64 or 128) with fp16 scales (section 3.1.1, Figure 1;
 *     section 3.1.2; section 2.1 for the two quantizer formulas);
 *   - activations X [M, K] are quantized to 8-bit symmetric codes, one fp16
 *     scale per token (section 3.1.2);
 *   - Y = dequant(Xq) dequant(Wq)^T is computed by two-step dequantization:
 *     int8 products of A_q and (W_q - z) summed per group into int32, then
 *     both scales applied per group in fp32 (section 3.3); the two row sets
 *     are independent sub-problems whose outputs are scattered back into one
 *     Y by the epilogue (section 3.3, "parallel execution of sub-problems").
 *
 * Conventions shared by every entry point:
 *   - Every pointer named "device" is caller-owned device memory (for example
 *     a torch tensor).  The library never allocates device memory and keeps no
 *     device state between calls.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  All device work is enqueued asynchronously on it.
 *   - Argument errors are detected on the host BEFORE anything is enqueued and
 *     returned as an mx_status; mx_last_error() then holds a one-line message
 *     for the calling thread.  Errors found by a kernel while it runs are
 *     written to the optional device `status` word (0 = ok) and never trap.
 *   - fp16 values cross the boundary as uint16_t bit patterns (IEEE binary16).
 *   - Device pointers must be 16-byte aligned; leading dimensions are in
 *     elements and must keep every row 16-byte aligned.
 */
#ifndef MX_H
#define MX_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MX_ABI_VERSION 2
#define MX_BLOB_VERSION 1          /* packed-blob layout version, in the blob header */

typedef enum mx_status {
    MX_OK = 0,
    MX_ERR_INVALID_ARG = 1,   /* null/negative/inconsistent argument */
    MX_ERR_UNSUPPORTED = 2,   /* valid for the method, not supported by this build */
    MX_ERR_ALIGNMENT = 3,     /* pointer or leading dimension not 16-byte aligned */
    MX_ERR_CUDA = 4,          /* a CUDA runtime/driver call failed (message says which) */
    MX_ERR_TIMEOUT = 5,       /* device status only: a bounded wait gave up */
    MX_ERR_BAD_BLOB = 6,      /* packed-weight header does not match the layout */
    MX_ERR_WORKSPACE = 7      /* workspace missing or smaller than required */
} mx_status;

typedef enum mx_dtype { MX_F32 = 0, MX_F16 = 1 } mx_dtype;

/* Rows per packed row tile and K columns per packed k-block. */
#define MX_TILE_ROWS 128
#define MX_KBLOCK 128
#define MX_HEADER_BYTES 256
#define MX_BLOB_MAGIC 0x4B50584Du /* "MXPK" */

/*
 * Geometry of one packed layer.  Filled by mx_layout_init (or read back from a
 * blob header by mx_layout_from_header); treated as read-only afterwards.
 *
 * Packed blob (one device buffer, `total_bytes` long, every section 256-byte
 * aligned, offsets from the blob start):
 *   header   [256 B]   magic, MX_BLOB_VERSION, N, K, group, n8 (see mx_layout_from_header)
 *   rowmap   int32 [(t8 + t4) * 128]   packed slot -> original row of W, -1 for
 *                      padding.  Slots 0 .. 128*t8-1 hold the 8-bit rows in
 *                      ascending original index; slots from 128*t8 on hold the
 *                      4-bit rows in ascending original index.
 *   scales8  fp16  [t8][G][128]        scale of (row tile, group, row in tile)
 *   codes8   int8  [t8][K/128][128 x 128 B]  one 16 KB block per (tile, k-block):
 *                      row r's 128 codes occupy bytes r*128 .. r*128+127, and
 *                      the 16-byte chunk holding k = 16c .. 16c+15 sits at chunk
 *                      position (c XOR (r mod 8)) -- the 128-byte swizzle that
 *                      the tensor-core shared-memory operand layout expects.
 *   scales4  fp16  [t4][G][128]
 *   zeros4   uint8 [t4][G][128]        zero point z in 0..15 (one byte each)
 *   codes4   uint8 [t4][K/128][128 x 64 B]   one 8 KB block per (tile, k-block):
 *                      row r's 64 bytes at r*64; the 32-bit word w (0..15) of a
 *                      row holds k = 8w .. 8w+7: byte b has k = 8w+b in its low
 *                      nibble and k = 8w+4+b in its high nibble.
 * Padding rows have zero codes, zero scales and zero zero-points.
 */
typedef struct mx_layout {
    int32_t N, K, group, n8;   /* problem: W is [N, K]; n8 rows at 8 bits */
    int32_t n4, G;             /* N - n8, K / group */
    int32_t t8, t4;            /* row tiles of 128 in each part (ceil) */
    int32_t kblocks;           /* K / 128 */
    int32_t reserved0;
    uint64_t off_rowmap, off_scales8, off_codes8, off_scales4, off_zeros4, off_codes4;
    uint64_t total_bytes;
} mx_layout;

/* Options of mx_gemm; pass NULL for the defaults (all fields zero). */
typedef struct mx_gemm_opts {
    int32_t path;              /* 0 auto; 1 split-K CUDA-core path; 2 tensor-core path;
                                  3 row CUDA-core path (whole rows per CTA); 4 tensor-core
                                  path on CTA pairs (cta_group::2, 256 rows x 128 tokens);
                                  5 tensor-core path on CTA pairs with 256-token tiles
                                  (256 rows x 256 tokens, no K split); 6 tensor-core
                                  path for decode-sized M <= 128 (one CTA per tile:
                                  128 rows x the batch rounded up to 16 tokens) */
    int32_t split;             /* path 1: CTAs (a thread-block cluster, 1..8) that split
                                  the K range of each row unit (0 = auto); a split
                                  asked for under auto selects path 1 for M <= 16.
                                  path 4: K splits (1..8; 0 = auto: more than one only
                                  when the unsplit grid leaves CTA pairs idle and the
                                  workspace holds the split sums).  path 6: K splits
                                  (1..16; 0 = auto, taken when the workspace holds the
                                  split sums) */
    int32_t* debug_partials;   /* device int32 [M][N][G] or NULL: every per-group
                                  int32 partial P[m][n][g] (original row order) */
    int32_t* status;           /* device int32 or NULL: kernel-side error code */
    int32_t wait_timeout_us;   /* bound on every in-kernel wait of the tensor-core
                                  path (0 = 2 s); on expiry the kernel writes
                                  MX_ERR_TIMEOUT to *status, frees what it holds
                                  and returns */
    int32_t test_stall;        /* testing only: the tensor-core loader issues no
                                  copies, so the waits run out (needs status) */
    int32_t act_group;         /* activation scales: 0 = one per token, s_a [M];
                                  g (must equal the weight group) = one per token and
                                  group of g columns, s_a [M][K/g] (MixLLM section
                                  3.1.2: group-wise activations), as written by
                                  mx_quant_act_grouped */
} mx_gemm_opts;

/* ABI version of the loaded library (MX_ABI_VERSION). */
int mx_version(void);

/* One-line description of the calling thread's last error ("" if none). */
const char* mx_last_error(void);

/*
 * mx_layout_init -- host only, no device work.  Computes the packed geometry
 * and the blob size of a layer with W [N, K], group size `group` and `n8`
 * 8-bit rows (the rest 4-bit).
 * Constraints: N >= 1, 0 <= n8 <= N, group in {64, 128}, K a positive multiple
 * of 128 (the k-block of the packed layout).  Groups of 64/128 columns follow
 * the MixLLM experimental setting (group 128) and keep every group's int8 dot
 * product inside the fast int-to-float window (section 3.3).
 * Returns MX_ERR_INVALID_ARG / MX_ERR_UNSUPPORTED otherwise.
 */
mx_status mx_layout_init(int N, int K, int group, int n8, mx_layout* out);

/*
 * mx_layout_from_header -- host only.  Validates a copy of a blob's first
 * MX_HEADER_BYTES bytes (copied to host memory by the caller) and rebuilds its
 * layout.  Returns MX_ERR_BAD_BLOB if the magic, version or geometry is wrong.
 */
mx_status mx_layout_from_header(const void* host_header, size_t bytes, mx_layout* out);

/*
 * mx_pack_weights -- offline weight packing (MixLLM section 3.3: the weight
 * layout is pre-packed so that no permutation happens at run time; section
 * 3.1.1: the 8-bit and 4-bit rows form separate sub-problems).
 *   W       device [N][ldw] fp32 or fp16 (wdtype), row-major, ldw >= K
 *   is8     device uint8 [N], nonzero = the row is salient and stays 8-bit;
 *           exactly L->n8 entries must be nonzero
 *   blob    device, L->total_bytes bytes, written completely
 *   status  device int32 or NULL; set to MX_ERR_INVALID_ARG if the mask does
 *           not hold exactly n8 ones (the blob is then unusable)
 * 8-bit rows: s = fp16(absmax/127) (zero scale -> 1, fp16 overflow saturates),
 *   q = clamp(round_half_even(w / s), -127, 127)        (section 2.1, symmetric)
 * 4-bit rows: lo = min(0, min w), hi = max(0, max w), s = fp16((hi - lo)/15),
 *   z = clamp(round(-lo / s), 0, 15), q = clamp(round(w / s) + z, 0, 15)
 *                                                       (section 2.1, affine)
 * Every fp32 step is one IEEE operation (no contraction, true division).
 */
mx_status mx_pack_weights(const mx_layout* L, const void* W, mx_dtype wdtype, int64_t ldw,
                          const uint8_t* is8, void* blob, int32_t* status, void* stream);

/*
 * mx_quant_act -- per-token 8-bit symmetric activation quantization
 * (MixLLM section 3.1.2; quantizer of section 2.1, range +-127).
 *   X    device [M][ldx] fp32 or fp16 (xdtype), ldx >= K
 *   Aq   device int8 [M][K] (dense, row stride K)
 *   s_a  device fp16 bits [M]: s_a = fp16(max_k |X[m,k]| / 127), 0 -> 1
 *   Aq[m,k] = clamp(round_half_even(X[m,k] / s_a[m]), -127, 127)
 * M = 0 is a no-op.  K must be a positive multiple of 8.
 */
mx_status mx_quant_act(const void* X, mx_dtype xdtype, int M, int K, int64_t ldx,
                       int8_t* Aq, uint16_t* s_a, void* stream);

/*
 * mx_quant_act_grouped -- group-wise 8-bit symmetric activation quantization
 * (MixLLM section 3.1.2: activations quantized group-wise, group 128 as the
 * weights).  act_group = 0 is mx_quant_act.  Otherwise, with G = K / act_group:
 *   s_a  device fp16 bits [M][G]: s_a[m,g] = fp16(max |X[m, g*act_group ..
 *        (g+1)*act_group)| / 127), 0 -> 1
 *   Aq[m,k] = clamp(round_half_even(X[m,k] / s_a[m, k / act_group]), -127, 127)
 * act_group must be 0, 64 or 128 and divide K.  Other arguments and errors as
 * mx_quant_act.  A GEMM reads these scales when its options carry the same
 * act_group (which must equal the layer's weight group).
 */
mx_status mx_quant_act_grouped(const void* X, mx_dtype xdtype, int M, int K, int64_t ldx, int act_group,
                               int8_t* Aq, uint16_t* s_a, void* stream);

/*
 * mx_gemm_workspace_size -- host only.  Bytes of device workspace mx_gemm
 * uses for this layer at M tokens with these options: S * M * N * 4 (rounded up
 * to 256) when path 4 splits K S > 1 ways, else 0.  A negative split is
 * MX_ERR_INVALID_ARG.
 */
mx_status mx_gemm_workspace_size(const mx_layout* L, int M, const mx_gemm_opts* opts,
                                 size_t* bytes);

/*
 * mx_gemm_select_path -- host only.  The GEMM path mx_gemm will take for this
 * layer at M tokens with these options.  The decode-sized paths are HBM-bound
 * and run on CUDA cores:
 *   3 = row path: M <= 4, K <= 4096 and one wave of CTAs; every CTA owns 32
 *       4-bit (or 16 8-bit) rows over the whole K, no reduction between CTAs;
 *   1 = split-K path: M <= 16; the K split of each row unit is one thread-block
 *       cluster reduced through distributed shared memory;
 *   4 = tensor cores on CTA pairs: tcgen05.mma.cta_group::2 over 256 weight
 *       rows x 128 tokens per pair of CTAs, with a K split when the grid would
 *       leave pairs idle;
 *   5 = tensor cores on CTA pairs with 256-token tiles (prefill M): 256 weight
 *       rows x 256 tokens per pair, M = N = 256 per MMA.
 * Auto selection tries them in that order (5 from MX_PATH5_MIN_M tokens when
 * its tiles fill the device).  2 = the one-CTA tensor-core kernel (128 x 128
 * tiles) is taken only when opts->path asks for it.  Negative mx_status on bad
 * arguments.
 */
int mx_gemm_select_path(const mx_layout* L, int M, const mx_gemm_opts* opts);

/* Smallest M at which automatic selection takes path 5. */
#define MX_PATH5_MIN_M 512

/*
 * mx_gemm -- Y = dequant(Aq, s_a) . dequant(W_packed)^T  (MixLLM section 3.3).
 *   L       host layout of the blob (mx_layout_init / mx_layout_from_header)
 *   blob    device, produced by mx_pack_weights for the same layout
 *   Aq      device int8 [M][K] row-major (dense); s_a device fp16 bits [M]
 *   Y       device fp16 [M][ldy], ldy >= N; column n is original row n of W
 *   workspace / ws_bytes: device scratch, 16-byte aligned, of
 *           mx_gemm_workspace_size(L, M, opts) bytes (NULL if 0).  Path 4 splits
 *           K S > 1 ways only into such a workspace: each split writes fp32 sums
 *           [S][M][N] and a second kernel adds them in split order.  Without it
 *           an automatic split runs unsplit; an asked-for split returns
 *           MX_ERR_WORKSPACE.
 * Per group g: P = sum_{k in g} Aq[m,k] (W_q[n,k] - z[n,g]) exactly in int32
 * (|P| <= 127*127*128 < 2^22), acc[m,n] = sum_g float(P) * s_w[n,g] in fp32,
 * then Y[m,n] = fp16_rn(acc * s_a[m]).  The fp32 summation order depends on the
 * path and split but is fixed for a given configuration (deterministic).
 * M = 0 is a no-op; M <= 65535.
 */
mx_status mx_gemm(const mx_layout* L, const void* blob, const int8_t* Aq, const uint16_t* s_a,
                  int M, uint16_t* Y, int64_t ldy, void* workspace, size_t ws_bytes,
                  const mx_gemm_opts* opts, void* stream);

/*
 * mx_linear_workspace_size -- host only.  Bytes of device scratch mx_linear
 * needs at M tokens of activations of type xdtype: 0 when the call is served by
 * the decode kernel that quantizes X itself, else room for Aq (M*K bytes) and
 * s_a (2*M bytes, or 2*M*G with group-wise scales), each rounded up to 16
 * bytes, followed (from the next 256-byte boundary) by mx_gemm's workspace when
 * it needs one.  Less than that but at least Aq and s_a runs unsplit.
 */
mx_status mx_linear_workspace_size(const mx_layout* L, int M, mx_dtype xdtype,
                                   const mx_gemm_opts* opts, size_t* bytes);

/*
 * mx_linear -- Y = X W^T for a packed layer in one call: per-token 8-bit
 * quantization of X (MixLLM section 3.1.2) followed by the two-step
 * dequantized GEMM (section 3.3).
 *   X       device [M][ldx] fp32 or fp16 (xdtype), rows 16-byte aligned, ldx >= K
 *   Y       device fp16 [M][ldy], ldy >= N; column n is original row n of W
 *   workspace / ws_bytes: device scratch of at least mx_linear_workspace_size
 *           bytes (may be NULL when that is 0)
 * One kernel does both steps on the row path (mx_gemm_select_path == 3: each CTA
 * quantizes the whole token rows it needs) and on the split-K path when M <= 4
 * and the activation rows take at most 64 KB (each CTA takes the row absmax from
 * its cluster and quantizes only its own K slice).  Both use the operations of
 * mx_quant_act, so the codes -- and Y -- are identical to mx_quant_act followed
 * by mx_gemm.  Otherwise mx_quant_act and mx_gemm run back to back on `stream`
 * with Aq and s_a in the workspace.
 * Returns MX_ERR_WORKSPACE if the workspace is missing or too small.
 */
mx_status mx_linear(const mx_layout* L, const void* blob, const void* X, mx_dtype xdtype, int M,
                    int64_t ldx, uint16_t* Y, int64_t ldy, void* workspace, size_t ws_bytes,
                    const mx_gemm_opts* opts, void* stream);

/*
 * MX_NOALLOC_SCRATCH_BYTES -- size of the fixed device array (one per device)
 * that mx_linear_noalloc uses as its scratch: 4 MiB.
 */
#define MX_NOALLOC_SCRATCH_BYTES (4u << 20)

/*
 * mx_linear_noalloc -- mx_linear with no workspace argument and no allocation.
 * The method has no counterpart of this call; it exists for callers that
 * cannot hand out device memory.  Where mx_linear needs scratch (the
 * two-kernel path: Aq of M*K bytes, then s_a of 2*M bytes with one scale per
 * token or 2*M*(K/g) bytes with act_group = g, each rounded up to 16 bytes, as
 * mx_linear_workspace_size reports), this call uses a file-scope device array
 * of MX_NOALLOC_SCRATCH_BYTES bytes instead.  Its address in the calling
 * thread's current device context is looked up with cudaGetSymbolAddress on
 * the first call that needs it on that device and kept for later calls; it is
 * looked up again when the device's context has changed since (after
 * cudaDeviceReset, for example).
 *   Arguments as mx_linear, less workspace and ws_bytes.
 * Nothing in the array has to start at zero: the quantizer writes every byte
 * of it that the GEMM then reads.  The call never allocates or frees device
 * or host memory.
 * A K split of the tensor-core GEMM (see mx_gemm) uses the rest of the array
 * when its sums fit there, else the GEMM runs unsplit: the result is that of
 * mx_linear given a workspace of MX_NOALLOC_SCRATCH_BYTES bytes.
 * Returns MX_ERR_WORKSPACE, before anything is launched, when Aq and s_a
 * exceed MX_NOALLOC_SCRATCH_BYTES; MX_ERR_CUDA when the address lookup fails;
 * otherwise what mx_linear returns.
 * All calls on one device share the one array, so two calls whose kernels can
 * run at the same time (streams with no order between them, or several host
 * threads) race on it; calls in one stream are ordered and safe.  Make the
 * first call on each device outside any stream capture.
 */
mx_status mx_linear_noalloc(const mx_layout* L, const void* blob, const void* X, mx_dtype xdtype, int M,
                            int64_t ldx, uint16_t* Y, int64_t ldy, const mx_gemm_opts* opts,
                            void* stream);

/*
 * mx_saliency -- channel saliency of the global precision search (MixLLM
 * section 3.2: Eq. 4 with the gradient of one calibration batch, as Algorithm 1
 * scores a layer) for every output row of one layer:
 *   dW = dequant(quantize(W)) - W, with the 4-bit asymmetric group quantizer of
 *        mx_pack_weights (the precision a row drops to when it is not chosen),
 *   S1 = sum_k G[n,k] * dW[n,k]  (summed in fp64),
 *   S[n] = |S1 + S1^2 / 2|, rounded to fp32 once.
 *   W, G   device [N][ld] row-major, fp32 or fp16 each (wdtype, gdtype);
 *          G is the loss gradient with respect to W
 *   N, K   rows and columns; group 64 or 128 dividing K
 *   S      device fp32 [N], written
 * The method has no other use for G; the scores feed mx_select_top.  Returns
 * MX_ERR_INVALID_ARG / MX_ERR_UNSUPPORTED on bad arguments before any launch.
 * Asynchronous in `stream`.
 */
mx_status mx_saliency(const void* W, mx_dtype wdtype, int64_t ldw, const void* G, mx_dtype gdtype, int64_t ldg,
                      int N, int K, int group, float* S, void* stream);

/* Bytes of device workspace mx_select_top needs (a fixed few hundred bytes). */
mx_status mx_select_top_workspace_size(int64_t n, size_t* bytes);

/*
 * mx_select_top -- the global choice of Algorithm 1: over the
 * scores S of all layers' rows, concatenated in layer order (n rows in all),
 * is8[i] = 1 for the n_top largest scores and 0 for the rest; ties go to the
 * lower index (the earlier layer, then the lower row).  Exact: a radix select
 * over (score bits, complemented index) keys, deterministic.  The slice of is8
 * of each layer is that layer's mask for mx_pack_weights.
 *   S          device fp32 [n], finite and >= 0 (as mx_saliency writes them)
 *   n, n_top   0 <= n_top <= n < 2^32
 *   is8        device uint8 [n], written
 *   workspace  device, 16-byte aligned, mx_select_top_workspace_size bytes
 * Asynchronous in `stream`.
 */
mx_status mx_select_top(const float* S, int64_t n, int64_t n_top, uint8_t* is8, void* workspace, size_t ws_bytes,
                        void* stream);

/*
 * mx_copy_mapped -- copy `bytes` bytes from src to dst with a kernel, where each
 * of the two may be device memory of the current device or pinned host memory
 * (page-locked and mapped into the device's address space, as cudaHostAlloc
 * and torch's pin_memory give).  The method has no counterpart of this call:
 * it moves a layer's input in and its output out without the copy engines, so
 * that a graph of [copy in, mx_linear, copy out] holds kernels only, and the
 * copy-in kernel lets the next kernel start streaming its weights while the
 * input crosses the bus (programmatic dependent launch).
 *   dst, src  the two buffers; they must not overlap.  The caller guarantees
 *             that both ranges lie inside their allocations.
 *   bytes     0 is a no-op.
 *   stream    cudaStream_t (NULL: the legacy default stream).
 * Reads of host memory bypass the caches (ld.global.cv), so a buffer the host
 * rewrote between two calls is read afresh; writes to host memory are seen by
 * the host once the stream is synchronised.
 * Returns MX_ERR_INVALID_ARG for a NULL pointer, pageable (unregistered) host
 * memory, a host allocation without a device mapping, or another device's
 * memory; MX_ERR_CUDA when the launch fails.  Asynchronous in `stream`.
 */
mx_status mx_copy_mapped(void* dst, const void* src, size_t bytes, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* MX_H */
