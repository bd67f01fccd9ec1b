// mx_internal.cuh -- device helpers and launch declarations shared by the
// library's translation units (never by the CPU oracle).
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "mx.h"

namespace mx {

constexpr int kTileRows = MX_TILE_ROWS;       // weight rows per packed tile
constexpr int kKBlock = MX_KBLOCK;            // K columns per packed k-block
constexpr int kBlock8Bytes = kTileRows * kKBlock;       // 16 KB of int8 codes
constexpr int kBlock4Bytes = kTileRows * kKBlock / 2;   //  8 KB of uint4 codes

// Fast int -> float of a value |v| < 2^22 (MixLLM section 3.3, Figure 3): the
// int32 bit pattern of 0x4B400000 + v is the fp32 number 12582912 + v, so one
// integer add and one fp32 subtract replace the conversion instruction.
constexpr uint32_t kI2FBiasBits = 0x4B400000u;
constexpr float kI2FBias = 12582912.0f;

__device__ __forceinline__ float i2f_biased(int32_t v) {
    return __fsub_rn(__int_as_float(int32_t(kI2FBiasBits) + v), kI2FBias);
}

// ---- 8-bit symmetric activation quantizer (MixLLM section 3.1.2; the symmetric
// quantizer of section 2.1 with range +-127).  Shared by the standalone
// quantizer and the GEMM that quantizes its own activation slice, so both take
// every decision with the same IEEE operations.

// eight consecutive elements as fp32 (16-byte aligned)
__device__ __forceinline__ void load8(const __half* p, float (&v)[8]) {
    const uint4 raw = __ldg(reinterpret_cast<const uint4*>(p));
    const __half2* h = reinterpret_cast<const __half2*>(&raw);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 f = __half22float2(h[i]);
        v[2 * i] = f.x;
        v[2 * i + 1] = f.y;
    }
}
__device__ __forceinline__ void load8(const float* p, float (&v)[8]) {
    const float4 a = __ldg(reinterpret_cast<const float4*>(p));
    const float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

// s_a = fp16(amax / 127), saturated at the largest finite fp16, 0 -> 1
__device__ __forceinline__ __half act_scale(float amax) {
    __half h = __float2half_rn(fminf(__fdiv_rn(amax, 127.0f), 65504.0f));
    if (__half2float(h) == 0.0f) h = __float2half_rn(1.0f);
    return h;
}

// One code clamp(round_half_even(fl(x / s)), -127, 127), with fl the IEEE fp32
// division.  t = fl(x * fl(1/s)) is within 1.5 * 2^-23 |t| of fl(x / s) (two
// roundings of at most 2^-24 each), so wherever t is farther than that from a
// half-integer, round(t) is the code; only values closer than 1e-4 to a rounding
// boundary (and NaN) take the IEEE division.  Beyond |t| = 200 both round past
// 127 and clamp alike.  round(t) is t + 1.5 * 2^23 in fp32 (round-half-even to an
// integer for |t| < 2^22), read back from the sum's bits, so no conversion
// instruction is needed on the fast path.
__device__ __forceinline__ int32_t quant_code_exact(float x, float s) {
    return int32_t(fminf(fmaxf(rintf(__fdiv_rn(x, s)), -127.0f), 127.0f));
}

// The fast path without branches; *slow is set when x needs quant_code_exact.
__device__ __forceinline__ int32_t quant_code_fast(float x, float rs, bool* slow) {
    constexpr float kMagic = 12582912.0f;            // 1.5 * 2^23
    const float t = __fmul_rn(x, rs);
    const float tb = __fadd_rn(t, kMagic);
    const float gap = __fsub_rn(0.5f, fabsf(__fsub_rn(t, __fsub_rn(tb, kMagic))));
    const bool big = fabsf(t) > 200.0f;               // false for NaN
    const int32_t q = min(max(__float_as_int(tb) - __float_as_int(kMagic), -127), 127);
    *slow = !big && !(gap > 1.0e-4f);                 // near a boundary, or NaN
    return big ? (t > 0.0f ? 127 : -127) : q;
}

__device__ __forceinline__ int32_t quant_code(float x, float s, float rs) {
    bool slow;
    const int32_t q = quant_code_fast(x, rs, &slow);
    return slow ? quant_code_exact(x, s) : q;
}

// |x| maximum of eight values (exact in the input type; fp16 stays packed)
__device__ __forceinline__ float absmax8(const __half* p, float m) {
    const uint4 raw = *reinterpret_cast<const uint4*>(p);
    const __half2* h = reinterpret_cast<const __half2*>(&raw);
    __half2 a = __hmax2(__habs2(h[0]), __habs2(h[1]));
    a = __hmax2(a, __hmax2(__habs2(h[2]), __habs2(h[3])));
    return fmaxf(m, fmaxf(__low2float(a), __high2float(a)));
}
__device__ __forceinline__ float absmax8(const float* p, float m) {
    const float4 a = *reinterpret_cast<const float4*>(p);
    const float4 b = *reinterpret_cast<const float4*>(p + 4);
    m = fmaxf(m, fmaxf(fmaxf(fabsf(a.x), fabsf(a.y)), fmaxf(fabsf(a.z), fabsf(a.w))));
    return fmaxf(m, fmaxf(fmaxf(fabsf(b.x), fabsf(b.y)), fmaxf(fabsf(b.z), fabsf(b.w))));
}

// four codes packed little-endian; rs = __frcp_rn(s).  One branch for all four,
// taken only when one of them lies at a rounding boundary.
__device__ __forceinline__ uint32_t quant4(const float* v, float s, float rs) {
    bool sl[4];
    int32_t q[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) q[i] = quant_code_fast(v[i], rs, &sl[i]);
    if (sl[0] | sl[1] | sl[2] | sl[3]) {
#pragma unroll
        for (int i = 0; i < 4; ++i)
            if (sl[i]) q[i] = quant_code_exact(v[i], s);
    }
    return (uint32_t(q[0]) & 0xFFu) | ((uint32_t(q[1]) & 0xFFu) << 8) | ((uint32_t(q[2]) & 0xFFu) << 16) |
           (uint32_t(q[3]) << 24);
}

// Byte offset of the 16-byte chunk holding k = 16c..16c+15 of row r inside a
// 128-row x 128-byte block stored with the 128-byte swizzle.
__device__ __forceinline__ int swz128_offset(int r, int c) {
    return r * 128 + ((c ^ (r & 7)) << 4);
}

// Sub-problem geometry as the kernels see it.
struct Geom {
    const uint8_t* blob;
    const int32_t* rowmap;
    const __half* scales8;
    const int8_t* codes8;
    const __half* scales4;
    const uint8_t* zeros4;
    const uint8_t* codes4;
    int N, K, group, G, n8, t8, t4, kblocks;
};

Geom make_geom(const mx_layout& L, const void* blob);

// ---- launchers (host side, one per translation unit) ----
cudaError_t launch_pack(const mx_layout& L, const void* W, mx_dtype wdt, int64_t ldw,
                        const uint8_t* is8, void* blob, int32_t* status, cudaStream_t s);

cudaError_t launch_copy_mapped(void* dst, const void* src, size_t bytes, bool src_host, bool dst_host,
                               cudaStream_t s);

cudaError_t launch_quant_act_grouped(const void* X, mx_dtype xdt, int M, int K, int64_t ldx, int ag,
                                     int8_t* Aq, uint16_t* s_a, cudaStream_t s);
cudaError_t launch_quant_act(const void* X, mx_dtype xdt, int M, int K, int64_t ldx,
                             int8_t* Aq, uint16_t* s_a, cudaStream_t s);

// cuTensorMapEncodeTiled, looked up once through the runtime (no -lcuda)
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn encode_fn(cudaError_t* err);

struct DecodePlan {
    int mt;             // tokens per CTA (1, 2, 4, 8, 16)
    int m_tiles;        // ceil(M / mt)
    int units;          // 2 * t8 + t4: 64-row 8-bit units and 128-row 4-bit units
    int S;              // CTAs per unit = cluster size (split of K)
    int kbu;            // k-blocks per CTA
    int kps;            // k-blocks per ring slot (one copy per operand per slot)
    int ns;             // weight ring slots per CTA
    bool ok;            // the activation slice and the ring fit in shared memory
    size_t smem;        // dynamic shared memory per CTA
    int off_act, off_sa64, off_part, off_raw, off_sag;   // its layout
    bool xfull;         // in-kernel quantization stages whole X rows
};

// x_bytes: 0 when the kernel reads Aq, else 2 / 4 (it stages and quantizes fp16 / fp32 X)
DecodePlan plan_decode(const mx_layout& L, int M, int split_hint, int x_bytes = 0);

// ag (every launch below): 0 -- s_a holds one scale per token; the weight group g --
// s_a holds [M][G] scales per token and group (group-wise activations)
cudaError_t launch_gemm_decode(const mx_layout& L, const void* blob, const int8_t* Aq,
                               const uint16_t* s_a, int M, uint16_t* Y, int64_t ldy,
                               const DecodePlan& plan, int ag, int32_t* debug_partials, int32_t* status,
                               cudaStream_t s);

// decode GEMM for short K (<= 4096) and M <= 4: every CTA owns whole rows (32 4-bit
// or 16 8-bit), no split of K.  Reads Aq / s_a, or quantizes X (fp16 / fp32) itself.
struct RowsPlan {
    bool ok;            // shape served (K, M, one wave, shared memory)
    int mt, m_tiles;    // tokens per CTA (1, 2, 4); ceil(M / mt)
    int n8u, units;     // 8-bit units; all units
    size_t smem;
    int off_sc, off_z, off_act, off_sa64, off_red, off_sag;
};
// the same plan serves Aq, fp16 and fp32 inputs (raw rows are read into registers)
RowsPlan plan_rows(const mx_layout& L, int M);
cudaError_t launch_gemm_rows(const mx_layout& L, const void* blob, const int8_t* Aq, const uint16_t* s_a,
                             const void* X, mx_dtype xdt, int64_t ldx, int M, uint16_t* Y, int64_t ldy,
                             const RowsPlan& p, int ag, int32_t* debug_partials, int32_t* status,
                             cudaStream_t s);

// decode GEMM that quantizes X itself (M <= kMaxFusedTokens): one launch per call
constexpr int kMaxFusedTokens = 4;
bool decode_can_fuse(const mx_layout& L, int M, mx_dtype xdt);
cudaError_t launch_gemm_decode_fused(const mx_layout& L, const void* blob, const void* X, mx_dtype xdt,
                                     int64_t ldx, int M, uint16_t* Y, int64_t ldy, const DecodePlan& plan,
                                     int ag, int32_t* debug_partials, int32_t* status, cudaStream_t s);

cudaError_t launch_gemm_tc(const mx_layout& L, const void* blob, const int8_t* Aq,
                           const uint16_t* s_a, int M, uint16_t* Y, int64_t ldy, int ag,
                           int32_t* debug_partials, int32_t* status, uint64_t timeout_ns,
                           int stall_test, cudaStream_t s);

// the same GEMM on CTA pairs (cta_group::2): 256 weight rows x 128 tokens per tile.
// With S > 1 the stages are split S ways over more units; each split writes fp32
// sums to part [S][M][N] and a second kernel adds them in split order into Y.
constexpr int kTc2MaxSplit = 8;
int tc2_stages(const mx_layout& L);                            // stages of two k-blocks
int tc2_auto_split(const mx_layout& L, int M, int clusters);   // 1 when the grid is full
size_t tc2_split_bytes(const mx_layout& L, int M, int S);      // part's bytes (0 for S = 1)
cudaError_t launch_gemm_tc2(const mx_layout& L, const void* blob, const int8_t* Aq,
                            const uint16_t* s_a, int M, uint16_t* Y, int64_t ldy, int ag, int S,
                            float* part, int32_t* debug_partials, int32_t* status,
                            uint64_t timeout_ns, int stall_test, cudaStream_t s);

// Y[m][n] = fp16(the S fp32 split sums part[k][m][n] added in split order, x s_a[m]) (group-
// wise activation scales were applied per group when ag > 0): the second kernel of a K split
cudaError_t launch_split_reduce(const float* part, int S, int M, int N, const uint16_t* s_a, int ag, uint16_t* Y,
                                int64_t ldy, int sms, cudaStream_t s);

// the same GEMM on CTA pairs with 256-token tiles (cta_group::2, M = N = 256 per MMA):
// two group accumulators of 256 TMEM columns, one-k-block stages
int tc3_units(const mx_layout& L, int M);                       // row-tile pairs x token tiles
cudaError_t launch_gemm_tc3(const mx_layout& L, const void* blob, const int8_t* Aq,
                            const uint16_t* s_a, int M, uint16_t* Y, int64_t ldy, int ag,
                            int32_t* debug_partials, int32_t* status, uint64_t timeout_ns,
                            int stall_test, cudaStream_t s);

// decode-sized M on the tensor cores of one SM each (cta_group::1, 128 weight rows x the
// batch rounded up to 16 tokens): a unit is a row tile and a range of its k-blocks; with
// S > 1 splits the fp32 sums [S][M][N] go to part and launch_split_reduce adds them
constexpr int kTcdMaxM = 128;
constexpr int kTcdMaxSplit = 16;
int tcd_tokens(int M);                                          // the token tile NT
int tcd_auto_split(const mx_layout& L, int M, int sms);
size_t tcd_split_bytes(const mx_layout& L, int M, int S);       // part's bytes (0 for S = 1)
cudaError_t launch_gemm_tcd(const mx_layout& L, const void* blob, const int8_t* Aq, const uint16_t* s_a, int M,
                            uint16_t* Y, int64_t ldy, int ag, int S, float* part, int32_t* debug_partials,
                            int32_t* status, uint64_t timeout_ns, int stall_test, int sms, cudaStream_t s);

}  // namespace mx
