// mx_internal.cuh -- device helpers and launch declarations shared by the
// library's translation units (never by the CPU oracle).
#pragma once

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

cudaError_t launch_quant_act(const void* X, mx_dtype xdt, int M, int K, int64_t ldx,
                             int8_t* Aq, uint16_t* s_a, cudaStream_t s);

struct DecodePlan {
    int mt;             // tokens per CTA (1, 2, 4, 8, 16)
    int m_tiles;        // ceil(M / mt)
    int units;          // 2 * t8 + t4: 64-row 8-bit units and 128-row 4-bit units
    int S;              // CTAs per unit = cluster size (split of K)
    int kbu;            // k-blocks per CTA
    bool ok;            // the activation slice fits in shared memory
    size_t smem;        // dynamic shared memory per CTA
};

DecodePlan plan_decode(const mx_layout& L, int M, int split_hint);

cudaError_t launch_gemm_decode(const mx_layout& L, const void* blob, const int8_t* Aq,
                               const uint16_t* s_a, int M, uint16_t* Y, int64_t ldy,
                               const DecodePlan& plan, int32_t* debug_partials, int32_t* status,
                               cudaStream_t s);

cudaError_t launch_gemm_tc(const mx_layout& L, const void* blob, const int8_t* Aq,
                           const uint16_t* s_a, int M, uint16_t* Y, int64_t ldy,
                           int32_t* debug_partials, int32_t* status, uint64_t timeout_ns,
                           int stall_test, cudaStream_t s);

}  // namespace mx
