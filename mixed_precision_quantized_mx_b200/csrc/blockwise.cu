// blockwise.cu -- block-wise bit widths (ScaleBITS blog page: section 1.2.2, one
// width per 64 x 128 block; section 3.2, block-wise layout with 2-bit metadata)
// on MixLLM's int8 two-step dequantization (section 3.3).
//
// Packing: one warp per (row, column block).  The row's 128 weights in the block
// are one group: a width-b asymmetric quantizer for b < 8 (the packer's fp32
// decisions with 2^b - 1 levels), the symmetric 8-bit one for b = 8 stored in
// offset binary (code q + 128, zero 128).  Lane l quantizes weights 4l .. 4l + 3
// and ORs their 4 b bits into the row's 16 b-byte bit string in shared memory;
// lanes below 4 b then store its words.
//
// GEMM (decode-sized M): one warp per output row, the tokens of one tile of 8 per
// CTA row.  The eight rows of a CTA lie in one block row, whose blocks' widths and
// code offsets the CTA stages in shared memory first; a warp then issues the loads
// of 16 blocks (codes, and the zero points and scales one per lane) before using
// any, so enough bytes are in flight.  Per column block a lane takes codes 4l .. 4l + 3: their 4 b bits come
// from one or two of the row's 4 b words (one coalesced load, two shuffles, a
// funnel shift), are spread into four bytes, and one byte-wise subtract of the
// zero point gives four int8 (q - z) for dp4a with the token's activations.  The
// lane keeps s_w * (its partial) in fp32 per token; one warp sum and s_a at the
// end give Y.  With a partials buffer the exact int32 P[m, n, kb] is also
// reduced and stored.  The CTA's token rows (at most 8 x K bytes) are staged in
// shared memory once when they fit, so no warp waits on L2 for activations inside
// the block loop; otherwise every warp reads them from global memory.
#include <algorithm>

#include "mx_internal.cuh"
#include "mx_blockwise.h"

namespace mx {
namespace {

constexpr int kBR = MX_BW_BLOCK_ROWS;
constexpr int kBC = MX_BW_BLOCK_COLS;
constexpr int kPackWarps = 8;
constexpr int kGemmWarps = 8;
constexpr int kTok = 8;           // tokens per CTA row of the grid
constexpr int kPre = 16;          // column blocks whose loads are issued together (<= 32)

// fp16 scale of an fp32 value: saturate at 65504, zero -> 1 (the packer's rule)
__device__ __forceinline__ float scale16(float s32) {
    __half h = __float2half_rn(fminf(s32, 65504.0f));
    if (__half2float(h) == 0.0f) h = __float2half_rn(1.0f);
    return __half2float(h);
}

__device__ __forceinline__ float ld1(const float* p) { return __ldg(p); }
__device__ __forceinline__ float ld1(const __half* p) { return __half2float(__ldg(p)); }

// width of block bi from the packed 2-bit codes and the table (one byte per entry)
__device__ __forceinline__ int block_width(const uint8_t* meta, int64_t bi, uint32_t table4) {
    const int code = (__ldg(meta + (bi >> 2)) >> (2 * int(bi & 3))) & 3;
    return int(table4 >> (8 * code)) & 0xFF;
}

template <typename T>
__global__ void __launch_bounds__(kPackWarps * 32)
bw_pack_kernel(const T* __restrict__ W, int64_t ldw, int N, int KB, uint32_t table4,
               const uint8_t* __restrict__ meta, const uint32_t* __restrict__ offsets,
               __half* __restrict__ scales, uint8_t* __restrict__ zeros, uint8_t* __restrict__ codes) {
    __shared__ uint32_t words[kPackWarps][32];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t unit = int64_t(blockIdx.x) * kPackWarps + warp;        // n * KB + kb
    if (unit >= int64_t(N) * KB) return;                                  // the whole warp
    const int n = int(unit / KB), kb = int(unit % KB);
    const int rb = n / kBR, r = n % kBR;
    const int64_t bi = int64_t(rb) * KB + kb;
    const int b = block_width(meta, bi, table4);

    const T* w = W + int64_t(n) * ldw + int64_t(kb) * kBC + lane * 4;
    float v[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) v[e] = ld1(w + e);
    uint32_t u[4];
    float sc;
    uint32_t z;
    if (b == 8) {
        float amax = fmaxf(fmaxf(fabsf(v[0]), fabsf(v[1])), fmaxf(fabsf(v[2]), fabsf(v[3])));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        sc = scale16(__fdiv_rn(amax, 127.0f));
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float q = fminf(fmaxf(rintf(__fdiv_rn(v[e], sc)), -127.0f), 127.0f);
            u[e] = uint32_t(int(q) + 128);
        }
        z = 128;
    } else {
        const float qmax = float((1 << b) - 1);
        float lo = 0.0f, hi = 0.0f;
#pragma unroll
        for (int e = 0; e < 4; ++e) lo = fminf(lo, v[e]), hi = fmaxf(hi, v[e]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
            hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
        }
        sc = scale16(__fdiv_rn(__fsub_rn(hi, lo), qmax));
        const float zf = fminf(fmaxf(rintf(__fdiv_rn(-lo, sc)), 0.0f), qmax);
#pragma unroll
        for (int e = 0; e < 4; ++e) u[e] = uint32_t(fminf(fmaxf(rintf(__fdiv_rn(v[e], sc)) + zf, 0.0f), qmax));
        z = uint32_t(zf);
    }
    if (lane == 0) {
        scales[int64_t(n) * KB + kb] = __float2half_rn(sc);     // exact: sc is an fp16 value
        zeros[int64_t(n) * KB + kb] = uint8_t(z);
    }
    // the lane's 4 b bits at bit 4 b l of the row's bit string (4 b <= 32)
    words[warp][lane] = 0;
    __syncwarp();
    const uint32_t packed = u[0] | (u[1] << b) | (u[2] << (2 * b)) | (u[3] << (3 * b));
    const int bit = 4 * b * lane, w0 = bit >> 5, sh = bit & 31;
    atomicOr(&words[warp][w0], packed << sh);
    if (sh + 4 * b > 32) atomicOr(&words[warp][w0 + 1], packed >> (32 - sh));
    __syncwarp();
    uint32_t* dst = reinterpret_cast<uint32_t*>(codes + (size_t(__ldg(offsets + bi)) << 4) + size_t(r) * 16 * b);
    if (lane < 4 * b) dst[lane] = words[warp][lane];
}

template <bool STAGED>
__global__ void __launch_bounds__(kGemmWarps * 32)
bw_gemm_kernel(const uint8_t* __restrict__ codes, const uint32_t* __restrict__ offsets,
               const uint8_t* __restrict__ meta, uint32_t table4, const __half* __restrict__ scales,
               const uint8_t* __restrict__ zeros, const int8_t* __restrict__ Aq, const __half* __restrict__ s_a,
               int M, int N, int K, int KB, __half* __restrict__ Y, int64_t ldy, int32_t* __restrict__ P) {
    // the CTA's rows share one block row: its blocks' widths and code offsets, once
    extern __shared__ uint32_t binfo[];                  // [KB]: offset in 16-byte units | width << 28
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int n0 = blockIdx.x * kGemmWarps;
    const int rb = n0 / kBR;
    const int m0 = blockIdx.y * kTok;
    const int mt = min(kTok, M - m0);
    for (int kb = threadIdx.x; kb < KB; kb += kGemmWarps * 32) {
        const int64_t bi = int64_t(rb) * KB + kb;
        binfo[kb] = __ldg(offsets + bi) | (uint32_t(block_width(meta, bi, table4)) << 28);
    }
    // [mt][K] token codes after the block infos (16-byte aligned)
    int8_t* act = reinterpret_cast<int8_t*>(binfo + ((KB + 3) & ~3));
    if constexpr (STAGED) {
        const int chunks = K / 16;                        // K is a multiple of 128
        for (int i = threadIdx.x; i < mt * chunks; i += kGemmWarps * 32) {
            const int t = i / chunks, c = i % chunks;
            reinterpret_cast<uint4*>(act + int64_t(t) * K)[c] =
                __ldg(reinterpret_cast<const uint4*>(Aq + int64_t(m0 + t) * K) + c);
        }
    }
    __syncthreads();
    const int n = n0 + warp;
    if (n >= N) return;                                   // the whole warp; no block barrier follows
    const int r = n % kBR;
    const int8_t* a_base = (STAGED ? act : Aq + int64_t(m0) * K) + lane * 4;
    const uint8_t* zrow = zeros + int64_t(n) * KB;
    const __half* srow = scales + int64_t(n) * KB;
    float yacc[kTok];
#pragma unroll
    for (int t = 0; t < kTok; ++t) yacc[t] = 0.0f;

    for (int kb0 = 0; kb0 < KB; kb0 += kPre) {
        // issue the loads of up to kPre blocks before using any: each lane below 4 b its
        // word of the block's codes, lane j the zero point and scale of block kb0 + j
        uint32_t mine[kPre];
        const uint32_t zl = kb0 + lane < KB && lane < kPre ? uint32_t(__ldg(zrow + kb0 + lane)) : 0u;
        const float sl = kb0 + lane < KB && lane < kPre ? __half2float(__ldg(srow + kb0 + lane)) : 0.0f;
#pragma unroll
        for (int j = 0; j < kPre; ++j) {
            mine[j] = 0;
            const int kb = kb0 + j;
            if (kb < KB) {                                // warp-uniform
                const uint32_t info = binfo[kb];
                const int b = int(info >> 28);
                const uint32_t* row = reinterpret_cast<const uint32_t*>(
                    codes + (size_t(info & 0x0FFFFFFFu) << 4) + size_t(r) * 16 * b);
                if (lane < 4 * b) mine[j] = __ldg(row + lane);
            }
        }
#pragma unroll
        for (int j = 0; j < kPre; ++j) {
            const int kb = kb0 + j;
            if (kb >= KB) break;                          // warp-uniform
            const int b = int(binfo[kb] >> 28);
            const uint32_t zz = __shfl_sync(0xffffffffu, zl, j) * 0x01010101u;
            const float sw = __shfl_sync(0xffffffffu, sl, j);
            const int bit = 4 * b * lane, w0 = bit >> 5, sh = bit & 31;
            const uint32_t lo_w = __shfl_sync(0xffffffffu, mine[j], w0);
            const uint32_t hi_w = __shfl_sync(0xffffffffu, mine[j], min(w0 + 1, 31));
            const uint32_t x = __funnelshift_r(lo_w, hi_w, sh);
            uint32_t bytes = x;
            if (b < 8) {
                const uint32_t mask = (1u << b) - 1u;
                bytes = (x & mask) | (((x >> b) & mask) << 8) | (((x >> (2 * b)) & mask) << 16) |
                        (((x >> (3 * b)) & mask) << 24);
            }
            const int d = int(__vsub4(bytes, zz));        // four int8 (q - z)
            const int8_t* a = a_base + int64_t(kb) * kBC;
#pragma unroll
            for (int t = 0; t < kTok; ++t) {
                if (t < mt) {                             // warp-uniform
                    const int av = STAGED ? *reinterpret_cast<const int*>(a + int64_t(t) * K)
                                          : __ldg(reinterpret_cast<const int*>(a + int64_t(t) * K));
                    const int p = __dp4a(d, av, 0);
                    yacc[t] = fmaf(sw, float(p), yacc[t]);
                    if (P != nullptr) {
                        int s = p;
#pragma unroll
                        for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
                        if (lane == 0) P[(int64_t(m0 + t) * N + n) * KB + kb] = s;
                    }
                }
            }
        }
    }
#pragma unroll
    for (int t = 0; t < kTok; ++t) {
        if (t < mt) {
            float v = yacc[t];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
            if (lane == 0) Y[int64_t(m0 + t) * ldy + n] = __float2half_rn(v * __half2float(__ldg(s_a + m0 + t)));
        }
    }
}

}  // namespace

cudaError_t launch_bw_pack(const mx_bw_layout& L, const void* W, mx_dtype wdt, int64_t ldw, uint8_t* blob,
                           cudaStream_t s) {
    const uint32_t table4 = uint32_t(L.table[0]) | uint32_t(L.table[1]) << 8 | uint32_t(L.table[2]) << 16 |
                            uint32_t(L.table[3]) << 24;
    const int64_t units = int64_t(L.N) * L.KB;
    const dim3 grid(unsigned((units + kPackWarps - 1) / kPackWarps)), block(kPackWarps * 32);
    const uint8_t* meta = blob + L.off_meta;
    const uint32_t* offs = reinterpret_cast<const uint32_t*>(blob + L.off_offsets);
    __half* sc = reinterpret_cast<__half*>(blob + L.off_scales);
    uint8_t* zr = blob + L.off_zeros;
    uint8_t* cd = blob + L.off_codes;
    if (wdt == MX_F16)
        bw_pack_kernel<__half><<<grid, block, 0, s>>>(static_cast<const __half*>(W), ldw, L.N, L.KB, table4, meta,
                                                      offs, sc, zr, cd);
    else
        bw_pack_kernel<float><<<grid, block, 0, s>>>(static_cast<const float*>(W), ldw, L.N, L.KB, table4, meta,
                                                     offs, sc, zr, cd);
    return cudaGetLastError();
}

cudaError_t launch_bw_gemm(const mx_bw_layout& L, const uint8_t* blob, const int8_t* Aq, const __half* s_a, int M,
                           __half* Y, int64_t ldy, int32_t* P, cudaStream_t s) {
    const uint32_t table4 = uint32_t(L.table[0]) | uint32_t(L.table[1]) << 8 | uint32_t(L.table[2]) << 16 |
                            uint32_t(L.table[3]) << 24;
    const dim3 grid(unsigned((L.N + kGemmWarps - 1) / kGemmWarps), unsigned((M + kTok - 1) / kTok));
    const size_t info = size_t((L.KB + 3) & ~3) * 4;     // the block row's widths and offsets
    if (info > 48 * 1024) return cudaErrorInvalidValue;
    if ((L.code_bytes >> 4) >= (uint64_t(1) << 28)) return cudaErrorInvalidValue;   // offsets packed in 28 bits
    // the token rows of a CTA (up to kTok) staged when they fit: 96 KB leaves two CTAs per SM
    const size_t staged = info + size_t(std::min(M, kTok)) * size_t(L.K);
    const bool stage = staged <= 96 * 1024;
    static bool configured[64] = {};
    int dev = 0;
    cudaError_t e;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!configured[dev]) {
        if ((e = cudaFuncSetAttribute(bw_gemm_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, 96 * 1024)) !=
            cudaSuccess)
            return e;
        configured[dev] = true;
    }
    auto k = stage ? bw_gemm_kernel<true> : bw_gemm_kernel<false>;
    k<<<grid, kGemmWarps * 32, stage ? staged : info, s>>>(
        blob + L.off_codes, reinterpret_cast<const uint32_t*>(blob + L.off_offsets), blob + L.off_meta, table4,
        reinterpret_cast<const __half*>(blob + L.off_scales), blob + L.off_zeros, Aq, s_a, M, L.N, L.K, L.KB, Y, ldy,
        P);
    return cudaGetLastError();
}

}  // namespace mx
