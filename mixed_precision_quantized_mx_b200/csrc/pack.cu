// pack.cu -- offline packing of W into the mixed-precision blob.
//
// MixLLM section 3.1.1 (Figure 1): the salient output rows and the rest form
// independent sub-problems; section 3.3: the weight layout is pre-packed so the
// GEMM never permutes at run time.  Quantizers follow section 2.1:
//   8-bit rows, symmetric:  s = fp16(absmax/127), q = clamp(rint(w/s), -127, 127)
//   4-bit rows, affine:     lo = min(0, min w), hi = max(0, max w),
//                           s = fp16((hi-lo)/15), z = clamp(rint(-lo/s), 0, 15),
//                           q = clamp(rint(w/s) + z, 0, 15)
// with zero scales replaced by 1 and fp16 overflow saturated at 65504.
//
// Kernel 1 (one CTA): the row split -- a block-wide scan of the saliency mask
// gives every row its packed slot (8-bit rows first, each part in ascending
// original order), padding slots get -1; it also writes the blob header.
// Kernel 2: one warp per (slot, group): coalesced reads of the group's values,
// warp-shuffle min/max/absmax, one lane decides (s, z), then the lanes write
// 32-bit words of codes straight into the tile-contiguous layout of mx.h.
#include "mx_internal.cuh"

namespace mx {
namespace {

constexpr int kScanThreads = 1024;

__global__ void __launch_bounds__(kScanThreads)
pack_rowmap_kernel(const uint8_t* __restrict__ is8, int N, int K, int group, int n8, int t8,
                   int t4, int32_t* __restrict__ rowmap, uint32_t* __restrict__ header,
                   int32_t* __restrict__ status) {
    const int slots = (t8 + t4) * kTileRows;
    const int n4 = N - n8;
    for (int i = threadIdx.x; i < slots; i += kScanThreads) rowmap[i] = -1;
    if (threadIdx.x < MX_HEADER_BYTES / 4) {
        uint32_t v = 0;
        switch (threadIdx.x) {
            case 0: v = MX_BLOB_MAGIC; break;
            case 1: v = MX_BLOB_VERSION; break;
            case 2: v = uint32_t(N); break;
            case 3: v = uint32_t(K); break;
            case 4: v = uint32_t(group); break;
            case 5: v = uint32_t(n8); break;
            default: v = 0;
        }
        header[threadIdx.x] = v;
    }
    __syncthreads();

    __shared__ int warp_tot[kScanThreads / 32];
    __shared__ int carry;
    __shared__ int bad;
    if (threadIdx.x == 0) { carry = 0; bad = 0; }
    __syncthreads();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    for (int base = 0; base < N; base += kScanThreads) {
        const int i = base + threadIdx.x;
        const int flag = (i < N && is8[i] != 0) ? 1 : 0;
        // inclusive scan inside the warp
        int v = flag;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int t = __shfl_up_sync(0xffffffffu, v, o);
            if (lane >= o) v += t;
        }
        if (lane == 31) warp_tot[warp] = v;
        __syncthreads();
        if (warp == 0) {
            int w = warp_tot[lane];
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                int t = __shfl_up_sync(0xffffffffu, w, o);
                if (lane >= o) w += t;
            }
            warp_tot[lane] = w;   // inclusive prefix over warps
        }
        __syncthreads();
        const int rank8 = carry + (warp ? warp_tot[warp - 1] : 0) + v - flag;  // exclusive
        if (i < N) {
            if (flag) {
                if (rank8 < n8) rowmap[rank8] = i;
                else bad = 1;
            } else {
                const int rank4 = i - rank8;
                if (rank4 < n4) rowmap[t8 * kTileRows + rank4] = i;
                else bad = 1;
            }
        }
        __syncthreads();
        if (threadIdx.x == 0) carry += warp_tot[31];
        __syncthreads();
    }
    if (threadIdx.x == 0 && status != nullptr && (bad || carry != n8)) *status = MX_ERR_INVALID_ARG;
}

template <typename T> __device__ __forceinline__ float ldf(const T* p);
template <> __device__ __forceinline__ float ldf<float>(const float* p) { return __ldg(p); }
template <> __device__ __forceinline__ float ldf<__half>(const __half* p) {
    return __half2float(__ldg(p));
}

// fp16 scale of an fp32 value: saturate at 65504, zero -> 1
__device__ __forceinline__ __half to_scale(float s32) {
    __half h = __float2half_rn(fminf(s32, 65504.0f));
    if (__half2float(h) == 0.0f) h = __float2half_rn(1.0f);
    return h;
}

constexpr int kPackWarps = 8;

template <typename T>
__global__ void __launch_bounds__(kPackWarps * 32)
pack_quant_kernel(const T* __restrict__ W, int64_t ldw, Geom g) {
    const int lane = threadIdx.x & 31;
    const int slot = blockIdx.x * kPackWarps + (threadIdx.x >> 5);
    const int gi = blockIdx.y;
    const int slots8 = g.t8 * kTileRows;
    if (slot >= (g.t8 + g.t4) * kTileRows) return;
    const bool eight = slot < slots8;
    const int tile = eight ? (slot >> 7) : ((slot - slots8) >> 7);
    const int r = slot & (kTileRows - 1);
    const int orig = g.rowmap[slot];
    const int k0 = gi * g.group;          // first column of the group
    const size_t meta = (size_t(tile) * g.G + gi) * kTileRows + r;

    float amax = 0.0f, lo = 0.0f, hi = 0.0f;
    const T* w = W + (orig >= 0 ? int64_t(orig) * ldw + k0 : 0);
    if (orig >= 0) {
        for (int k = lane; k < g.group; k += 32) {
            float v = ldf(w + k);
            amax = fmaxf(amax, fabsf(v));
            lo = fminf(lo, v);
            hi = fmaxf(hi, v);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
            lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
            hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
        }
    }

    if (eight) {
        __half hs = to_scale(__fdiv_rn(amax, 127.0f));
        const float s = __half2float(hs);
        if (lane == 0) const_cast<__half*>(g.scales8)[meta] = orig >= 0 ? hs : __half(0.0f);
        // one 32-bit word (4 consecutive k) per lane
        const int words = g.group / 4;
        if (lane < words) {
            const int k = k0 + lane * 4;
            uint32_t word = 0;
            if (orig >= 0) {
#pragma unroll
                for (int b = 0; b < 4; ++b) {
                    float q = rintf(__fdiv_rn(ldf(w + lane * 4 + b), s));
                    q = fminf(fmaxf(q, -127.0f), 127.0f);
                    word |= (uint32_t(int32_t(q)) & 0xFFu) << (8 * b);
                }
            }
            const int kb = k / kKBlock, kin = k % kKBlock;
            uint8_t* blk = reinterpret_cast<uint8_t*>(const_cast<int8_t*>(g.codes8)) +
                           (size_t(tile) * g.kblocks + kb) * kBlock8Bytes;
            *reinterpret_cast<uint32_t*>(blk + swz128_offset(r, kin >> 4) + (kin & 15)) = word;
        }
    } else {
        __half hs = to_scale(__fdiv_rn(__fsub_rn(hi, lo), 15.0f));
        const float s = __half2float(hs);
        const float zf = fminf(fmaxf(rintf(__fdiv_rn(-lo, s)), 0.0f), 15.0f);
        if (lane == 0) {
            const_cast<__half*>(g.scales4)[meta] = orig >= 0 ? hs : __half(0.0f);
            const_cast<uint8_t*>(g.zeros4)[meta] = orig >= 0 ? uint8_t(zf) : uint8_t(0);
        }
        // one 32-bit word (8 consecutive k, two nibbles per byte) per lane
        const int words = g.group / 8;
        if (lane < words) {
            const int k = k0 + lane * 8;
            uint32_t word = 0;
            if (orig >= 0) {
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    float q = rintf(__fdiv_rn(ldf(w + lane * 8 + j), s)) + zf;
                    q = fminf(fmaxf(q, 0.0f), 15.0f);
                    const uint32_t code = uint32_t(q);
                    // byte b: low nibble k = 8w+b, high nibble k = 8w+4+b
                    word |= code << ((j & 3) * 8 + (j >> 2) * 4);
                }
            }
            const int kb = k / kKBlock, kin = k % kKBlock;
            uint8_t* blk = const_cast<uint8_t*>(g.codes4) +
                           (size_t(tile) * g.kblocks + kb) * kBlock4Bytes;
            *reinterpret_cast<uint32_t*>(blk + r * 64 + (kin / 8) * 4) = word;
        }
    }
}

}  // namespace

cudaError_t launch_pack(const mx_layout& L, const void* W, mx_dtype wdt, int64_t ldw,
                        const uint8_t* is8, void* blob, int32_t* status, cudaStream_t s) {
    Geom g = make_geom(L, blob);
    pack_rowmap_kernel<<<1, kScanThreads, 0, s>>>(is8, L.N, L.K, L.group, L.n8, L.t8, L.t4,
                                                  const_cast<int32_t*>(g.rowmap),
                                                  static_cast<uint32_t*>(blob), status);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const int slots = (L.t8 + L.t4) * kTileRows;
    dim3 grid((slots + kPackWarps - 1) / kPackWarps, L.G), block(kPackWarps * 32);
    if (wdt == MX_F16)
        pack_quant_kernel<__half><<<grid, block, 0, s>>>(static_cast<const __half*>(W), ldw, g);
    else
        pack_quant_kernel<float><<<grid, block, 0, s>>>(static_cast<const float*>(W), ldw, g);
    return cudaGetLastError();
}

}  // namespace mx
