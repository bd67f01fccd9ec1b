// saliency.cu -- the global precision search of MixLLM section 3.2 (Algorithm 1) on
// the GPU: per-row channel saliency of one layer, and the global choice of the
// rows that stay at 8 bits across all layers.
//
// Saliency (Eq. 4 with the gradient of one calibration batch, as Algorithm 1
// scores a layer): for output row n, dW = dequant(quantize(W)) - W with the 4-bit asymmetric
// group quantizer of the packer (the precision a row falls to when it is not
// selected: the same fp32 decisions, so the same codes), S1 = sum_k G[n,k] dW[n,k]
// and S = |S1 + S1^2 / 2|.  One warp per row; the products are summed in fp64 and
// S is rounded to fp32 once.  The kernel reads W and G once: HBM-bound.
//
// Selection (the global choice of Algorithm 1): the n_top largest scores of all layers
// (concatenated) become the 8-bit rows.  Ties go to the lower index, which is
// folded into one 64-bit key per row: the score's bits (a non-negative float's
// bits order like the float), then the complement of the index.  All keys are
// distinct, so the n_top-th largest key T is found exactly by a radix select
// (eight passes of an 8-bit histogram over the keys that match the digits chosen
// so far), and row i is selected iff key(i) >= T.
#include <algorithm>

#include "mx_internal.cuh"

namespace mx {
namespace {

constexpr int kSalWarps = 8;
constexpr int kSelThreads = 256;

template <typename T> __device__ __forceinline__ float ldv(const T* p);
template <> __device__ __forceinline__ float ldv<float>(const float* p) { return __ldg(p); }
template <> __device__ __forceinline__ float ldv<__half>(const __half* p) { return __half2float(__ldg(p)); }

// fp16 scale of an fp32 value: saturate at 65504, zero -> 1 (the packer's rule)
__device__ __forceinline__ float scale16(float s32) {
    __half h = __float2half_rn(fminf(s32, 65504.0f));
    if (__half2float(h) == 0.0f) h = __float2half_rn(1.0f);
    return __half2float(h);
}

template <typename TW, typename TG>
__global__ void __launch_bounds__(kSalWarps * 32)
saliency_kernel(const TW* __restrict__ W, int64_t ldw, const TG* __restrict__ G, int64_t ldg, int N, int K,
                int group, float* __restrict__ S) {
    const int lane = threadIdx.x & 31;
    const int n = blockIdx.x * kSalWarps + (threadIdx.x >> 5);
    if (n >= N) return;
    const TW* w = W + int64_t(n) * ldw;
    const TG* gr = G + int64_t(n) * ldg;
    double s1 = 0.0;
    for (int k0 = 0; k0 < K; k0 += group) {
        // the group's range, then its fp16 scale and zero point
        float lo = 0.0f, hi = 0.0f;
        for (int k = lane; k < group; k += 32) {
            const float v = ldv(w + k0 + k);
            lo = fminf(lo, v);
            hi = fmaxf(hi, v);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
            hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
        }
        const float s = scale16(__fdiv_rn(__fsub_rn(hi, lo), 15.0f));
        const float zf = fminf(fmaxf(rintf(__fdiv_rn(-lo, s)), 0.0f), 15.0f);
        for (int k = lane; k < group; k += 32) {
            const float v = ldv(w + k0 + k);
            const float q = fminf(fmaxf(rintf(__fdiv_rn(v, s)) + zf, 0.0f), 15.0f);
            const double d = double(__fmul_rn(q - zf, s)) - double(v);   // (q - z) s is exact in fp32
            s1 = fma(double(ldv(gr + k0 + k)), d, s1);
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s1 += __shfl_xor_sync(0xffffffffu, s1, o);
    if (lane == 0) S[n] = float(fabs(s1 + 0.5 * s1 * s1));
}

// 64-bit key of row i: score bits, then the complemented index (ties: lower first)
__device__ __forceinline__ uint64_t sel_key(const float* S, int64_t i) {
    return (uint64_t(__float_as_uint(S[i])) << 32) | uint64_t(0xFFFFFFFFu - uint32_t(i));
}

struct SelState {
    uint64_t prefix;        // digits of T chosen so far
    uint64_t above;         // keys known to be above the prefix's range
    uint32_t hist[256];
};

// histogram of digit `shift` over the keys whose higher digits equal the prefix's
__global__ void __launch_bounds__(kSelThreads)
select_hist_kernel(const float* __restrict__ S, int64_t n, int shift, SelState* st) {
    __shared__ uint32_t h[256];
    for (int b = threadIdx.x; b < 256; b += kSelThreads) h[b] = 0;
    __syncthreads();
    const uint64_t hi_mask = shift >= 56 ? 0 : ~uint64_t(0) << (shift + 8);
    const uint64_t want = st->prefix & hi_mask;
    for (int64_t i = int64_t(blockIdx.x) * kSelThreads + threadIdx.x; i < n; i += int64_t(gridDim.x) * kSelThreads) {
        const uint64_t k = sel_key(S, i);
        if ((k & hi_mask) == want) atomicAdd(&h[(k >> shift) & 255], 1u);
    }
    __syncthreads();
    for (int b = threadIdx.x; b < 256; b += kSelThreads)
        if (h[b]) atomicAdd(&st->hist[b], h[b]);
}

// choose digit `shift` of T: the bucket holding the (n_top - above)-th largest key
__global__ void select_pick_kernel(int64_t n_top, int shift, SelState* st) {
    uint64_t cum = st->above;
    int pick = 0;
    for (int b = 255; b >= 0; --b) {
        const uint64_t c = st->hist[b];
        if (cum + c >= uint64_t(n_top)) {
            pick = b;
            break;
        }
        cum += c;
    }
    st->above = cum;
    st->prefix |= uint64_t(pick) << shift;
    for (int b = 0; b < 256; ++b) st->hist[b] = 0;
}

__global__ void __launch_bounds__(kSelThreads)
select_mark_kernel(const float* __restrict__ S, int64_t n, int64_t n_top, const SelState* st,
                   uint8_t* __restrict__ is8) {
    const uint64_t T = st->prefix;
    for (int64_t i = int64_t(blockIdx.x) * kSelThreads + threadIdx.x; i < n; i += int64_t(gridDim.x) * kSelThreads)
        is8[i] = n_top >= n ? 1 : (n_top == 0 ? 0 : (sel_key(S, i) >= T ? 1 : 0));
}

}  // namespace

cudaError_t launch_saliency(const void* W, mx_dtype wdt, int64_t ldw, const void* G, mx_dtype gdt, int64_t ldg,
                            int N, int K, int group, float* S, cudaStream_t s) {
    if (N == 0) return cudaSuccess;
    const dim3 grid((N + kSalWarps - 1) / kSalWarps), block(kSalWarps * 32);
    if (wdt == MX_F16 && gdt == MX_F16)
        saliency_kernel<__half, __half><<<grid, block, 0, s>>>(static_cast<const __half*>(W), ldw,
                                                              static_cast<const __half*>(G), ldg, N, K, group, S);
    else if (wdt == MX_F16)
        saliency_kernel<__half, float><<<grid, block, 0, s>>>(static_cast<const __half*>(W), ldw,
                                                             static_cast<const float*>(G), ldg, N, K, group, S);
    else if (gdt == MX_F16)
        saliency_kernel<float, __half><<<grid, block, 0, s>>>(static_cast<const float*>(W), ldw,
                                                             static_cast<const __half*>(G), ldg, N, K, group, S);
    else
        saliency_kernel<float, float><<<grid, block, 0, s>>>(static_cast<const float*>(W), ldw,
                                                            static_cast<const float*>(G), ldg, N, K, group, S);
    return cudaGetLastError();
}

size_t select_workspace_bytes() { return (sizeof(SelState) + 255) & ~size_t(255); }

cudaError_t launch_select_top(const float* S, int64_t n, int64_t n_top, uint8_t* is8, void* workspace,
                              cudaStream_t s) {
    if (n == 0) return cudaSuccess;
    SelState* st = static_cast<SelState*>(workspace);
    cudaError_t e = cudaMemsetAsync(st, 0, sizeof(SelState), s);
    if (e != cudaSuccess) return e;
    const int blocks = int(std::min<int64_t>((n + kSelThreads - 1) / kSelThreads, 148 * 4));
    if (n_top > 0 && n_top < n) {
        for (int shift = 56; shift >= 0; shift -= 8) {
            select_hist_kernel<<<blocks, kSelThreads, 0, s>>>(S, n, shift, st);
            select_pick_kernel<<<1, 1, 0, s>>>(n_top, shift, st);
        }
    }
    select_mark_kernel<<<blocks, kSelThreads, 0, s>>>(S, n, n_top, st, is8);
    return cudaGetLastError();
}

}  // namespace mx
