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

// fp16 scale of an fp32 value: saturate at 65504, zero -> 1 (the packer's rule)
__device__ __forceinline__ float scale16(float s32) {
    __half h = __float2half_rn(fminf(s32, 65504.0f));
    if (__half2float(h) == 0.0f) h = __float2half_rn(1.0f);
    return __half2float(h);
}

// E consecutive elements as fp32: 16-byte vector loads (streaming, read once) when
// kVec, else E scalar loads
template <typename T, int E, bool kVec> struct Vec;
template <int E> struct Vec<float, E, false> {
    static __device__ __forceinline__ void load(const float* p, float (&v)[E]) {
#pragma unroll
        for (int e = 0; e < E; ++e) v[e] = __ldg(p + e);
    }
};
template <int E> struct Vec<__half, E, false> {
    static __device__ __forceinline__ void load(const __half* p, float (&v)[E]) {
#pragma unroll
        for (int e = 0; e < E; ++e) v[e] = __half2float(__ldg(p + e));
    }
};
template <int E> struct Vec<float, E, true> {
    static_assert(E % 4 == 0, "whole float4 loads");
    static __device__ __forceinline__ void load(const float* p, float (&v)[E]) {
#pragma unroll
        for (int j = 0; j < E / 4; ++j) {
            const float4 x = __ldcs(reinterpret_cast<const float4*>(p) + j);
            v[4 * j] = x.x, v[4 * j + 1] = x.y, v[4 * j + 2] = x.z, v[4 * j + 3] = x.w;
        }
    }
};
template <int E> struct Vec<__half, E, true> {
    static_assert(E % 8 == 0, "whole 16-byte loads");
    static __device__ __forceinline__ void load(const __half* p, float (&v)[E]) {
#pragma unroll
        for (int j = 0; j < E / 8; ++j) {
            const uint4 x = __ldcs(reinterpret_cast<const uint4*>(p) + j);
            const uint32_t wv[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
            for (int h = 0; h < 4; ++h) {
                const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&wv[h]));
                v[8 * j + 2 * h] = f.x, v[8 * j + 2 * h + 1] = f.y;
            }
        }
    }
};

// One row is scored by `split` warps (1, 2, 4 or 8), each over a contiguous range of
// groups.  A group of kL * E columns is kL lanes of E consecutive elements, so a warp
// takes 32 / kL groups at a time: the group's range needs log2(kL) shuffle steps and
// its scale and zero point are computed once per E elements of a lane.  U such steps
// are loaded before any is used (U (E of W + E of G) per lane in flight).  The warps'
// fp64 partial sums are added in warp order (deterministic for a shape).
template <typename TW, typename TG, int E, int kL, int U, bool kVec>
__global__ void __launch_bounds__(kSalWarps * 32)
saliency_kernel(const TW* __restrict__ W, int64_t ldw, const TG* __restrict__ G, int64_t ldg, int N, int K,
                int split, float* __restrict__ S) {
    constexpr int kGroup = kL * E, kGPW = 32 / kL;   // columns per group, groups per warp step
    __shared__ double part_sum[kSalWarps];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int slot = warp / split, part = warp % split;
    const int n = blockIdx.x * (kSalWarps / split) + slot;
    const int n_groups = K / kGroup;
    const int per = (n_groups + split - 1) / split;
    const int g_begin = min(n_groups, part * per), g_end = min(n_groups, g_begin + per);
    const int sub = lane / kL;                       // this lane's group within a warp step
    double s1 = 0.0;
    if (n < N) {                                     // warp-uniform
        const TW* w_row = W + int64_t(n) * ldw + (lane % kL) * E;
        const TG* g_row = G + int64_t(n) * ldg + (lane % kL) * E;
        for (int gi = g_begin; gi < g_end; gi += U * kGPW) {
            float w[U][E], gv[U][E];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int grp = gi + u * kGPW + sub;
                if (grp < g_end) {
                    Vec<TW, E, kVec>::load(w_row + int64_t(grp) * kGroup, w[u]);
                    Vec<TG, E, kVec>::load(g_row + int64_t(grp) * kGroup, gv[u]);
                } else {
#pragma unroll
                    for (int e = 0; e < E; ++e) w[u][e] = 0.0f, gv[u][e] = 0.0f;
                }
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                if (gi + u * kGPW >= g_end) break;   // warp-uniform: no group of this step
                const bool valid = gi + u * kGPW + sub < g_end;
                // the group's range (0 included), then its fp16 scale and zero point
                float lo = 0.0f, hi = 0.0f;
#pragma unroll
                for (int e = 0; e < E; ++e) lo = fminf(lo, w[u][e]), hi = fmaxf(hi, w[u][e]);
#pragma unroll
                for (int o = kL / 2; o > 0; o >>= 1) {   // within the group's kL lanes
                    lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
                    hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
                }
                if (!valid) continue;
                const float sc = scale16(__fdiv_rn(__fsub_rn(hi, lo), 15.0f));
                const float zf = fminf(fmaxf(rintf(__fdiv_rn(-lo, sc)), 0.0f), 15.0f);
                const float rc = __frcp_rn(sc);
#pragma unroll
                for (int e = 0; e < E; ++e) {
                    // round(w / s) from w * (1 / s): the two differ by at most 3 2^-24 |w / s|,
                    // so they round alike unless the product is within 2^-11 of a half-integer
                    // (for |w / s| <= 1024; beyond that both clamp alike); there the exact
                    // quotient decides, as in the packer
                    const float t = __fmul_rn(w[u][e], rc);
                    // nearest integer, ties to even: adding and subtracting 1.5 2^23 rounds
                    // exactly for |t| < 2^22 (the adds run on the FMA pipe, where a rounding
                    // instruction would take the conversion unit the fp64 widenings need)
                    float rq = fabsf(t) < 4194304.0f ? __fsub_rn(__fadd_rn(t, 12582912.0f), 12582912.0f) : rintf(t);
                    // |t - rq| is 0.5 exactly at a half-integer, as |frac(t) - 0.5| is 0 there
                    if (fabsf(t) <= 1024.0f && fabsf(fabsf(__fsub_rn(t, rq)) - 0.5f) < 4.8828125e-4f)
                        rq = rintf(__fdiv_rn(w[u][e], sc));
                    const float q = fminf(fmaxf(rq + zf, 0.0f), 15.0f);
                    // (q - z) s is exact in fp32; the difference with w is taken in fp64
                    const double d = double(__fmul_rn(q - zf, sc)) - double(w[u][e]);
                    s1 = fma(double(gv[u][e]), d, s1);
                }
            }
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s1 += __shfl_xor_sync(0xffffffffu, s1, o);
    if (lane == 0) part_sum[warp] = s1;
    __syncthreads();
    if (part == 0 && lane == 0 && n < N) {
        double t = 0.0;
        for (int p = 0; p < split; ++p) t += part_sum[slot * split + p];
        S[n] = float(fabs(t + 0.5 * t * t));
    }
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

template <typename TW, typename TG, int E, int kL, int U>
cudaError_t launch_saliency_t(const void* W, int64_t ldw, const void* G, int64_t ldg, int N, int K, int split,
                              float* S, cudaStream_t s) {
    const TW* w = static_cast<const TW*>(W);
    const TG* g = static_cast<const TG*>(G);
    // vector loads when every row's E-element runs start on 16 bytes
    const bool vec = reinterpret_cast<uintptr_t>(W) % 16 == 0 && (ldw * int64_t(sizeof(TW))) % 16 == 0 &&
                     reinterpret_cast<uintptr_t>(G) % 16 == 0 && (ldg * int64_t(sizeof(TG))) % 16 == 0 &&
                     (E * sizeof(TW)) % 16 == 0 && (E * sizeof(TG)) % 16 == 0;
    const dim3 grid((N + kSalWarps / split - 1) / (kSalWarps / split)), block(kSalWarps * 32);
    if (vec)
        saliency_kernel<TW, TG, E, kL, U, true><<<grid, block, 0, s>>>(w, ldw, g, ldg, N, K, split, S);
    else
        saliency_kernel<TW, TG, E, kL, U, false><<<grid, block, 0, s>>>(w, ldw, g, ldg, N, K, split, S);
    return cudaGetLastError();
}

template <typename TW, typename TG>
cudaError_t launch_saliency_g(const void* W, int64_t ldw, const void* G, int64_t ldg, int N, int K, int group,
                              float* S, cudaStream_t s) {
    // 8 lanes per group (16 elements each at group 128, 8 at 64): four groups per warp
    // step.  Warps per row: enough rows' warps to fill every SM about 32 warps deep,
    // while each warp keeps at least two steps of groups
    constexpr int kL = 8, kGPW = 32 / kL;
    int split = 1;
    while (split < kSalWarps && int64_t(N) * split < 148 * 32 && 2 * split * 2 * kGPW <= K / group) split *= 2;
    return group == 128 ? launch_saliency_t<TW, TG, 16, kL, 2>(W, ldw, G, ldg, N, K, split, S, s)
                        : launch_saliency_t<TW, TG, 8, kL, 4>(W, ldw, G, ldg, N, K, split, S, s);
}

}  // namespace

cudaError_t launch_saliency(const void* W, mx_dtype wdt, int64_t ldw, const void* G, mx_dtype gdt, int64_t ldg,
                            int N, int K, int group, float* S, cudaStream_t s) {
    if (N == 0) return cudaSuccess;
    if (wdt == MX_F16 && gdt == MX_F16) return launch_saliency_g<__half, __half>(W, ldw, G, ldg, N, K, group, S, s);
    if (wdt == MX_F16) return launch_saliency_g<__half, float>(W, ldw, G, ldg, N, K, group, S, s);
    if (gdt == MX_F16) return launch_saliency_g<float, __half>(W, ldw, G, ldg, N, K, group, S, s);
    return launch_saliency_g<float, float>(W, ldw, G, ldg, N, K, group, S, s);
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
