// quant_act.cu -- per-token 8-bit symmetric activation quantization.
//
// MixLLM section 3.1.2 keeps activations at 8 bits, symmetric; the quantizer is
// the symmetric form of section 2.1 with the restricted range +-127:
//   s_a[m] = fp16(max_k |X[m,k]| / 127)   (0 -> 1, fp16 overflow saturates)
//   Aq[m,k] = clamp(round_half_even(X[m,k] / s_a[m]), -127, 127)
// Every fp32 step is a single IEEE operation (__fdiv_rn, no contraction) so the
// integer codes are decided exactly as the definition states.
//
// act_group: group-wise scales instead (section 3.1.2 says activations are
// quantized group-wise, group 128 as the weights): s_a[m, g] over columns
// g*ag .. (g+1)*ag, the same decisions per group.
//
// One CTA per token row.  Pass 1 reads the row with 16-byte vector loads and
// reduces |x| with warp shuffles and one shared-memory step; pass 2 re-reads
// the row (an L2 hit: the row was just streamed) and writes 8 codes per store.
// HBM traffic is the algorithmic 2 MK (fp16 in) + MK + 2M bytes.
#include "mx_internal.cuh"

namespace mx {
namespace {

constexpr int kThreads = 256;

template <typename T>
__global__ void __launch_bounds__(kThreads)
quant_act_kernel(const T* __restrict__ X, int K, int64_t ldx, int8_t* __restrict__ Aq,
                 __half* __restrict__ s_a) {
    // This grid may be launched as a programmatic dependent of the previous kernel
    // (for example the GEMM that produced X): wait for it before reading anything.
    // Then let the GEMM that consumes Aq launch and start streaming its weights; it
    // waits for this grid to finish before reading Aq.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;");
    const int m = blockIdx.x;
    const T* x = X + int64_t(m) * ldx;
    const int nvec = K / 8;

    float amax = 0.0f;
    for (int i = threadIdx.x; i < nvec; i += kThreads) amax = absmax8(x + i * 8, amax);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    __shared__ float red[kThreads / 32];
    __shared__ float s_shared;
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
    __syncthreads();
    if (threadIdx.x == 0) {
        float a = red[0];
#pragma unroll
        for (int w = 1; w < kThreads / 32; ++w) a = fmaxf(a, red[w]);
        const __half h = act_scale(a);
        s_a[m] = h;
        s_shared = __half2float(h);
    }
    __syncthreads();
    const float s = s_shared, rs = __frcp_rn(s);

    int8_t* q = Aq + int64_t(m) * K;
    for (int i = threadIdx.x; i < nvec; i += kThreads) {
        float v[8];
        load8(x + i * 8, v);
        uint2 out;
        out.x = quant4(v, s, rs);
        out.y = quant4(v + 4, s, rs);
        *reinterpret_cast<uint2*>(q + i * 8) = out;
    }
}

// Group-wise scales (one per token and group of ag columns, ag = 64 or 128): one
// pass.  A group's 8-element chunks sit in ag/8 consecutive lanes, so its absmax
// is a shuffle reduction inside that lane segment; every lane then quantizes the
// eight values it already holds.
template <typename T>
__global__ void __launch_bounds__(kThreads)
quant_act_grouped_kernel(const T* __restrict__ X, int K, int64_t ldx, int ag, int8_t* __restrict__ Aq,
                         __half* __restrict__ s_a) {
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;");
    const int m = blockIdx.x;
    const T* x = X + int64_t(m) * ldx;
    const int nvec = K / 8, cpg = ag / 8, G = K / ag;
    int8_t* q = Aq + int64_t(m) * K;
    for (int i0 = 0; i0 < nvec; i0 += kThreads) {     // same trip count in every lane
        const int i = i0 + threadIdx.x;
        const bool live = i < nvec;
        float v[8];
        if (live) load8(x + i * 8, v);
        else
#pragma unroll
            for (int e = 0; e < 8; ++e) v[e] = 0.0f;
        float amax = 0.0f;
#pragma unroll
        for (int e = 0; e < 8; ++e) amax = fmaxf(amax, fabsf(v[e]));
        for (int o = cpg / 2; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        const __half h = act_scale(amax);
        const float s = __half2float(h), rs = __frcp_rn(s);
        if (live) {
            if (i % cpg == 0) s_a[int64_t(m) * G + i / cpg] = h;
            uint2 out;
            out.x = quant4(v, s, rs);
            out.y = quant4(v + 4, s, rs);
            *reinterpret_cast<uint2*>(q + i * 8) = out;
        }
    }
}

}  // namespace

cudaError_t launch_quant_act_grouped(const void* X, mx_dtype xdt, int M, int K, int64_t ldx, int ag,
                                     int8_t* Aq, uint16_t* s_a, cudaStream_t s) {
    if (M == 0) return cudaSuccess;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(M);
    cfg.blockDim = dim3(kThreads);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    __half* sa = reinterpret_cast<__half*>(s_a);
    if (xdt == MX_F16)
        return cudaLaunchKernelEx(&cfg, quant_act_grouped_kernel<__half>, static_cast<const __half*>(X), K, ldx,
                                  ag, Aq, sa);
    return cudaLaunchKernelEx(&cfg, quant_act_grouped_kernel<float>, static_cast<const float*>(X), K, ldx, ag,
                              Aq, sa);
}

cudaError_t launch_quant_act(const void* X, mx_dtype xdt, int M, int K, int64_t ldx,
                             int8_t* Aq, uint16_t* s_a, cudaStream_t s) {
    if (M == 0) return cudaSuccess;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(M);
    cfg.blockDim = dim3(kThreads);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;   // resident early, waits in-kernel
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    __half* sa = reinterpret_cast<__half*>(s_a);
    if (xdt == MX_F16)
        return cudaLaunchKernelEx(&cfg, quant_act_kernel<__half>, static_cast<const __half*>(X), K, ldx, Aq, sa);
    return cudaLaunchKernelEx(&cfg, quant_act_kernel<float>, static_cast<const float*>(X), K, ldx, Aq, sa);
}

}  // namespace mx
