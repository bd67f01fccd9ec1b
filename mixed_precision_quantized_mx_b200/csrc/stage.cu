// stage.cu -- a layer's input in and its output out by kernel: copies where
// either side may be pinned host memory mapped into the device address space.
// Not part of the method; it keeps host-to-host passes free of copy-engine
// hand-offs.
#include "mx_internal.cuh"

namespace mx {
namespace {

constexpr int kThreads = 256;

// Host memory is read with ld.global.cv (no stale cached line survives a host
// rewrite) and written through (st.global.wt).
__device__ __forceinline__ uint4 load16(const uint4* p, bool host) { return host ? __ldcv(p) : __ldcg(p); }
__device__ __forceinline__ void store16(uint4* p, uint4 v, bool host) {
    if (host) __stwt(p, v);
    else __stcg(p, v);
}

__global__ void __launch_bounds__(kThreads) copy_mapped_kernel(uint8_t* dst, const uint8_t* src, size_t bytes,
                                                              bool src_host, bool dst_host) {
    // the next kernel may launch now (it waits for this one before reading dst);
    // this one waits for its predecessor before touching either buffer
    asm volatile("griddepcontrol.launch_dependents;");
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const size_t t0 = size_t(blockIdx.x) * kThreads + threadIdx.x, step = size_t(gridDim.x) * kThreads;
    const bool vec = ((reinterpret_cast<uintptr_t>(dst) | reinterpret_cast<uintptr_t>(src)) & 15) == 0;
    size_t head = 0;
    if (vec) {
        const size_t n16 = bytes / 16;
        const uint4* s = reinterpret_cast<const uint4*>(src);
        uint4* d = reinterpret_cast<uint4*>(dst);
        for (size_t i = t0; i < n16; i += step) store16(d + i, load16(s + i, src_host), dst_host);
        head = n16 * 16;
    }
    for (size_t i = head + t0; i < bytes; i += step) {
        const volatile uint8_t* s = src + i;
        dst[i] = *s;
    }
}

}  // namespace

cudaError_t launch_copy_mapped(void* dst, const void* src, size_t bytes, bool src_host, bool dst_host,
                               cudaStream_t s) {
    if (bytes == 0) return cudaSuccess;
    const bool vec = ((reinterpret_cast<uintptr_t>(dst) | reinterpret_cast<uintptr_t>(src)) & 15) == 0;
    const size_t items = vec ? bytes / 16 + bytes % 16 : bytes;
    const size_t blocks = (items + kThreads - 1) / kThreads;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(unsigned(blocks < 1184 ? blocks : 1184));   // 8 per SM on 148 SMs
    cfg.blockDim = dim3(kThreads);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, copy_mapped_kernel, static_cast<uint8_t*>(dst),
                              static_cast<const uint8_t*>(src), bytes, src_host, dst_host);
}

}  // namespace mx
