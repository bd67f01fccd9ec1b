// gemm_decode.cu -- decode-sized mixed-precision GEMM (a few tokens, HBM-bound).
//
// Two-step dequantization of MixLLM section 3.3 on CUDA cores:
//   step 1: per group, P = sum_k Aq[m,k] (W_q[n,k] - z[n,g]) in exact int32
//           (dp4a on the int8 codes / the uint4 codes, which are valid int8
//           operands as they are),
//   step 2: acc[m,n] += float(P) s_w[n,g] in fp32 with the fast int-to-float of
//           section 3.3 (Figure 3); Y = fp16(acc s_a[m]) at the end.
// For 4-bit rows the zero point is folded out of the dot product:
//   sum (q - z) a = sum q a - z sum a,
// with the activation sums of every 64-column half-block computed once per CTA.
//
// Work split.  A "unit" is 128 packed 4-bit rows, or 64 packed 8-bit rows (an
// 8-bit tile is two units), so every unit streams 8 KB of codes per 128-column
// k-block.  The S CTAs that split one unit's K range form a thread-block
// cluster: each streams its k-blocks, leaves its per-row partial sums in shared
// memory, and after a cluster barrier rank 0 adds the S partials in rank order
// (deterministic) through distributed shared memory, applies s_a and scatters
// the rows to their original columns of Y (section 3.3, fused scatter).  No
// workspace and no second kernel.
//
// The kernel is launched as a programmatic dependent of the activation
// quantizer: its weight, scale and zero-point loads are in flight before
// griddepcontrol.wait, which it passes only once the quantized activations exist.
// It lets its own dependents launch at once, so the next step's quantizer is
// resident (and waiting) when this kernel finishes.
#include <algorithm>
#include <cooperative_groups.h>
#include <type_traits>

#include "mx_internal.cuh"

namespace mx {
namespace {

namespace cg = cooperative_groups;

constexpr int kThreads = 256;
constexpr int kBatch = 4;                  // k-blocks whose code loads are in flight together
constexpr int kMaxActSmem = 64 * 1024;     // activation slice staged in shared memory
constexpr int kMaxSmem = 200 * 1024;       // activation slice + partial sums of all ranks
constexpr int kMaxCluster = 8;             // portable cluster size

struct DecArgs {
    Geom g;
    const int8_t* Aq;      // quantized activations (when the kernel is not fed X)
    const __half* s_a;
    const void* X;         // raw activations fp16 / fp32 (when it quantizes them itself)
    int64_t ldx;
    __half* Y;
    int64_t ldy;
    int M;
    int S;            // CTAs per unit (cluster size)
    int kbu;          // k-blocks per CTA
    int32_t* debug;
    int32_t* status;  // MX_ERR_TIMEOUT if the reduction wait ran out (never expected)
};

__device__ __forceinline__ uint4 ldg_stream(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

__device__ __forceinline__ int dp4a(uint32_t a, uint32_t b, int c) {
    return __dp4a(int(a), int(b), c);
}

__device__ __forceinline__ void griddep_wait() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// the same shared-memory address in CTA `rank` of this cluster
__device__ __forceinline__ uint32_t map_rank(uint32_t addr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
    return r;
}

__device__ __forceinline__ void st_cluster_f32(uint32_t addr, float v) {
    asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(addr), "f"(v) : "memory");
}

// arrive on an mbarrier of another CTA of the cluster, releasing this CTA's
// earlier writes to the cluster
__device__ __forceinline__ void mbar_arrive_remote(uint32_t remote_bar) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(remote_bar) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait_cluster(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok) : "r"(smem_addr(bar)), "r"(parity) : "memory");
    return ok != 0;
}

__device__ __forceinline__ uint64_t globaltimer() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// resident CTAs per SM each variant is compiled for (register budget)
__host__ __device__ constexpr int decode_ctas_per_sm(int mt, int nb) {
    return mt >= 16 ? 1 : (mt <= 2 && nb == 1) ? 3 : 2;
}

// NB: register buffers of kBatch k-blocks (2 = the next batch streams while one
// is computed; 1 when a CTA's whole K range is a single batch).
// XT: void -- read Aq and s_a produced by the activation quantizer; __half or
// float -- read X and quantize in-kernel: each CTA takes the absmax of the whole
// row (the scale needs all K) and quantizes only its own K slice into shared
// memory, with the quantizer's own device code, so the codes are identical.
template <int MT, int NB, bool DEBUG, typename XT>
__global__ void __launch_bounds__(kThreads, decode_ctas_per_sm(MT, NB))
gemm_decode_kernel(const __grid_constant__ DecArgs a) {
    extern __shared__ __align__(16) uint8_t smem[];
    const Geom& g = a.g;
    cg::cluster_group cluster = cg::this_cluster();
    const int rank = int(cluster.block_rank());
    const int unit = blockIdx.x / a.S;
    const bool eight = unit < 2 * g.t8;
    const int tile = eight ? unit >> 1 : unit - 2 * g.t8;
    const int rows = eight ? 64 : 128;
    const int row0 = eight ? (unit & 1) * 64 : 0;          // first row of the unit in its tile
    const int kb0 = rank * a.kbu;
    const int kb1 = min(kb0 + a.kbu, g.kblocks);
    const int nkb = max(kb1 - kb0, 0);
    const int m0 = blockIdx.y * MT;
    const int tid = threadIdx.x;

    // thread -> (row, 32-byte slice of a k-block row)
    int r, sub;
    if (eight) { r = row0 + (tid >> 2); sub = tid & 3; }   // 4 slices of 32 B per 128-B row
    else { r = tid >> 1; sub = tid & 1; }                   // 2 slices of 32 B per 64-B row
    const uint8_t* wbase = eight
        ? reinterpret_cast<const uint8_t*>(g.codes8) + size_t(tile) * g.kblocks * kBlock8Bytes + r * 128 + sub * 32
        : g.codes4 + size_t(tile) * g.kblocks * kBlock4Bytes + r * 64 + sub * 32;
    const size_t wstride = eight ? kBlock8Bytes : kBlock4Bytes;
    // logical 16-column chunks held by this thread (the 8-bit rows are stored swizzled)
    const int lc0 = eight ? (2 * sub) ^ (r & 7) : 4 * sub;
    const int lc1 = eight ? (2 * sub + 1) ^ (r & 7) : 4 * sub + 2;   // 4-bit: second 32 codes
    const size_t meta_base = size_t(tile) * g.G * kTileRows + r;
    const __half* scales = eight ? g.scales8 : g.scales4;

    // the next kernel (the following step's activation quantizer) may become
    // resident now; it waits for this grid to complete before it reads anything
    asm volatile("griddepcontrol.launch_dependents;");

    // ---- loads that do not depend on the previous kernel: codes, scales, zeros.
    // Two register buffers of kBatch k-blocks: batch i+1 is in flight while batch i
    // is computed.
    uint4 w[NB][kBatch][2];
    __half sw[NB][kBatch];
    uint8_t zw[NB][kBatch];
    auto load_batch = [&](int buf, int kbb) {
#pragma unroll
        for (int u = 0; u < kBatch; ++u)
            if (kbb + u < kb1) {
                const int kb = kbb + u;
                w[buf][u][0] = ldg_stream(wbase + size_t(kb) * wstride);
                w[buf][u][1] = ldg_stream(wbase + size_t(kb) * wstride + 16);
                const size_t gi = size_t((kb * kKBlock + lc0 * 16) / g.group);
                sw[buf][u] = scales[meta_base + gi * kTileRows];
                zw[buf][u] = eight ? uint8_t(0) : g.zeros4[meta_base + gi * kTileRows];
            }
    };
    load_batch(0, kb0);
    if (NB > 1 && kb0 + kBatch < kb1) load_batch(NB - 1, kb0 + kBatch);

    // rank 0 collects the partial sums: its barrier must exist before anyone arrives
    __shared__ uint64_t red_bar;
    if (tid == 0) {
        asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(&red_bar)), "r"(max(a.S - 1, 1)));
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    cluster.sync();
    griddep_wait();

    const int rowb = a.kbu * kKBlock;
    int8_t* act = reinterpret_cast<int8_t*>(smem);
    int32_t* sa64 = reinterpret_cast<int32_t*>(smem + size_t(MT) * rowb);
    // partial sums of every rank, [S][MT][128]; only rank 0's copy is used
    float* part = reinterpret_cast<float*>(smem + size_t(MT) * rowb + size_t(MT) * 2 * a.kbu * 4);
    __shared__ float sa_loc[MT];              // token scales quantized in-kernel
    if constexpr (std::is_void_v<XT>) {
        // ---- stage Aq[m0 .. m0+MT)[kb0*128 .. kb1*128) (zero rows beyond M)
        const int chunks = nkb * (kKBlock / 16);
        for (int i = tid; i < MT * chunks; i += kThreads) {
            const int j = i / chunks, c = i % chunks;
            uint4 v = make_uint4(0, 0, 0, 0);
            if (m0 + j < a.M)
                v = __ldg(reinterpret_cast<const uint4*>(a.Aq + int64_t(m0 + j) * g.K + kb0 * kKBlock) + c);
            *reinterpret_cast<uint4*>(act + j * rowb + c * 16) = v;
        }
    } else {
        // ---- per-token absmax over the whole row, then this CTA's slice quantized
        const XT* X = static_cast<const XT*>(a.X);
        __shared__ float red[kThreads / 32][MT];
        float am[MT];
#pragma unroll
        for (int j = 0; j < MT; ++j) {
            am[j] = 0.0f;
            if (m0 + j < a.M) {
                const XT* x = X + int64_t(m0 + j) * a.ldx;
                for (int v = tid; v < g.K / 8; v += kThreads) {
                    float f[8];
                    load8(x + v * 8, f);
#pragma unroll
                    for (int e = 0; e < 8; ++e) am[j] = fmaxf(am[j], fabsf(f[e]));
                }
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) am[j] = fmaxf(am[j], __shfl_xor_sync(0xffffffffu, am[j], o));
            if ((tid & 31) == 0) red[tid >> 5][j] = am[j];
        }
        __syncthreads();
        if (tid < MT) {
            float m = red[0][tid];
#pragma unroll
            for (int w = 1; w < kThreads / 32; ++w) m = fmaxf(m, red[w][tid]);
            sa_loc[tid] = __half2float(act_scale(m));
        }
        __syncthreads();
        const int units8 = nkb * (kKBlock / 8);
        for (int i = tid; i < MT * units8; i += kThreads) {
            const int j = i / units8, c = i % units8;
            uint2 o = make_uint2(0, 0);
            if (m0 + j < a.M) {
                float f[8];
                load8(X + int64_t(m0 + j) * a.ldx + kb0 * kKBlock + c * 8, f);
                o.x = quant4(f, sa_loc[j]);
                o.y = quant4(f + 4, sa_loc[j]);
            }
            *reinterpret_cast<uint2*>(act + j * rowb + c * 8) = o;
        }
    }
    __syncthreads();
    if (!eight) {
        for (int i = tid; i < MT * nkb * 2; i += kThreads) {
            const int j = i / (nkb * 2), hb = i % (nkb * 2);
            const uint4* p = reinterpret_cast<const uint4*>(act + j * rowb + hb * 64);
            int s = 0;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const uint4 v = p[c];
                s = dp4a(v.x, 0x01010101u, s);
                s = dp4a(v.y, 0x01010101u, s);
                s = dp4a(v.z, 0x01010101u, s);
                s = dp4a(v.w, 0x01010101u, s);
            }
            sa64[j * 2 * a.kbu + hb] = s;
        }
        __syncthreads();
    }

    const int slot = eight ? tile * kTileRows + r : (g.t8 + tile) * kTileRows + r;
    const int orig = DEBUG ? g.rowmap[slot] : 0;
    float out[MT];
#pragma unroll
    for (int j = 0; j < MT; ++j) out[j] = 0.0f;

    auto compute_batch = [&](int buf, int kbb) {
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            const int kb = kbb + u;
            if (kb >= kb1) break;
            const int kl = kb - kb0;
            const int gi = (kb * kKBlock + lc0 * 16) / g.group;
            const float s = __half2float(sw[buf][u]);
            int acc[MT];
#pragma unroll
            for (int j = 0; j < MT; ++j) acc[j] = 0;
            if (eight) {
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                    const int lc = i ? lc1 : lc0;
#pragma unroll
                    for (int j = 0; j < MT; ++j) {
                        const uint4 av = *reinterpret_cast<const uint4*>(act + j * rowb + kl * kKBlock + lc * 16);
                        acc[j] = dp4a(w[buf][u][i].x, av.x, acc[j]);
                        acc[j] = dp4a(w[buf][u][i].y, av.y, acc[j]);
                        acc[j] = dp4a(w[buf][u][i].z, av.z, acc[j]);
                        acc[j] = dp4a(w[buf][u][i].w, av.w, acc[j]);
                    }
                }
                // threads holding the same group: the 4 slices of a row (g = 128) or the two
                // slices of one logical half (g = 64)
#pragma unroll
                for (int j = 0; j < MT; ++j) {
                    acc[j] += __shfl_xor_sync(0xffffffffu, acc[j], 1);
                    if (g.group == 128) acc[j] += __shfl_xor_sync(0xffffffffu, acc[j], 2);
                }
            } else {
                const int z = zw[buf][u];
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                    const uint32_t wd[4] = {w[buf][u][i].x, w[buf][u][i].y, w[buf][u][i].z, w[buf][u][i].w};
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const uint32_t lo = wd[q] & 0x0F0F0F0Fu;          // k = 8w .. 8w+3
                        const uint32_t hi = (wd[q] >> 4) & 0x0F0F0F0Fu;   // k = 8w+4 .. 8w+7
                        const int koff = sub * 64 + i * 32 + q * 8;
#pragma unroll
                        for (int j = 0; j < MT; ++j) {
                            const uint2 av = *reinterpret_cast<const uint2*>(act + j * rowb + kl * kKBlock + koff);
                            acc[j] = dp4a(lo, av.x, acc[j]);
                            acc[j] = dp4a(hi, av.y, acc[j]);
                        }
                    }
                }
#pragma unroll
                for (int j = 0; j < MT; ++j) {
                    acc[j] -= z * sa64[j * 2 * a.kbu + kl * 2 + sub];
                    if (g.group == 128) acc[j] += __shfl_xor_sync(0xffffffffu, acc[j], 1);
                }
            }
#pragma unroll
            for (int j = 0; j < MT; ++j) out[j] = __fmaf_rn(i2f_biased(acc[j]), s, out[j]);
            if (DEBUG && orig >= 0) {
                const bool writer = eight ? (g.group == 128 ? sub == 0 : (sub & 1) == 0)
                                          : (g.group == 128 ? sub == 0 : true);
                if (writer) {
#pragma unroll
                    for (int j = 0; j < MT; ++j)
                        if (m0 + j < a.M) a.debug[(size_t(m0 + j) * g.N + orig) * g.G + gi] = acc[j];
                }
            }
        }
    };
    if (NB == 1) {
        compute_batch(0, kb0);                  // the whole range is one batch
    } else {
        // unrolled by two so both register buffers are indexed with constants
        for (int kbb = kb0; kbb < kb1; kbb += 2 * kBatch) {
            compute_batch(0, kbb);
            if (kbb + 2 * kBatch < kb1) load_batch(0, kbb + 2 * kBatch);
            if (kbb + kBatch < kb1) compute_batch(NB - 1, kbb + kBatch);
            if (kbb + 3 * kBatch < kb1) load_batch(NB - 1, kbb + 3 * kBatch);
        }
    }
    // with g = 64 the slices of a row hold different groups: add them up
    if (g.group == 64) {
#pragma unroll
        for (int j = 0; j < MT; ++j)
            out[j] = __fadd_rn(out[j], __shfl_xor_sync(0xffffffffu, out[j], eight ? 2 : 1));
    }
    const bool lead = sub == 0;
    const int rl = r - row0;                       // row within the unit
    if (rank != 0) {
        // push this CTA's partials into rank 0's slot `rank`, then arrive there
        if (lead) {
            const uint32_t dst = map_rank(smem_addr(part + (size_t(rank) * MT) * 128 + rl), 0);
#pragma unroll
            for (int j = 0; j < MT; ++j) st_cluster_f32(dst + j * 128 * 4, out[j]);
        }
        __syncthreads();
        if (tid == 0) mbar_arrive_remote(map_rank(smem_addr(&red_bar), 0));
        return;
    }
    if (lead) {
#pragma unroll
        for (int j = 0; j < MT; ++j) part[j * 128 + rl] = out[j];
    }
    // rank 0: wait (bounded) for the S-1 other partials, then add them in rank order
    bool ok = true;
    if (a.S > 1) {
        if (tid == 0) {
            const uint64_t t0 = globaltimer();
            while (!mbar_try_wait_cluster(&red_bar, 0)) {
                if (globaltimer() - t0 > 2000000000ull) {
                    ok = false;
                    if (a.status) atomicExch(a.status, MX_ERR_TIMEOUT);
                    break;
                }
            }
        }
    }
    ok = __syncthreads_and(ok);
    if (!ok) return;
    for (int i = tid; i < MT * rows; i += kThreads) {
        const int j = i / rows, rr = i % rows;
        if (m0 + j >= a.M) continue;
        float sum = 0.0f;
        for (int q = 0; q < a.S; ++q) sum = __fadd_rn(sum, part[(size_t(q) * MT + j) * 128 + rr]);
        const int sl = eight ? tile * kTileRows + row0 + rr : (g.t8 + tile) * kTileRows + rr;
        const int o = g.rowmap[sl];
        float sa;
        if constexpr (std::is_void_v<XT>) sa = __half2float(a.s_a[m0 + j]);
        else sa = sa_loc[j];
        if (o >= 0) a.Y[int64_t(m0 + j) * a.ldy + o] = __float2half_rn(__fmul_rn(sum, sa));
    }
}

int ceil_div(int a, int b) { return (a + b - 1) / b; }

template <int MT, int NB, bool DEBUG, typename XT>
cudaError_t launch_t(const DecArgs& args, int units, int m_tiles, size_t smem, cudaStream_t s) {
    auto k = gemm_decode_kernel<MT, NB, DEBUG, XT>;
    static bool configured[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!configured[dev]) {
        e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxSmem);
        if (e != cudaSuccess) return e;
        configured[dev] = true;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(units * args.S, m_tiles);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = args.S;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, k, args);
}

template <int MT, bool DEBUG, typename XT>
cudaError_t launch_nb(const DecArgs& a, int units, int m_tiles, size_t smem, cudaStream_t s) {
    return a.kbu <= kBatch ? launch_t<MT, 1, DEBUG, XT>(a, units, m_tiles, smem, s)
                           : launch_t<MT, 2, DEBUG, XT>(a, units, m_tiles, smem, s);
}

template <bool DEBUG>
cudaError_t launch_mt(const DecArgs& a, int mt, int units, int m_tiles, size_t smem, cudaStream_t s) {
    switch (mt) {
        case 1: return launch_nb<1, DEBUG, void>(a, units, m_tiles, smem, s);
        case 2: return launch_nb<2, DEBUG, void>(a, units, m_tiles, smem, s);
        case 4: return launch_nb<4, DEBUG, void>(a, units, m_tiles, smem, s);
        case 8: return launch_nb<8, DEBUG, void>(a, units, m_tiles, smem, s);
        default: return launch_nb<16, DEBUG, void>(a, units, m_tiles, smem, s);
    }
}

// in-kernel quantization of X: up to four tokens per CTA
template <bool DEBUG, typename XT>
cudaError_t launch_mt_fused(const DecArgs& a, int mt, int units, int m_tiles, size_t smem, cudaStream_t s) {
    switch (mt) {
        case 1: return launch_nb<1, DEBUG, XT>(a, units, m_tiles, smem, s);
        case 2: return launch_nb<2, DEBUG, XT>(a, units, m_tiles, smem, s);
        case 4: return launch_nb<4, DEBUG, XT>(a, units, m_tiles, smem, s);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

DecodePlan plan_decode(const mx_layout& L, int M, int split_hint) {
    DecodePlan p{};
    p.mt = M <= 1 ? 1 : M <= 2 ? 2 : M <= 4 ? 4 : M <= 8 ? 8 : 16;
    p.m_tiles = std::max(1, ceil_div(M, p.mt));
    p.units = 2 * L.t8 + L.t4;
    const int kb = L.kblocks;
    // at least as many CTAs per unit as the activation slice needs to fit in shared memory
    const int s_min = ceil_div(kb * p.mt * kKBlock, kMaxActSmem);
    // fill the resident capacity of a 148-SM B200 once (clusters of up to 8 CTAs
    // must also pack into GPCs, so aim a little below it); the single-batch
    // variant keeps three CTAs per SM resident
    int S = split_hint;
    if (S <= 0) {
        const int work = std::max(1, p.units * p.m_tiles);
        const int s1 = ceil_div(decode_ctas_per_sm(p.mt, 1) * 148 * 7 / 8, work);
        if (ceil_div(kb, s1) <= kBatch) {
            S = s1;
        } else {
            // long K ranges: at most ~32 k-blocks per CTA, so several waves of CTAs
            // keep enough loads in flight
            S = std::max(ceil_div(decode_ctas_per_sm(p.mt, 2) * 148 * 7 / 8, work), ceil_div(kb, 32));
        }
    }
    S = std::max(S, s_min);
    S = std::min(S, std::min(kMaxCluster, kb));
    p.S = S;
    p.kbu = ceil_div(kb, S);
    p.ok = S >= s_min && p.kbu * p.mt * kKBlock <= kMaxActSmem;
    p.smem = size_t(p.mt) * p.kbu * kKBlock + size_t(p.mt) * 2 * p.kbu * 4 + size_t(S) * p.mt * 128 * 4;
    p.ok = p.ok && p.smem <= size_t(kMaxSmem);
    return p;
}

cudaError_t launch_gemm_decode(const mx_layout& L, const void* blob, const int8_t* Aq,
                               const uint16_t* s_a, int M, uint16_t* Y, int64_t ldy,
                               const DecodePlan& plan, int32_t* debug_partials, int32_t* status,
                               cudaStream_t s) {
    if (M == 0) return cudaSuccess;
    DecArgs a{};
    a.g = make_geom(L, blob);
    a.Aq = Aq;
    a.s_a = reinterpret_cast<const __half*>(s_a);
    a.Y = reinterpret_cast<__half*>(Y);
    a.ldy = ldy;
    a.M = M;
    a.S = plan.S;
    a.kbu = plan.kbu;
    a.debug = debug_partials;
    a.status = status;
    return debug_partials ? launch_mt<true>(a, plan.mt, plan.units, plan.m_tiles, plan.smem, s)
                          : launch_mt<false>(a, plan.mt, plan.units, plan.m_tiles, plan.smem, s);
}

bool decode_can_fuse(const mx_layout& L, int M, mx_dtype xdt) {
    // every CTA reads whole activation rows for the scales: keep that to 64 KB
    return M >= 1 && M <= kMaxFusedTokens &&
           size_t(M) * L.K * (xdt == MX_F16 ? 2 : 4) <= size_t(64) * 1024;
}

cudaError_t launch_gemm_decode_fused(const mx_layout& L, const void* blob, const void* X, mx_dtype xdt,
                                     int64_t ldx, int M, uint16_t* Y, int64_t ldy, const DecodePlan& plan,
                                     int32_t* debug_partials, int32_t* status, cudaStream_t s) {
    if (M == 0) return cudaSuccess;
    if (plan.mt > kMaxFusedTokens) return cudaErrorInvalidValue;
    DecArgs a{};
    a.g = make_geom(L, blob);
    a.X = X;
    a.ldx = ldx;
    a.Y = reinterpret_cast<__half*>(Y);
    a.ldy = ldy;
    a.M = M;
    a.S = plan.S;
    a.kbu = plan.kbu;
    a.debug = debug_partials;
    a.status = status;
    if (xdt == MX_F16)
        return debug_partials ? launch_mt_fused<true, __half>(a, plan.mt, plan.units, plan.m_tiles, plan.smem, s)
                              : launch_mt_fused<false, __half>(a, plan.mt, plan.units, plan.m_tiles, plan.smem, s);
    return debug_partials ? launch_mt_fused<true, float>(a, plan.mt, plan.units, plan.m_tiles, plan.smem, s)
                          : launch_mt_fused<false, float>(a, plan.mt, plan.units, plan.m_tiles, plan.smem, s);
}

}  // namespace mx
