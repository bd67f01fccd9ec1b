// gemm_splitk.cu -- decode-sized mixed-precision GEMM (few tokens, HBM-bound).
//
// Two-step dequantization of MixLLM section 3.3 on CUDA cores:
//   step 1: per group, P = sum_k Aq[m,k] (W_q[n,k] - z[n,g]) in exact int32
//           (dp4a on the int8 / widened uint4 codes),
//   step 2: acc[m,n] += float(P) s_w[n,g] in fp32 with the fast int-to-float
//           of section 3.3 (Figure 3), and Y = fp16(acc s_a[m]) at the end.
// For 4-bit rows the zero point is folded out of the dot product:
//   sum (q - z) a = sum q a - z sum a,
// with the per-token activation sums of every 64-column half-block computed
// once per CTA in shared memory, so the widening is just two mask operations
// per 8 codes (q in 0..15 is already a valid int8 operand).
//
// Work split: a "unit" is (row tile of 128 packed rows, range of k-blocks);
// 8-bit tiles get half as many k-blocks per unit as 4-bit tiles so that every
// unit streams about the same number of weight bytes.  Units write fp32
// partial outputs to the workspace; the reduce kernel sums them in unit order
// (deterministic), applies s_a and scatters each packed row back to its
// original column of Y (section 3.3, fused scatter of the sub-problem outputs).
#include <algorithm>

#include "mx_internal.cuh"

namespace mx {
namespace {

constexpr int kThreads = 256;           // 128 rows x 2 halves of a k-block
constexpr int kUnroll = 4;              // k-blocks whose loads are in flight together
constexpr int kMaxActSmem = 96 * 1024;  // activation slice staged in shared memory

struct SplitArgs {
    Geom g;
    const int8_t* Aq;
    int M;
    int mt_tokens, m_tiles;
    int kbu8, kbu4, s8, s4, kbu_max;
    float* ws;
    int32_t* debug;
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

template <int MT, bool DEBUG>
__global__ void __launch_bounds__(kThreads)
gemm_splitk_kernel(const __grid_constant__ SplitArgs a) {
    extern __shared__ __align__(16) uint8_t smem[];
    const Geom& g = a.g;
    const int unit = blockIdx.x;
    const int mtile = blockIdx.y;
    const bool eight = unit < g.t8 * a.s8;
    int tile, sidx, kbu;
    if (eight) {
        tile = unit / a.s8; sidx = unit % a.s8; kbu = a.kbu8;
    } else {
        const int u = unit - g.t8 * a.s8;
        tile = u / a.s4; sidx = u % a.s4; kbu = a.kbu4;
    }
    const int kb0 = sidx * kbu;
    const int kb1 = min(kb0 + kbu, g.kblocks);
    const int nkb = kb1 - kb0;
    const int rowb = a.kbu_max * kKBlock;            // smem bytes per token
    int8_t* act = reinterpret_cast<int8_t*>(smem);
    int32_t* sa64 = reinterpret_cast<int32_t*>(smem + size_t(MT) * rowb);
    const int m0 = mtile * MT;
    const int tid = threadIdx.x;

    // stage Aq[m0 .. m0+MT)[kb0*128 .. kb1*128) (zero rows beyond M)
    const int chunks = nkb * (kKBlock / 16);
    for (int i = tid; i < MT * chunks; i += kThreads) {
        const int j = i / chunks, c = i % chunks;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (m0 + j < a.M)
            v = __ldg(reinterpret_cast<const uint4*>(a.Aq + int64_t(m0 + j) * g.K +
                                                     kb0 * kKBlock) + c);
        *reinterpret_cast<uint4*>(act + j * rowb + c * 16) = v;
    }
    __syncthreads();
    if (!eight) {
        // activation sums of every 64-column half-block: sa64[j][2*kl + h]
        for (int i = tid; i < MT * nkb * 2; i += kThreads) {
            const int j = i / (nkb * 2), hb = i % (nkb * 2);
            const uint4* p = reinterpret_cast<const uint4*>(act + j * rowb + hb * 64);
            int s = 0;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                uint4 v = p[c];
                s = dp4a(v.x, 0x01010101u, s);
                s = dp4a(v.y, 0x01010101u, s);
                s = dp4a(v.z, 0x01010101u, s);
                s = dp4a(v.w, 0x01010101u, s);
            }
            sa64[j * 2 * a.kbu_max + hb] = s;
        }
        __syncthreads();
    }

    const int r = tid >> 1, h = tid & 1;
    const int slot = (eight ? 0 : g.t8 * kTileRows) + tile * kTileRows + r;
    const int orig = DEBUG ? g.rowmap[slot] : 0;
    float out[MT];
#pragma unroll
    for (int j = 0; j < MT; ++j) out[j] = 0.0f;

    if (eight) {
        const int lh = h ^ ((r & 7) >> 2);   // logical half held by physical half h
        const uint8_t* base = reinterpret_cast<const uint8_t*>(g.codes8) +
                              size_t(tile) * g.kblocks * kBlock8Bytes + r * 128 + h * 64;
        for (int kbb = kb0; kbb < kb1; kbb += kUnroll) {
            uint4 c[kUnroll][4];
#pragma unroll
            for (int u = 0; u < kUnroll; ++u)
                if (kbb + u < kb1)
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        c[u][i] = ldg_stream(base + size_t(kbb + u) * kBlock8Bytes + i * 16);
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) {
                const int kb = kbb + u;
                if (kb >= kb1) break;
                const int kl = kb - kb0;
                const int gi = (kb * kKBlock + lh * 64) / g.group;
                const float s = __half2float(g.scales8[(size_t(tile) * g.G + gi) * kTileRows + r]);
                int acc[MT];
#pragma unroll
                for (int j = 0; j < MT; ++j) acc[j] = 0;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int lc = (4 * h + i) ^ (r & 7);   // logical 16-column chunk
#pragma unroll
                    for (int j = 0; j < MT; ++j) {
                        const uint4 av = *reinterpret_cast<const uint4*>(act + j * rowb +
                                                                         kl * kKBlock + lc * 16);
                        acc[j] = dp4a(c[u][i].x, av.x, acc[j]);
                        acc[j] = dp4a(c[u][i].y, av.y, acc[j]);
                        acc[j] = dp4a(c[u][i].z, av.z, acc[j]);
                        acc[j] = dp4a(c[u][i].w, av.w, acc[j]);
                    }
                }
                if (g.group == 128) {
#pragma unroll
                    for (int j = 0; j < MT; ++j) acc[j] += __shfl_xor_sync(0xffffffffu, acc[j], 1);
                }
#pragma unroll
                for (int j = 0; j < MT; ++j) out[j] = __fmaf_rn(i2f_biased(acc[j]), s, out[j]);
                if (DEBUG && (g.group == 64 || h == 0) && orig >= 0) {
#pragma unroll
                    for (int j = 0; j < MT; ++j)
                        if (m0 + j < a.M)
                            a.debug[(size_t(m0 + j) * g.N + orig) * g.G + gi] = acc[j];
                }
            }
        }
    } else {
        const uint8_t* base = g.codes4 + size_t(tile) * g.kblocks * kBlock4Bytes + r * 64 + h * 32;
        for (int kbb = kb0; kbb < kb1; kbb += kUnroll) {
            uint4 c[kUnroll][2];
#pragma unroll
            for (int u = 0; u < kUnroll; ++u)
                if (kbb + u < kb1)
#pragma unroll
                    for (int i = 0; i < 2; ++i)
                        c[u][i] = ldg_stream(base + size_t(kbb + u) * kBlock4Bytes + i * 16);
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) {
                const int kb = kbb + u;
                if (kb >= kb1) break;
                const int kl = kb - kb0;
                const int gi = (kb * kKBlock + h * 64) / g.group;
                const size_t meta = (size_t(tile) * g.G + gi) * kTileRows + r;
                const float s = __half2float(g.scales4[meta]);
                const int z = g.zeros4[meta];
                int acc[MT];
#pragma unroll
                for (int j = 0; j < MT; ++j) acc[j] = 0;
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                    const uint32_t wd[4] = {c[u][i].x, c[u][i].y, c[u][i].z, c[u][i].w};
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const uint32_t lo = wd[q] & 0x0F0F0F0Fu;          // k = 8w .. 8w+3
                        const uint32_t hi = (wd[q] >> 4) & 0x0F0F0F0Fu;   // k = 8w+4 .. 8w+7
                        const int koff = h * 64 + i * 32 + q * 8;
#pragma unroll
                        for (int j = 0; j < MT; ++j) {
                            const uint2 av = *reinterpret_cast<const uint2*>(
                                act + j * rowb + kl * kKBlock + koff);
                            acc[j] = dp4a(lo, av.x, acc[j]);
                            acc[j] = dp4a(hi, av.y, acc[j]);
                        }
                    }
                }
#pragma unroll
                for (int j = 0; j < MT; ++j) acc[j] -= z * sa64[j * 2 * a.kbu_max + kl * 2 + h];
                if (g.group == 128) {
#pragma unroll
                    for (int j = 0; j < MT; ++j) acc[j] += __shfl_xor_sync(0xffffffffu, acc[j], 1);
                }
#pragma unroll
                for (int j = 0; j < MT; ++j) out[j] = __fmaf_rn(i2f_biased(acc[j]), s, out[j]);
                if (DEBUG && (g.group == 64 || h == 0) && orig >= 0) {
#pragma unroll
                    for (int j = 0; j < MT; ++j)
                        if (m0 + j < a.M)
                            a.debug[(size_t(m0 + j) * g.N + orig) * g.G + gi] = acc[j];
                }
            }
        }
    }

    if (g.group == 64) {
#pragma unroll
        for (int j = 0; j < MT; ++j) out[j] = __fadd_rn(out[j], __shfl_xor_sync(0xffffffffu, out[j], 1));
    }
    if (h == 0) {
        float* w = a.ws + (size_t(unit) * a.m_tiles + mtile) * MT * kTileRows + r;
#pragma unroll
        for (int j = 0; j < MT; ++j) w[j * kTileRows] = out[j];
    }
}

__global__ void __launch_bounds__(256)
splitk_reduce_kernel(const float* __restrict__ ws, const int32_t* __restrict__ rowmap,
                     const __half* __restrict__ s_a, int M, int t8, int t4, int s8, int s4,
                     int m_tiles, int mt_tokens, __half* __restrict__ Y, int64_t ldy) {
    const int slot = blockIdx.x * blockDim.x + threadIdx.x;
    const int m = blockIdx.y;
    if (slot >= (t8 + t4) * kTileRows || m >= M) return;
    const int orig = rowmap[slot];
    if (orig < 0) return;
    const int tile = slot >> 7, r = slot & (kTileRows - 1);
    int ubase, cnt;
    if (tile < t8) { ubase = tile * s8; cnt = s8; }
    else { ubase = t8 * s8 + (tile - t8) * s4; cnt = s4; }
    const int mt = m / mt_tokens, j = m % mt_tokens;
    float acc = 0.0f;
    for (int u = 0; u < cnt; ++u)
        acc = __fadd_rn(acc, ws[((size_t(ubase + u) * m_tiles + mt) * mt_tokens + j) * kTileRows + r]);
    Y[int64_t(m) * ldy + orig] = __float2half_rn(__fmul_rn(acc, __half2float(s_a[m])));
}

template <int MT, bool DEBUG>
cudaError_t launch_t(const SplitArgs& a, size_t smem, cudaStream_t s) {
    auto k = gemm_splitk_kernel<MT, DEBUG>;
    // the shared-memory opt-in is per device: set it once for each one used
    static bool configured[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!configured[dev]) {
        e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 kMaxActSmem + 16 * 1024);
        if (e != cudaSuccess) return e;
        configured[dev] = true;
    }
    k<<<dim3(a.s8 * a.g.t8 + a.s4 * a.g.t4, a.m_tiles), kThreads, smem, s>>>(a);
    return cudaGetLastError();
}

template <bool DEBUG>
cudaError_t launch_mt(const SplitArgs& a, size_t smem, cudaStream_t s) {
    switch (a.mt_tokens) {
        case 1: return launch_t<1, DEBUG>(a, smem, s);
        case 2: return launch_t<2, DEBUG>(a, smem, s);
        case 4: return launch_t<4, DEBUG>(a, smem, s);
        case 8: return launch_t<8, DEBUG>(a, smem, s);
        default: return launch_t<16, DEBUG>(a, smem, s);
    }
}

int ceil_div(int a, int b) { return (a + b - 1) / b; }

}  // namespace

SplitPlan plan_splitk(const mx_layout& L, int M, int split_hint) {
    SplitPlan p{};
    p.mt = M <= 1 ? 1 : M <= 2 ? 2 : M <= 4 ? 4 : M <= 8 ? 8 : 16;
    p.m_tiles = std::max(1, ceil_div(M, p.mt));
    const int kb = L.kblocks;
    const int kbu_cap = std::max(1, kMaxActSmem / (p.mt * kKBlock));
    int s4;
    if (split_hint > 0) {
        s4 = split_hint;
    } else {
        // about four units per SM of a 148-SM B200, weighting 8-bit tiles double
        const int weight = std::max(1, L.t4 + 2 * L.t8);
        s4 = (4 * 148 / p.m_tiles + weight / 2) / weight;
    }
    s4 = std::min(std::max(s4, 1), kb);
    p.kbu4 = std::min(ceil_div(kb, s4), kbu_cap);
    p.s4 = ceil_div(kb, p.kbu4);
    p.kbu8 = std::max(1, ceil_div(p.kbu4, 2));
    p.s8 = ceil_div(kb, p.kbu8);
    p.units = L.t8 * p.s8 + L.t4 * p.s4;
    p.ws_bytes = size_t(p.units) * p.m_tiles * p.mt * kTileRows * sizeof(float);
    return p;
}

cudaError_t launch_gemm_splitk(const mx_layout& L, const void* blob, const int8_t* Aq,
                               const uint16_t* s_a, int M, uint16_t* Y, int64_t ldy,
                               float* ws, const SplitPlan& plan, int32_t* debug_partials,
                               cudaStream_t s) {
    if (M == 0) return cudaSuccess;
    SplitArgs a{};
    a.g = make_geom(L, blob);
    a.Aq = Aq;
    a.M = M;
    a.mt_tokens = plan.mt;
    a.m_tiles = plan.m_tiles;
    a.kbu8 = plan.kbu8;
    a.kbu4 = plan.kbu4;
    a.s8 = plan.s8;
    a.s4 = plan.s4;
    a.kbu_max = std::max(plan.kbu8, plan.kbu4);
    a.ws = ws;
    a.debug = debug_partials;
    const size_t smem = size_t(plan.mt) * a.kbu_max * kKBlock + size_t(plan.mt) * 2 * a.kbu_max * 4;
    cudaError_t e = debug_partials ? launch_mt<true>(a, smem, s) : launch_mt<false>(a, smem, s);
    if (e != cudaSuccess) return e;
    const int slots = (L.t8 + L.t4) * kTileRows;
    splitk_reduce_kernel<<<dim3(ceil_div(slots, 256), M), 256, 0, s>>>(
        ws, a.g.rowmap, reinterpret_cast<const __half*>(s_a), M, L.t8, L.t4, plan.s8, plan.s4,
        plan.m_tiles, plan.mt, reinterpret_cast<__half*>(Y), ldy);
    return cudaGetLastError();
}

}  // namespace mx
