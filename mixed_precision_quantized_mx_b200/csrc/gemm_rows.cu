// gemm_rows.cu -- decode-sized mixed-precision GEMM for short K: every CTA owns
// whole output rows, so there is no split of K and no reduction between CTAs.
//
// The arithmetic is the two-step dequantization of MixLLM section 3.3 on CUDA
// cores, as in the split-K decode kernel: per group an exact int32 dot product
// of the codes with the 8-bit activations (dp4a; for 4-bit rows the zero point
// is folded out as sum q a - z sum a), then acc += float(P) s_w in fp32 with the
// fast int-to-float, and Y = fp16(acc s_a) scattered through the row map.
//
// A unit is 32 packed 4-bit rows or 16 packed 8-bit rows: 2 KB of codes per
// 128-column k-block either way.  One 4-D tensor copy brings the unit's codes
// for the whole K (the 4-bit rows with the 64-byte swizzle, so that eight lanes
// reading one 16-byte chunk of eight consecutive rows hit distinct banks; the
// 8-bit rows are stored pre-swizzled already).  The group scales and zero points
// follow as 16-byte asynchronous copies.  None of this depends on the previous
// kernel, so it is issued before griddepcontrol.wait; the CTAs are small (256
// threads, the codes of at most 64 KB), so the next launch's CTAs can be
// resident and stream their weights while this one finishes.
//
// Thread t takes row t % R of the unit and every P-th k-block from t / R
// (P = 256 / R); the P partial sums of a row are added in a fixed order in
// shared memory, so the result is deterministic.  Activations are read as
// quantized codes (Aq, s_a) or as raw fp16 / fp32 rows that the CTA quantizes
// itself with the activation quantizer's device functions (whole rows: the
// scale needs the row's absmax), so both inputs give identical codes.
#include <algorithm>
#include <cstring>
#include <type_traits>

#include "mx_internal.cuh"
#include "sm100.cuh"

namespace mx {
namespace {

using namespace sm100;

// threads per CTA: one-token tiles take 512 (more warps to hide the latency of the
// dot products; two CTAs still fit on an SM), wider tiles 256
template <int MT>
constexpr int rows_threads() { return MT == 1 ? 512 : 256; }
constexpr int kMaxThreads = 512;
constexpr int kRows4 = 32;                  // 4-bit rows per unit
constexpr int kRows8 = 16;                  // 8-bit rows per unit
constexpr int kUnitKbBytes = 2048;          // codes of one unit per k-block
constexpr int kMaxK = 4096;
constexpr size_t kMaxSmem = 160 * 1024;
constexpr uint64_t kTimeoutNs = 2000000000ull;

struct RowsArgs {
    Geom g;
    const int8_t* Aq;       // quantized activations (when the kernel is not fed X)
    const __half* s_a;
    const void* X;          // raw activations fp16 / fp32 (when it quantizes them itself)
    int64_t ldx;
    __half* Y;
    int64_t ldy;
    int M;
    int n8u;                // 8-bit units (t8 * 16); 4-bit units follow
    int off_sc, off_z, off_act, off_sa64, off_red, off_sag;   // dynamic shared memory
    int ag;                 // 0: one activation scale per token; g: one per token and group
    int32_t* debug;
    int32_t* status;
};

__device__ __forceinline__ int dp4a(uint32_t a, uint32_t b, int c) {
    return __dp4a(int(a), int(b), c);
}

// unsigned bytes of a times signed bytes of b, accumulated into c
__device__ __forceinline__ int dp4a_us(uint32_t a, uint32_t b, int c) {
    int d;
    asm("dp4a.u32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

template <typename XT>
constexpr int x_size() {
    if constexpr (std::is_void_v<XT>) return 1;   // int8 codes
    else return int(sizeof(XT));
}

__device__ __forceinline__ void prefetch_l2(const void* p) {
    asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

__device__ __forceinline__ void griddep_wait() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

__device__ __forceinline__ void cp_async16(void* dst_smem, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst_smem)), "l"(src) : "memory");
}

__device__ __forceinline__ void cp_async_wait_all() {
    asm volatile("cp.async.wait_all;" ::: "memory");
}

__device__ __forceinline__ void tma_load_4d(void* dst, const CUtensorMap* map, int x, int y, int z, int w,
                                            uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4, %5}], [%6];"
        ::"r"(smem_u32(dst)), "l"(map), "r"(x), "r"(y), "r"(z), "r"(w), "r"(smem_u32(bar))
        : "memory");
}

// eight activations of one row held in registers: fp16 packed, fp32 as two float4
template <typename XT>
struct X8;
template <>
struct X8<__half> {
    uint4 v;
};
template <>
struct X8<float> {
    float4 lo, hi;
};
__device__ __forceinline__ void x8_load(X8<__half>& d, const __half* p) { d.v = __ldg(reinterpret_cast<const uint4*>(p)); }
__device__ __forceinline__ void x8_load(X8<float>& d, const float* p) {
    d.lo = __ldg(reinterpret_cast<const float4*>(p));
    d.hi = __ldg(reinterpret_cast<const float4*>(p) + 1);
}
__device__ __forceinline__ void x8_zero(X8<__half>& d) { d.v = make_uint4(0, 0, 0, 0); }
__device__ __forceinline__ void x8_zero(X8<float>& d) { d.lo = d.hi = make_float4(0.0f, 0.0f, 0.0f, 0.0f); }
// |x| maximum, exact in the input type (fp16 stays packed)
__device__ __forceinline__ float x8_absmax(const X8<__half>& d, float m) {
    const __half2* h = reinterpret_cast<const __half2*>(&d.v);
    __half2 a = __hmax2(__habs2(h[0]), __habs2(h[1]));
    a = __hmax2(a, __hmax2(__habs2(h[2]), __habs2(h[3])));
    return fmaxf(m, fmaxf(__low2float(a), __high2float(a)));
}
__device__ __forceinline__ float x8_absmax(const X8<float>& d, float m) {
    m = fmaxf(m, fmaxf(fmaxf(fabsf(d.lo.x), fabsf(d.lo.y)), fmaxf(fabsf(d.lo.z), fabsf(d.lo.w))));
    return fmaxf(m, fmaxf(fmaxf(fabsf(d.hi.x), fabsf(d.hi.y)), fmaxf(fabsf(d.hi.z), fabsf(d.hi.w))));
}
__device__ __forceinline__ void x8_float(const X8<__half>& d, float (&v)[8]) {
    const __half2* h = reinterpret_cast<const __half2*>(&d.v);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const float2 f = __half22float2(h[e]);
        v[2 * e] = f.x;
        v[2 * e + 1] = f.y;
    }
}
__device__ __forceinline__ void x8_float(const X8<float>& d, float (&v)[8]) {
    v[0] = d.lo.x; v[1] = d.lo.y; v[2] = d.lo.z; v[3] = d.lo.w;
    v[4] = d.hi.x; v[5] = d.hi.y; v[6] = d.hi.z; v[7] = d.hi.w;
}

// XT: void -- read Aq and s_a; __half or float -- quantize X in-kernel.
template <int MT, bool DEBUG, typename XT>
__global__ void __launch_bounds__(rows_threads<MT>(), 2)
gemm_rows_kernel(const __grid_constant__ CUtensorMap map4, const __grid_constant__ CUtensorMap map8,
                 const __grid_constant__ RowsArgs a) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // the 64-byte swizzle repeats every 512 bytes: the codes start on a 1 KB boundary
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const Geom& g = a.g;
    constexpr int NT = rows_threads<MT>();
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int u = blockIdx.x;
    const bool eight = u < a.n8u;
    const int R = eight ? kRows8 : kRows4;
    const int upt = kTileRows / R;                                 // units per tile
    const int tile = eight ? u / upt : (u - a.n8u) / upt;
    const int r0 = (eight ? u : u - a.n8u) % upt * R;              // first row in the tile
    const int m0 = blockIdx.y * MT;
    const int K = g.K, nkb = g.kblocks;
    const int gpk = kKBlock / g.group;

    __shared__ uint64_t wbar;
    __shared__ float sa_loc[MT];
    __shared__ float red_w[NT / 32][MT];
    if (tid == 0) {
        mbar_init(&wbar, 1);
        fence_mbar_init();
    }
    __syncthreads();
    asm volatile("griddepcontrol.launch_dependents;");

    // ---- weights: codes (one tensor copy), scales and zero points (16-byte copies)
    uint8_t* W = smem;                                             // [kb][R rows][64 or 128 B]
    __half* SC = reinterpret_cast<__half*>(smem + a.off_sc);       // [G][R]
    uint8_t* ZP = smem + a.off_z;                                  // [G][R]
    if (tid == 0) {
        mbar_arrive_expect_tx(&wbar, uint32_t(nkb) * kUnitKbBytes);
        if (eight) tma_load_4d(W, &map8, 0, r0, 0, tile, &wbar);
        else tma_load_4d(W, &map4, 0, r0, 0, tile, &wbar);
    }
    {
        const __half* scl = (eight ? g.scales8 : g.scales4) + size_t(tile) * g.G * kTileRows + r0;
        const int chunks = R * 2 / 16;                             // 16-byte chunks per group
        for (int i = tid; i < g.G * chunks; i += NT) {
            const int gi = i / chunks, c = i % chunks;
            cp_async16(SC + gi * R + c * 8, scl + size_t(gi) * kTileRows + c * 8);
        }
        if (!eight) {
            const uint8_t* zr = g.zeros4 + size_t(tile) * g.G * kTileRows + r0;
            const int zch = R / 16;                                  // 16-byte chunks per group
            for (int i = tid; i < g.G * zch; i += NT) {
                const int gi = i / zch, c = i % zch;
                cp_async16(ZP + gi * R + c * 16, zr + size_t(gi) * kTileRows + c * 16);
            }
        }
    }

    // ---- activations (these wait for the previous kernel)
    int8_t* act = reinterpret_cast<int8_t*>(smem + a.off_act);    // [MT][K]
    float* sag = reinterpret_cast<float*>(smem + a.off_sag);        // [MT][G] when a.ag
    int32_t* sa64 = reinterpret_cast<int32_t*>(smem + a.off_sa64);  // [MT][K / 64]
    bool sums_done = false;
    // this thread's row of the unit, its first k-block, and the row's output column
    // (weights too: read before the wait)
    const int P = NT / R;
    const int r = tid % R, kph = tid / R;
    const int slot_row = eight ? tile * kTileRows + r0 + r : (g.t8 + tile) * kTileRows + r0 + r;
    const int orig = g.rowmap[slot_row];
    // the activation rows of this token tile into L2 while the weights stream: a
    // prefetch cannot return stale data (L2 is where every write lands), so it may
    // run before the wait; each CTA takes a share of the 128-byte lines
    {
        const uint8_t* xb = std::is_void_v<XT> ? reinterpret_cast<const uint8_t*>(a.Aq)
                                               : static_cast<const uint8_t*>(a.X);
        const int64_t pitch = std::is_void_v<XT> ? int64_t(K) : a.ldx * int64_t(x_size<XT>());
        const int lines = (K * x_size<XT>() + 127) / 128;             // per row
        for (int i = blockIdx.x + tid * int(gridDim.x); i < MT * lines; i += NT * int(gridDim.x)) {
            const int j = i / lines, l = i % lines;
            if (m0 + j < a.M) prefetch_l2(xb + (m0 + j) * pitch + l * 128);
        }
    }
    griddep_wait();
    if constexpr (std::is_void_v<XT>) {
        const int chunks = K / 16;
        for (int i = tid; i < MT * chunks; i += NT) {
            const int j = i / chunks, c = i % chunks;
            if (m0 + j < a.M) cp_async16(act + size_t(j) * K + c * 16, a.Aq + int64_t(m0 + j) * K + c * 16);
            else *reinterpret_cast<uint4*>(act + size_t(j) * K + c * 16) = make_uint4(0, 0, 0, 0);
        }
        if (a.ag) {                       // group-wise activation scales s_a[m][g]
            for (int i = tid; i < MT * g.G; i += NT) {
                const int j = i / g.G, gi = i % g.G;
                sag[i] = m0 + j < a.M ? __half2float(a.s_a[int64_t(m0 + j) * g.G + gi]) : 0.0f;
            }
        }
        cp_async_wait_all();
        __syncthreads();
    } else if (a.ag) {
        // group-wise scales, in one pass: a group's 8-element chunks sit in consecutive
        // lanes, so its absmax is a shuffle reduction in that lane segment, and every
        // lane then quantizes the values it holds (the grouped quantizer's operations)
        const XT* X = static_cast<const XT*>(a.X);
        const int cpg = a.ag / 8;
#pragma unroll
        for (int j = 0; j < MT; ++j) {
            const bool row = m0 + j < a.M;
            for (int c0 = 0; c0 < K / 8; c0 += NT) {                // same trip count in every lane
                const int c = c0 + tid;
                const bool live = row && c < K / 8;
                float v[8];
                if (live) {
                    const XT* xp = X + int64_t(m0 + j) * a.ldx + c * 8;
                    if constexpr (std::is_same_v<XT, __half>) {
                        const uint4 raw = __ldg(reinterpret_cast<const uint4*>(xp));
                        const __half2* h2 = reinterpret_cast<const __half2*>(&raw);
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float2 f = __half22float2(h2[e]);
                            v[2 * e] = f.x;
                            v[2 * e + 1] = f.y;
                        }
                    } else {
                        const float4 f0 = __ldg(reinterpret_cast<const float4*>(xp));
                        const float4 f1 = __ldg(reinterpret_cast<const float4*>(xp) + 1);
                        v[0] = f0.x; v[1] = f0.y; v[2] = f0.z; v[3] = f0.w;
                        v[4] = f1.x; v[5] = f1.y; v[6] = f1.z; v[7] = f1.w;
                    }
                } else {
#pragma unroll
                    for (int e = 0; e < 8; ++e) v[e] = 0.0f;
                }
                float am = 0.0f;
#pragma unroll
                for (int e = 0; e < 8; ++e) am = fmaxf(am, fabsf(v[e]));
                for (int o = cpg / 2; o > 0; o >>= 1) am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, o));
                const float sg = __half2float(act_scale(am)), rg = __frcp_rn(sg);
                if (c < K / 8) {
                    uint2 o = make_uint2(0, 0);
                    if (live) {
                        o.x = quant4(v, sg, rg);
                        o.y = quant4(v + 4, sg, rg);
                    }
                    *reinterpret_cast<uint2*>(act + size_t(j) * K + c * 8) = o;
                    if (c % cpg == 0) sag[j * g.G + c / cpg] = live ? sg : 0.0f;
                }
            }
        }
        __syncthreads();
    } else {
        // whole rows from registers: every thread holds CPT chunks of eight values of
        // each row; the absmax (exact in the input type) takes one block reduction, then
        // the fp16 scale and the codes, with the quantizer's operations.  For 4-bit
        // units the 64-column code sums come in the same pass: eight consecutive chunks
        // sit in eight consecutive lanes.
        const XT* X = static_cast<const XT*>(a.X);
        constexpr int CPT = (kMaxK / 8 + NT - 1) / NT;            // chunks per thread and row
        X8<XT> xv[MT][CPT];
#pragma unroll
        for (int j = 0; j < MT; ++j)
#pragma unroll
            for (int i = 0; i < CPT; ++i) {
                const int c = tid + i * NT;
                if (m0 + j < a.M && c < K / 8) x8_load(xv[j][i], X + int64_t(m0 + j) * a.ldx + c * 8);
                else x8_zero(xv[j][i]);
            }
#pragma unroll
        for (int j = 0; j < MT; ++j) {
            float am = 0.0f;
#pragma unroll
            for (int i = 0; i < CPT; ++i) am = x8_absmax(xv[j][i], am);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, o));
            if (lane == 0) red_w[warp][j] = am;
        }
        __syncthreads();
#pragma unroll
        for (int j = 0; j < MT; ++j) {
            float m = red_w[0][j];
#pragma unroll
            for (int w = 1; w < NT / 32; ++w) m = fmaxf(m, red_w[w][j]);
            const float sc = __half2float(act_scale(m)), rsc = __frcp_rn(sc);
            if (tid == j) sa_loc[j] = sc;
            const bool live = m0 + j < a.M;
#pragma unroll
            for (int i = 0; i < CPT; ++i) {
                if (i * NT >= K / 8) break;                          // the same in every lane
                const int c = tid + i * NT;
                uint2 o = make_uint2(0, 0);
                if (live && c < K / 8) {
                    float v[8];
                    x8_float(xv[j][i], v);
                    o.x = quant4(v, sc, rsc);
                    o.y = quant4(v + 4, sc, rsc);
                }
                if (c < K / 8) *reinterpret_cast<uint2*>(act + size_t(j) * K + c * 8) = o;
                if (!eight) {
                    int sum = dp4a(o.x, 0x01010101u, dp4a(o.y, 0x01010101u, 0));
                    sum += __shfl_xor_sync(0xffffffffu, sum, 1);
                    sum += __shfl_xor_sync(0xffffffffu, sum, 2);
                    sum += __shfl_xor_sync(0xffffffffu, sum, 4);
                    if ((c & 7) == 0 && c < K / 8) sa64[j * (K / 64) + c / 8] = sum;
                }
            }
        }
        sums_done = true;
    }
    // activation sums of every 64 columns (the zero-point fold of 4-bit rows)
    if (!eight && !sums_done) {
        for (int i = tid; i < MT * (K / 64); i += NT) {
            const int j = i / (K / 64), h = i % (K / 64);
            const uint4* p = reinterpret_cast<const uint4*>(act + size_t(j) * K + h * 64);
            int s = 0;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const uint4 v = p[c];
                s = dp4a(v.x, 0x01010101u, s);
                s = dp4a(v.y, 0x01010101u, s);
                s = dp4a(v.z, 0x01010101u, s);
                s = dp4a(v.w, 0x01010101u, s);
            }
            sa64[i] = s;
        }
    }
    cp_async_wait_all();                 // scales and zero points

    // ---- codes landed (bounded wait; on expiry record it and let the copy drain);
    // the barrier below also publishes the activation codes and sums
    bool ok = true;
    if (tid == 0) {
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_try_wait(&wbar, 0)) {
            if (globaltimer_ns() - t0 > kTimeoutNs) {
                ok = false;
                if (a.status) atomicExch(a.status, MX_ERR_TIMEOUT);
                const uint64_t t1 = globaltimer_ns();
                while (!mbar_try_wait(&wbar, 0) && globaltimer_ns() - t1 < kTimeoutNs) {
                }
                break;
            }
        }
    }
    if (!__syncthreads_and(ok)) return;

    // ---- dot products: thread -> (row r of the unit, k-blocks kph, kph + P, ...)
    // physical 16-byte chunk = logical chunk ^ swz (8-bit rows: the stored 128-byte
    // swizzle of the tile; 4-bit rows: the copy's 64-byte swizzle)
    const int swz = eight ? (r & 7) : ((r >> 1) & 3);
    const int h64 = K / 64;
    float out[MT];
#pragma unroll
    for (int j = 0; j < MT; ++j) out[j] = 0.0f;
#pragma unroll 2
    for (int kb = kph; kb < nkb; kb += P) {
        const uint8_t* wrow = W + size_t(kb) * kUnitKbBytes + r * (eight ? 128 : 64);
        const int8_t* ak = act + kb * kKBlock;
#pragma unroll
        for (int gl = 0; gl < 2; ++gl) {
            if (gl >= gpk) break;
            const int gi = kb * gpk + gl;
            // two accumulators per token (even and odd chunks): shorter dependent chains
            int acc[MT], acc2[MT];
#pragma unroll
            for (int j = 0; j < MT; ++j) acc[j] = acc2[j] = 0;
            if (eight) {
                // 16 codes per logical chunk; a group is 8 / gpk chunks
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    if (c >= 8 / gpk) break;
                    const int lc = gl * (8 / gpk) + c;
                    const uint4 w = *reinterpret_cast<const uint4*>(wrow + ((lc ^ swz) << 4));
#pragma unroll
                    for (int j = 0; j < MT; ++j) {
                        const uint4 av = *reinterpret_cast<const uint4*>(ak + size_t(j) * K + lc * 16);
                        int& t = (c & 1) ? acc2[j] : acc[j];
                        t = dp4a(w.x, av.x, t);
                        t = dp4a(w.y, av.y, t);
                        t = dp4a(w.z, av.z, t);
                        t = dp4a(w.w, av.w, t);
                    }
                }
#pragma unroll
                for (int j = 0; j < MT; ++j) acc[j] += acc2[j];
            } else {
                // 32 codes per logical chunk: word q holds k = 8q .. 8q+7 of the chunk, the
                // low nibbles k = 8q .. 8q+3, the high nibbles (kept in place: 16 x code as
                // an unsigned byte) k = 8q+4 .. 8q+7; a group is 4 / gpk chunks
                int hi16[MT], hi16b[MT];
#pragma unroll
                for (int j = 0; j < MT; ++j) hi16[j] = hi16b[j] = 0;
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    if (c >= 4 / gpk) break;
                    const int lc = gl * (4 / gpk) + c;
                    const uint4 w = *reinterpret_cast<const uint4*>(wrow + ((lc ^ swz) << 4));
#pragma unroll
                    for (int j = 0; j < MT; ++j) {
                        const uint4 a0 = *reinterpret_cast<const uint4*>(ak + size_t(j) * K + lc * 32);
                        const uint4 a1 = *reinterpret_cast<const uint4*>(ak + size_t(j) * K + lc * 32 + 16);
                        int& lo = (c & 1) ? acc2[j] : acc[j];
                        int& hi = (c & 1) ? hi16b[j] : hi16[j];
                        lo = dp4a(w.x & 0x0F0F0F0Fu, a0.x, lo);
                        hi = dp4a_us(w.x & 0xF0F0F0F0u, a0.y, hi);
                        lo = dp4a(w.y & 0x0F0F0F0Fu, a0.z, lo);
                        hi = dp4a_us(w.y & 0xF0F0F0F0u, a0.w, hi);
                        lo = dp4a(w.z & 0x0F0F0F0Fu, a1.x, lo);
                        hi = dp4a_us(w.z & 0xF0F0F0F0u, a1.y, hi);
                        lo = dp4a(w.w & 0x0F0F0F0Fu, a1.z, lo);
                        hi = dp4a_us(w.w & 0xF0F0F0F0u, a1.w, hi);
                    }
                }
                const int z = ZP[gi * R + r];
#pragma unroll
                for (int j = 0; j < MT; ++j) {
                    const int32_t* s64 = sa64 + j * h64 + 2 * kb;
                    const int suma = gpk == 1 ? s64[0] + s64[1] : s64[gl];
                    // exact: the high-nibble sums are 16 x their value
                    acc[j] += acc2[j] + ((hi16[j] + hi16b[j]) >> 4) - z * suma;
                }
            }
            const float sw = __half2float(SC[gi * R + r]);
#pragma unroll
            for (int j = 0; j < MT; ++j) {
                // group-wise activations: the token's scale of this group joins the weight's
                const float s = a.ag ? __fmul_rn(sw, sag[j * g.G + gi]) : sw;
                out[j] = __fmaf_rn(i2f_biased(acc[j]), s, out[j]);
            }
            if (DEBUG && orig >= 0) {                                   // padding rows have no column
#pragma unroll
                for (int j = 0; j < MT; ++j)
                    if (m0 + j < a.M) a.debug[(size_t(m0 + j) * g.N + orig) * g.G + gi] = acc[j];
            }
        }
    }

    // ---- the P partial sums of every row, in k-phase order, then s_a and the scatter
    float* red = reinterpret_cast<float*>(smem + a.off_red);          // [P][R][MT]
#pragma unroll
    for (int j = 0; j < MT; ++j) red[(kph * R + r) * MT + j] = out[j];
    __syncthreads();
    if (tid < R * MT) {
        const int j = tid / R;                                          // tid % R == r
        if (m0 + j < a.M && orig >= 0) {
            float sum = 0.0f;
            for (int q = 0; q < P; ++q) sum = __fadd_rn(sum, red[(q * R + r) * MT + j]);
            float sa = 1.0f;                        // group-wise scales were applied per group
            if (!a.ag) {
                if constexpr (std::is_void_v<XT>) sa = __half2float(a.s_a[m0 + j]);
                else sa = sa_loc[j];
            }
            a.Y[int64_t(m0 + j) * a.ldy + orig] = __float2half_rn(__fmul_rn(sum, sa));
        }
    }
}

template <int MT, bool DEBUG, typename XT>
cudaError_t launch_t(const CUtensorMap& m4, const CUtensorMap& m8, const RowsArgs& args, int units, int m_tiles,
                     size_t smem, cudaStream_t s) {
    auto k = gemm_rows_kernel<MT, DEBUG, XT>;
    static bool configured[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!configured[dev]) {
        e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, int(kMaxSmem));
        if (e != cudaSuccess) return e;
        e = cudaFuncSetAttribute(k, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
        if (e != cudaSuccess) return e;
        configured[dev] = true;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(units, m_tiles);
    cfg.blockDim = dim3(rows_threads<MT>());
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, k, m4, m8, args);
}

template <bool DEBUG, typename XT>
cudaError_t launch_mt(const CUtensorMap& m4, const CUtensorMap& m8, const RowsArgs& a, const RowsPlan& p,
                      cudaStream_t s) {
    switch (p.mt) {
        case 1: return launch_t<1, DEBUG, XT>(m4, m8, a, p.units, p.m_tiles, p.smem, s);
        case 2: return launch_t<2, DEBUG, XT>(m4, m8, a, p.units, p.m_tiles, p.smem, s);
        case 4: return launch_t<4, DEBUG, XT>(m4, m8, a, p.units, p.m_tiles, p.smem, s);
        default: return cudaErrorInvalidValue;
    }
}

template <typename XT>
cudaError_t launch_dbg(const CUtensorMap& m4, const CUtensorMap& m8, const RowsArgs& a, const RowsPlan& p,
                       cudaStream_t s) {
    return a.debug ? launch_mt<true, XT>(m4, m8, a, p, s) : launch_mt<false, XT>(m4, m8, a, p, s);
}

// codes of one packed tile kind as a 4-D tensor [tile][k-block][row][bytes]; a box
// is one unit's rows over the whole K
cudaError_t unit_map(EncodeTiledFn enc, const void* base, int tiles, int kblocks, int row_bytes, int rows,
                     CUtensorMapSwizzle swizzle, CUtensorMap* map) {
    memset(map, 0, sizeof *map);
    if (tiles == 0) return cudaSuccess;                // this kind has no rows: never read
    const uint64_t kb_bytes = uint64_t(kTileRows) * row_bytes;
    const cuuint64_t dims[4] = {cuuint64_t(row_bytes), cuuint64_t(kTileRows), cuuint64_t(kblocks), cuuint64_t(tiles)};
    const cuuint64_t strides[3] = {cuuint64_t(row_bytes), cuuint64_t(kb_bytes), cuuint64_t(kb_bytes * kblocks)};
    const cuuint32_t box[4] = {cuuint32_t(row_bytes), cuuint32_t(rows), cuuint32_t(kblocks), 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, const_cast<void*>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

size_t align16(size_t v) { return (v + 15) & ~size_t(15); }

}  // namespace

RowsPlan plan_rows(const mx_layout& L, int M) {
    RowsPlan p{};
    p.mt = M <= 1 ? 1 : M <= 2 ? 2 : 4;
    p.m_tiles = std::max(1, (M + p.mt - 1) / p.mt);
    p.n8u = L.t8 * (kTileRows / kRows8);
    p.units = p.n8u + L.t4 * (kTileRows / kRows4);
    // shared memory: codes | scales | zero points | activation codes | 64-column sums |
    // partial sums | group-wise activation scales.  Raw activation rows are read into
    // registers, so Aq, fp16 and fp32 inputs of one shape take the same plan.
    size_t off = size_t(L.kblocks) * kUnitKbBytes;
    p.off_sc = int(off);
    off += align16(size_t(L.G) * kRows4 * 2);
    p.off_z = int(off);
    off += align16(size_t(L.G) * kRows4);
    p.off_act = int(off);
    off += align16(size_t(p.mt) * L.K);
    p.off_sa64 = int(off);
    off += align16(size_t(p.mt) * (L.K / 64) * 4);
    p.off_red = int(off);
    off += size_t(kMaxThreads) * p.mt * 4;
    p.off_sag = int(off);
    off += align16(size_t(p.mt) * L.G * 4);
    p.smem = off + 1024;                                // + room to align the base
    // one wave with room left for the next launch's CTAs
    p.ok = M >= 1 && M <= 4 && L.K <= kMaxK && p.units * p.m_tiles <= 2 * 148 && p.smem <= kMaxSmem;
    return p;
}

cudaError_t launch_gemm_rows(const mx_layout& L, const void* blob, const int8_t* Aq, const uint16_t* s_a,
                             const void* X, mx_dtype xdt, int64_t ldx, int M, uint16_t* Y, int64_t ldy,
                             const RowsPlan& p, int ag, int32_t* debug_partials, int32_t* status,
                             cudaStream_t s) {
    if (M == 0) return cudaSuccess;
    if (!p.ok) return cudaErrorInvalidValue;
    cudaError_t e;
    EncodeTiledFn enc = encode_fn(&e);
    if (e != cudaSuccess) return e;
    const uint8_t* b = static_cast<const uint8_t*>(blob);
    CUtensorMap m4, m8;
    if ((e = unit_map(enc, b + L.off_codes4, L.t4, L.kblocks, kKBlock / 2, kRows4, CU_TENSOR_MAP_SWIZZLE_64B,
                      &m4)) != cudaSuccess)
        return e;
    if ((e = unit_map(enc, b + L.off_codes8, L.t8, L.kblocks, kKBlock, kRows8, CU_TENSOR_MAP_SWIZZLE_NONE,
                      &m8)) != cudaSuccess)
        return e;
    RowsArgs a{};
    a.g = make_geom(L, blob);
    a.Aq = Aq;
    a.s_a = reinterpret_cast<const __half*>(s_a);
    a.X = X;
    a.ldx = ldx;
    a.Y = reinterpret_cast<__half*>(Y);
    a.ldy = ldy;
    a.M = M;
    a.n8u = p.n8u;
    a.off_sc = p.off_sc;
    a.off_z = p.off_z;
    a.off_act = p.off_act;
    a.off_sa64 = p.off_sa64;
    a.off_red = p.off_red;
    a.off_sag = p.off_sag;
    a.ag = ag;
    a.debug = debug_partials;
    a.status = status;
    if (X == nullptr) return launch_dbg<void>(m4, m8, a, p, s);
    return xdt == MX_F16 ? launch_dbg<__half>(m4, m8, a, p, s) : launch_dbg<float>(m4, m8, a, p, s);
}

}  // namespace mx
