// gemm_tc.cu -- tensor-core mixed-precision GEMM for prefill-sized M (sm_100a).
//
// Two-step dequantization (MixLLM section 3.3) on 5th-generation tensor cores:
//   step 1: per quantization group, P = A_q . (W_q - z)^T with tcgen05.mma
//           kind::i8 (int8 x int8 -> int32) into a TMEM accumulator that holds
//           only that group's sum;
//   step 2: the epilogue warps read P from TMEM, convert it with the fast
//           int-to-float of section 3.3 (Figure 3) and accumulate
//           acc += float(P) * s_w[row, group] in fp32 registers; at the end of
//           the tile Y = fp16(acc * s_a[token]) is scattered to the original
//           output columns (section 3.3, fused scatter epilogue).
// The group tile of the paper's software pipeline (section 3.3, Figure 4)
// becomes a pair of TMEM buffers: the MMA fills one group's accumulator while
// the epilogue drains the other.
//
// Tile: 128 packed weight rows (UMMA M) x 128 tokens (UMMA N), the whole K.
// Warp roles (512 threads):
//   warp 0      loader: per k-block, one bulk copy of the pre-packed weight
//               block (16 KB int8, already in the 128-byte-swizzled operand
//               layout; or 8 KB of uint4 codes) and one TMA tile of
//               activations (128 tokens x 128 bytes, hardware-swizzled)
//   warp 1      MMA issuer (one thread)
//   warp 2      TMEM allocator
//   warps 4-7   widening (step one for 4-bit rows): uint4 codes -> int8 (q - z)
//               written in the swizzled operand layout, four codes per 32-bit
//               operation (the vsub4 idea of section 3.3, done with a biased add)
//   warps 8-15  epilogue (two warps per TMEM lane quarter, 64 tokens each)
// Persistent CTAs walk the (row tile, token tile) list; consecutive tiles share
// a row tile, so CTAs running together read each weight block once from HBM.
// Every wait is bounded; on expiry the kernel records MX_ERR_TIMEOUT, all roles
// leave their loops, in-flight copies and MMAs are drained and TMEM is freed.
#include <mutex>

#include "mx_internal.cuh"
#include "sm100.cuh"

namespace mx {
namespace {

using namespace sm100;

constexpr int BM = 128;
constexpr int BN = 128;
constexpr int kStages = 4;
constexpr int kABytes = BM * kKBlock;          // int8 weight operand per stage
constexpr int kBBytes = BN * kKBlock;          // int8 activation operand per stage
constexpr int kRawBytes = BM * kKBlock / 2;    // packed uint4 codes per stage
constexpr int kThreads = 512;
constexpr int kWidenThreads = 128;
constexpr int kEpiWarps = 8;
constexpr uint32_t kTmemCols = 2 * BN;         // two int32 group accumulators

struct __align__(1024) Smem {
    uint8_t A[kStages][kABytes];
    uint8_t B[kStages][kBBytes];
    uint8_t Raw[kStages][kRawBytes];
    uint64_t full[kStages];       // loader -> widen/MMA: stage bytes landed
    uint64_t wdone[kStages];      // widen -> MMA: operand A ready
    uint64_t empty[kStages];      // MMA -> loader: stage consumed
    uint64_t acc_full[2];         // MMA -> epilogue: group accumulator complete
    uint64_t acc_empty[2];        // epilogue -> MMA: accumulator drained
    uint64_t mma_done;
    uint32_t tmem_base;
    int abort;
};

struct TcArgs {
    Geom g;
    const __half* s_a;
    __half* Y;
    int64_t ldy;
    int M;
    int n_tt;          // token tiles
    int n_tiles;       // (t8 + t4) * n_tt
    int32_t* debug;
    int32_t* status;
    uint64_t timeout_ns;
    int stall_test;
};

__device__ __forceinline__ uint32_t widen_lo(uint32_t w, uint32_t zc) {
    return ((w & 0x0F0F0F0Fu) + zc) ^ 0x80808080u;   // bytes q + 128 - z, then -128
}
__device__ __forceinline__ uint32_t widen_hi(uint32_t w, uint32_t zc) {
    return (((w >> 4) & 0x0F0F0F0Fu) + zc) ^ 0x80808080u;
}

__global__ void __launch_bounds__(kThreads, 1)
gemm_tc_kernel(const __grid_constant__ CUtensorMap amap, const __grid_constant__ TcArgs a) {
    extern __shared__ uint8_t smem_raw[];
    Smem& S = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const Geom& g = a.g;
    const int gpk = kKBlock / g.group;            // groups per k-block (1 or 2)
    const int ksteps = g.group / 32;              // MMA k-steps per group
    volatile int* abort = &S.abort;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&S.full[s], 1);
            mbar_init(&S.wdone[s], kWidenThreads);
            mbar_init(&S.empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&S.acc_full[b], 1);
            mbar_init(&S.acc_empty[b], kEpiWarps);
        }
        mbar_init(&S.mma_done, 1);
        S.abort = 0;
        fence_mbar_init();
        prefetch_tensormap(&amap);
    }
    if (warp == 2) {
        tmem_alloc(&S.tmem_base, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = S.tmem_base;

    if (warp == 0) {
        // ------------------------------------------------------------ loader
        if (lane == 0 && !a.stall_test) {
            int it = 0;
            for (int t = blockIdx.x; t < a.n_tiles; t += gridDim.x) {
                const int rt = t / a.n_tt, tt = t % a.n_tt;
                const bool eight = rt < g.t8;
                const int lt = eight ? rt : rt - g.t8;
                const uint32_t wbytes = eight ? kABytes : kRawBytes;
                const uint8_t* wsrc = eight
                    ? reinterpret_cast<const uint8_t*>(g.codes8) + size_t(lt) * g.kblocks * kABytes
                    : g.codes4 + size_t(lt) * g.kblocks * kRawBytes;
                for (int kb = 0; kb < g.kblocks; ++kb, ++it) {
                    const int s = it % kStages;
                    const uint32_t ph = (it / kStages) & 1;
                    if (!mbar_wait_bounded(&S.empty[s], ph ^ 1, abort, a.status, a.timeout_ns)) goto load_done;
                    mbar_arrive_expect_tx(&S.full[s], wbytes + kBBytes);
                    bulk_g2s(eight ? S.A[s] : S.Raw[s], wsrc + size_t(kb) * wbytes, wbytes, &S.full[s]);
                    tma_load_2d(S.B[s], &amap, kb * kKBlock, tt * BN, &S.full[s]);
                }
            }
        load_done:
            // every issued copy must land before the CTA can exit
            for (int j = max(0, it - kStages); j < it; ++j) {
                int dummy = 0;
                mbar_wait_bounded(&S.full[j % kStages], (j / kStages) & 1, &dummy, nullptr, a.timeout_ns);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t idesc = idesc_i8(BM, BN);
            int it = 0;
            uint32_t gc = 0;
            for (int t = blockIdx.x; t < a.n_tiles; t += gridDim.x) {
                for (int kb = 0; kb < g.kblocks; ++kb, ++it) {
                    const int s = it % kStages;
                    const uint32_t ph = (it / kStages) & 1;
                    if (!mbar_wait_bounded(&S.full[s], ph, abort, a.status, a.timeout_ns)) goto mma_out;
                    if (!mbar_wait_bounded(&S.wdone[s], ph, abort, a.status, a.timeout_ns)) goto mma_out;
                    tc_fence_after();
                    const uint32_t a0 = smem_u32(S.A[s]), b0 = smem_u32(S.B[s]);
                    for (int j = 0; j < gpk; ++j, ++gc) {
                        const uint32_t b = gc & 1, u = gc >> 1;
                        if (!mbar_wait_bounded(&S.acc_empty[b], (u & 1) ^ 1, abort, a.status, a.timeout_ns))
                            goto mma_out;
                        tc_fence_after();
                        for (int kk = 0; kk < ksteps; ++kk) {
                            const uint32_t off = uint32_t(j * g.group + kk * 32);
                            mma_i8(tmem + b * BN, sw128_kmajor_desc(a0 + off), sw128_kmajor_desc(b0 + off),
                                   idesc, kk > 0 ? 1u : 0u);
                        }
                        mma_commit(&S.acc_full[b]);
                    }
                    mma_commit(&S.empty[s]);
                }
            }
        mma_out:
            mma_commit(&S.mma_done);      // all MMAs issued so far complete before teardown
            int dummy = 0;
            mbar_wait_bounded(&S.mma_done, 0, &dummy, nullptr, a.timeout_ns);
        }
    } else if (warp >= 4 && warp < 8) {
        // ------------------------------------------------------------ widening (4-bit rows)
        const int wt = threadIdx.x - 4 * 32;
        int it = 0;
        for (int t = blockIdx.x; t < a.n_tiles; t += gridDim.x) {
            const int rt = t / a.n_tt;
            const bool eight = rt < g.t8;
            const int lt = eight ? rt : rt - g.t8;
            for (int kb = 0; kb < g.kblocks; ++kb, ++it) {
                const int s = it % kStages;
                const uint32_t ph = (it / kStages) & 1;
                uint32_t zc[4];
                if (!eight) {
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const int i = wt + kWidenThreads * j, r = i >> 2, c = i & 3;
                        const int gi = (kb * kKBlock + c * 32) / g.group;
                        const uint32_t z = g.zeros4[(size_t(lt) * g.G + gi) * kTileRows + r];
                        zc[j] = (0x80u - z) * 0x01010101u;
                    }
                }
                if (!mbar_wait_bounded(&S.full[s], ph, abort, a.status, a.timeout_ns)) goto widen_done;
                if (!eight) {
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const int i = wt + kWidenThreads * j, r = i >> 2, c = i & 3;
                        const uint4 w = *reinterpret_cast<const uint4*>(S.Raw[s] + i * 16);
                        uint4 o0, o1;
                        o0.x = widen_lo(w.x, zc[j]); o0.y = widen_hi(w.x, zc[j]);
                        o0.z = widen_lo(w.y, zc[j]); o0.w = widen_hi(w.y, zc[j]);
                        o1.x = widen_lo(w.z, zc[j]); o1.y = widen_hi(w.z, zc[j]);
                        o1.z = widen_lo(w.w, zc[j]); o1.w = widen_hi(w.w, zc[j]);
                        *reinterpret_cast<uint4*>(S.A[s] + swz128_offset(r, 2 * c)) = o0;
                        *reinterpret_cast<uint4*>(S.A[s] + swz128_offset(r, 2 * c + 1)) = o1;
                    }
                    fence_proxy_async_smem();
                }
                mbar_arrive(&S.wdone[s]);
            }
        }
    widen_done:;
    } else if (warp >= 8) {
        // ------------------------------------------------------------ epilogue
        const int q = warp & 3;                      // TMEM lane quarter of this warp
        const int row = q * 32 + lane;               // packed row within the tile
        const int cb = ((warp - 8) >> 2) * 64;       // first of this warp's 64 tokens
        const uint32_t lane_addr = tmem + (uint32_t(q * 32) << 16);
        uint32_t gc = 0;
        for (int t = blockIdx.x; t < a.n_tiles; t += gridDim.x) {
            const int rt = t / a.n_tt, tt = t % a.n_tt;
            const bool eight = rt < g.t8;
            const int lt = eight ? rt : rt - g.t8;
            const __half* sc = (eight ? g.scales8 : g.scales4) + size_t(lt) * g.G * kTileRows + row;
            const int orig = g.rowmap[rt * kTileRows + row];
            float acc[64];
#pragma unroll
            for (int c = 0; c < 64; ++c) acc[c] = 0.0f;
            for (int gi = 0; gi < g.G; ++gi, ++gc) {
                const float sw = __half2float(sc[size_t(gi) * kTileRows]);
                const uint32_t b = gc & 1, u = gc >> 1;
                // every lane waits; the warp leaves together if any lane gave up, because
                // the TMEM loads below are warp-collective (.sync.aligned)
                const bool ok = mbar_wait_bounded(&S.acc_full[b], u & 1, abort, a.status, a.timeout_ns);
                if (!__all_sync(0xffffffffu, ok)) goto epi_done;
                tc_fence_after();
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    uint32_t v[32];
                    tmem_ld_x32(lane_addr + b * BN + cb + h * 32, v);
                    tmem_wait_ld();
                    if (h == 1) {
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&S.acc_empty[b]);
                    }
#pragma unroll
                    for (int c = 0; c < 32; ++c)
                        acc[h * 32 + c] = __fmaf_rn(i2f_biased(int32_t(v[c])), sw, acc[h * 32 + c]);
                    if (a.debug != nullptr && orig >= 0) {
                        for (int c = 0; c < 32; ++c) {
                            const int m = tt * BN + cb + h * 32 + c;
                            if (m < a.M) a.debug[(size_t(m) * g.N + orig) * g.G + gi] = int32_t(v[c]);
                        }
                    }
                }
            }
            if (orig >= 0) {
#pragma unroll
                for (int c = 0; c < 64; ++c) {
                    const int m = tt * BN + cb + c;
                    if (m < a.M)
                        a.Y[int64_t(m) * a.ldy + orig] =
                            __float2half_rn(__fmul_rn(acc[c], __half2float(a.s_a[m])));
                }
            }
        }
    epi_done:;
    }

    __syncwarp();            // single-thread roles: reconverge before the CTA barrier
    tc_fence_before();
    __syncthreads();
    if (warp == 2) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// ---------------------------------------------------------------- host side
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn(cudaError_t* err) {
    static EncodeTiledFn fn = nullptr;
    static cudaError_t status = cudaSuccess;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        status = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q);
        if (status == cudaSuccess && q != cudaDriverEntryPointSuccess) status = cudaErrorNotSupported;
        fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    *err = status;
    return fn;
}

}  // namespace

size_t tc_smem_bytes() { return sizeof(Smem) + 1024; }

cudaError_t launch_gemm_tc(const mx_layout& L, const void* blob, const int8_t* Aq,
                           const uint16_t* s_a, int M, uint16_t* Y, int64_t ldy,
                           int32_t* debug_partials, int32_t* status, uint64_t timeout_ns,
                           int stall_test, cudaStream_t s) {
    if (M == 0) return cudaSuccess;
    cudaError_t e;
    EncodeTiledFn enc = encode_fn(&e);
    if (e != cudaSuccess) return e;
    CUtensorMap map;
    const cuuint64_t dims[2] = {cuuint64_t(L.K), cuuint64_t(M)};
    const cuuint64_t strides[1] = {cuuint64_t(L.K)};
    const cuuint32_t box[2] = {cuuint32_t(kKBlock), cuuint32_t(BN)};
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(&map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<int8_t*>(Aq), dims, strides,
                     box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;

    int dev = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    static int sms[64] = {};
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (sms[dev] == 0) {
        if ((e = cudaFuncSetAttribute(gemm_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      int(tc_smem_bytes()))) != cudaSuccess)
            return e;
        int n = 0;
        if ((e = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
        sms[dev] = n;
    }
    TcArgs a{};
    a.g = make_geom(L, blob);
    a.s_a = reinterpret_cast<const __half*>(s_a);
    a.Y = reinterpret_cast<__half*>(Y);
    a.ldy = ldy;
    a.M = M;
    a.n_tt = (M + BN - 1) / BN;
    a.n_tiles = (L.t8 + L.t4) * a.n_tt;
    a.debug = debug_partials;
    a.status = status;
    a.timeout_ns = timeout_ns;
    a.stall_test = stall_test;
    const int grid = a.n_tiles < sms[dev] ? a.n_tiles : sms[dev];
    gemm_tc_kernel<<<grid, kThreads, tc_smem_bytes(), s>>>(map, a);
    return cudaGetLastError();
}

}  // namespace mx
