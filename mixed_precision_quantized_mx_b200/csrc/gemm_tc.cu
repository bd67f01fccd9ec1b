// gemm_tc.cu -- tensor-core mixed-precision GEMM for prefill-sized M (sm_100a).
//
// Two-step dequantization (MixLLM section 3.3) on 5th-generation tensor cores:
//   step 1: per quantization group, P = A_q . (W_q - z)^T with tcgen05.mma
//           kind::i8 (int8 x int8 -> int32) into a TMEM accumulator that holds
//           only that group's sum (the group's first MMA overwrites it),
//   step 2: the epilogue warps read P from TMEM, convert it with the fast
//           int-to-float of section 3.3 (Figure 3: add the bias integer, read the
//           bits as fp32, subtract the float bias) and accumulate
//           acc += float(P) * s_w[row, group]
//           in fp32 registers; at the end of the tile Y = fp16(acc * s_a[token])
//           is scattered to the original output columns (section 3.3, fused
//           scatter epilogue).
// The group tile of the paper's software pipeline (section 3.3, Figure 4)
// becomes a ring of four TMEM group accumulators: the MMA fills one while the
// epilogue drains the others.
//
// Tile: 128 packed weight rows (UMMA M) x 128 tokens (UMMA N), the whole K.
// A pipeline stage holds two k-blocks (256 columns of K): 32 KB of int8 weight
// operand and 32 KB of activations.  Each k-block of a stage is brought by its
// own copies from its own lane -- a bulk copy of the pre-packed weight block
// (int8 rows already in the 128-byte-swizzled operand layout, or the uint4 codes,
// which land in the upper half of the operand buffer) and a 3-D TMA box of
// activations -- because on sm_100a copies issued by one thread complete one
// after another, while copies from different lanes and warps overlap.
// Warp roles (512 threads):
//   warp 0      weight copies (lanes 0, 1) warp 3  activation copies (lanes 0, 1)
//   warps 1, 2  MMA issuers, one thread each, taking alternate groups: a thread
//               spends ~150 ns in every barrier wait or commit, about as long as
//               one group's MMAs take, so two of them keep the tensor core busy
//               (warp 2 also allocates TMEM)
//   warps 4-7   widening (step one for 4-bit rows): uint4 codes -> int8 (q - z)
//               in place, four codes per 32-bit operation (the vsub4 idea of
//               section 3.3, done with a biased add)
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
constexpr int kKbPerStage = 2;                 // k-blocks per pipeline stage
constexpr int kStages = 3;
constexpr int kABytes = BM * kKBlock;          // int8 weight operand of one k-block
constexpr int kBBytes = BN * kKBlock;          // int8 activation operand of one k-block
constexpr int kRawBytes = BM * kKBlock / 2;    // uint4 codes of one k-block
// the uint4 codes of a stage land at the top of its weight-operand buffer and are
// widened in place, k-block after k-block, into the int8 operand below them
constexpr int kRawBase = kKbPerStage * (kABytes - kRawBytes);
constexpr int kThreads = 512;
constexpr int kWidenThreads = 128;
constexpr int kEpiWarps = 8;
constexpr int kAccBufs = 4;                     // int32 group accumulators in TMEM
constexpr uint32_t kTmemCols = kAccBufs * BN;   // all 512 columns
constexpr int kWidenBarrier = 1;                // named barrier of the widening warps
constexpr int kMmaIssuers = 2;                  // MMA-issuing threads, alternating groups
constexpr int kScaleRing = 4;                   // group scales in flight per epilogue thread
constexpr int kSatGroups = 8;                   // group-wise activation scales staged per refill

struct __align__(1024) Smem {
    uint8_t A[kStages][kKbPerStage * kABytes];  // raw uint4 codes land at A + kRawBase
    uint8_t B[kStages][kKbPerStage * kBBytes];
    uint64_t full[kStages];       // both copies of the stage landed (2 arrivals + bytes)
    uint64_t wdone[kStages];      // widen -> MMA: weight operand ready
    uint64_t empty[kStages];      // MMA issuers -> loaders: stage consumed (one commit each)
    uint64_t acc_full[kAccBufs];  // MMA -> epilogue: group accumulator complete
    uint64_t acc_empty[kAccBufs]; // epilogue -> MMA: accumulator drained and re-armed
    uint64_t mma_done[kMmaIssuers];
    // group-wise activation scales: each epilogue warp's 64 tokens for 8 groups
    __align__(16) __half sat[kEpiWarps][kSatGroups][BN / 2];
    uint32_t tmem_base;
    int abort;
};

struct TcArgs {
    Geom g;
    const __half* s_a;   // [M], or [M][G] with group-wise activation scales (ag != 0)
    int ag;
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

// Drain every issued stage (bounded) so that no copy targets this CTA's shared
// memory after it exits.
__device__ __forceinline__ void drain_stages(Smem& S, int issued, uint64_t timeout_ns) {
    for (int j = max(0, issued - kStages); j < issued; ++j) {
        int dummy = 0;
        mbar_wait_bounded(&S.full[j % kStages], (j / kStages) & 1, &dummy, nullptr, timeout_ns);
    }
}

// AG: group-wise activation scales (s_a [M][G]) instead of one per token
template <bool DEBUG, bool AG>
__global__ void __launch_bounds__(kThreads, 1)
gemm_tc_kernel(const __grid_constant__ CUtensorMap amap, const __grid_constant__ TcArgs a) {
    extern __shared__ uint8_t smem_raw[];
    Smem& S = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const Geom& g = a.g;
    const int gpk = kKBlock / g.group;            // groups per k-block (1 or 2)
    const int ksteps = g.group / 32;              // MMA k-steps per group
    const int n_ss = (g.kblocks + kKbPerStage - 1) / kKbPerStage;   // stages per tile
    volatile int* abort = &S.abort;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&S.full[s], 2);
            mbar_init(&S.wdone[s], kWidenThreads / 32);
            mbar_init(&S.empty[s], kMmaIssuers);
        }
        for (int b = 0; b < kAccBufs; ++b) {
            mbar_init(&S.acc_full[b], 1);
            mbar_init(&S.acc_empty[b], kEpiWarps);
        }
        for (int m = 0; m < kMmaIssuers; ++m) mbar_init(&S.mma_done[m], 1);
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

    if (warp == 0 || warp == 3) {
        // ------------------------------------------------------------ loaders
        // lane kbi copies k-block kbi of each stage: copies from one thread complete
        // one after another, copies from different lanes overlap
        if (lane < kKbPerStage && !a.stall_test) {
            constexpr uint32_t kLanes = (1u << kKbPerStage) - 1u;   // the issuing lanes
            const bool weights = warp == 0;
            int it = 0;
            for (int t = blockIdx.x; t < a.n_tiles; t += gridDim.x) {
                const int rt = t / a.n_tt, tt = t % a.n_tt;
                const bool eight = rt < g.t8;
                const int lt = eight ? rt : rt - g.t8;
                for (int sp = 0; sp < n_ss; ++sp, ++it) {
                    const int s = it % kStages;
                    const uint32_t ph = (it / kStages) & 1;
                    bool ok = true;
                    if (lane == 0) ok = mbar_wait_bounded(&S.empty[s], ph ^ 1, abort, a.status, a.timeout_ns);
                    if (!__shfl_sync(kLanes, ok, 0)) goto load_done;
                    const int kb0 = sp * kKbPerStage;
                    const int nkb = min(kKbPerStage, g.kblocks - kb0);
                    if (weights) {
                        const uint32_t per = uint32_t(eight ? kABytes : kRawBytes);
                        if (lane == 0) mbar_arrive_expect_tx(&S.full[s], uint32_t(nkb) * per);
                        __syncwarp(kLanes);
                        if (lane < nkb) {
                            const uint8_t* src =
                                eight ? reinterpret_cast<const uint8_t*>(g.codes8) +
                                            (size_t(lt) * g.kblocks + kb0 + lane) * kABytes
                                      : g.codes4 + (size_t(lt) * g.kblocks + kb0 + lane) * kRawBytes;
                            bulk_g2s((eight ? S.A[s] : S.A[s] + kRawBase) + lane * per, src, per, &S.full[s]);
                        }
                    } else {
                        // one box per k-block; a missing last one reads as zeros
                        if (lane == 0) mbar_arrive_expect_tx(&S.full[s], kKbPerStage * kBBytes);
                        __syncwarp(kLanes);
                        tma_load_3d(S.B[s] + lane * kBBytes, &amap, 0, tt * BN, kb0 + lane, &S.full[s]);
                    }
                }
            }
        load_done:
            if (lane == 0) drain_stages(S, it, a.timeout_ns);
        }
    } else if (warp == 1 || warp == 2) {
        // ------------------------------------------------------------ MMA issuers
        if (lane == 0) {
            const uint32_t mine = warp - 1;              // this issuer takes groups gc % 2 == mine
            const uint32_t idesc = idesc_i8(BM, BN);
            int it = 0;
            uint32_t gc = 0;
            for (int t = blockIdx.x; t < a.n_tiles; t += gridDim.x) {
                for (int sp = 0; sp < n_ss; ++sp, ++it) {
                    const int s = it % kStages;
                    const uint32_t ph = (it / kStages) & 1;
                    if (!mbar_wait_bounded(&S.full[s], ph, abort, a.status, a.timeout_ns)) goto mma_out;
                    if (!mbar_wait_bounded(&S.wdone[s], ph, abort, a.status, a.timeout_ns)) goto mma_out;
                    tc_fence_after();
                    const int nkb = min(kKbPerStage, g.kblocks - sp * kKbPerStage);
                    for (int kbi = 0; kbi < nkb; ++kbi) {
                        const uint32_t a0 = smem_u32(S.A[s] + kbi * kABytes);
                        const uint32_t b0 = smem_u32(S.B[s] + kbi * kBBytes);
                        for (int j = 0; j < gpk; ++j, ++gc) {
                            if ((gc & 1) != mine) continue;
                            const uint32_t b = gc % kAccBufs, u = gc / kAccBufs;
                            if (!mbar_wait_bounded(&S.acc_empty[b], (u & 1) ^ 1, abort, a.status, a.timeout_ns))
                                goto mma_out;
                            tc_fence_after();
                            // the group's first k-step overwrites the accumulator, the rest add
                            for (int kk = 0; kk < ksteps; ++kk) {
                                const uint32_t off = uint32_t(j * g.group + kk * 32);
                                mma_i8(tmem + b * BN, sw128_kmajor_desc(a0 + off), sw128_kmajor_desc(b0 + off),
                                       idesc, kk > 0 ? 1u : 0u);
                            }
                            mma_commit(&S.acc_full[b]);
                        }
                    }
                    mma_commit(&S.empty[s]);   // arrives once this issuer's MMAs on the stage are done
                }
            }
        mma_out:
            mma_commit(&S.mma_done[mine]);  // all MMAs issued so far complete before teardown
            int dummy = 0;
            mbar_wait_bounded(&S.mma_done[mine], 0, &dummy, nullptr, a.timeout_ns);
        }
    } else if (warp >= 4 && warp < 8) {
        // ------------------------------------------------------------ widening (4-bit rows)
        const int wt = threadIdx.x - 4 * 32;
        int it = 0;
        for (int t = blockIdx.x; t < a.n_tiles; t += gridDim.x) {
            const int rt = t / a.n_tt;
            const bool eight = rt < g.t8;
            const int lt = eight ? rt : rt - g.t8;
            const uint8_t* zrow = g.zeros4 + size_t(lt) * g.G * kTileRows;
            // zero points of this thread's four chunks in the two k-blocks of stage sp, as
            // (128 - z) per byte; two register sets alternate between even and odd stages
            // so each is loaded two stages before its use
            auto load_z = [&](int sp, uint32_t (&zc)[2][4]) {
#pragma unroll
                for (int kbi = 0; kbi < kKbPerStage; ++kbi)
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const int kb = sp * kKbPerStage + kbi;
                        const int i = wt + kWidenThreads * j, r = i >> 2, c = i & 3;
                        const int gi = (kb * kKBlock + c * 32) / g.group;
                        zc[kbi][j] = kb < g.kblocks
                            ? (0x80u - uint32_t(zrow[size_t(gi) * kTileRows + r])) * 0x01010101u : 0u;
                    }
            };
            // one stage: wait for its copies, widen the uint4 codes in place, release it
            auto widen_stage = [&](int sp, const uint32_t (&zc)[2][4]) -> bool {
                const int s = it % kStages;
                const uint32_t ph = (it / kStages) & 1;
                const int nkb = min(kKbPerStage, g.kblocks - sp * kKbPerStage);
                const bool ok = mbar_wait_bounded(&S.full[s], ph, abort, a.status, a.timeout_ns);
                __syncwarp();   // the named barrier is warp-collective
                // one decision for all 128 widening threads: the in-place conversion below
                // needs every one of them at the named barrier
                if (!named_bar_and(kWidenBarrier, kWidenThreads, ok)) return false;
                if (!eight) {
                    const uint8_t* raw = S.A[s] + kRawBase;
                    for (int kbi = 0; kbi < nkb; ++kbi) {
                        uint4 w[4];
#pragma unroll
                        for (int j = 0; j < 4; ++j)
                            w[j] = *reinterpret_cast<const uint4*>(raw + kbi * kRawBytes + (wt + kWidenThreads * j) * 16);
                        // once the int8 block reaches the codes, every thread reads before any writes
                        if ((kbi + 1) * kABytes > kRawBase) named_bar_and(kWidenBarrier, kWidenThreads, true);
                        uint8_t* out = S.A[s] + kbi * kABytes;
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            const int i = wt + kWidenThreads * j, r = i >> 2, c = i & 3;
                            const uint32_t z = kbi ? zc[1][j] : zc[0][j];
                            uint4 o0, o1;
                            o0.x = widen_lo(w[j].x, z); o0.y = widen_hi(w[j].x, z);
                            o0.z = widen_lo(w[j].y, z); o0.w = widen_hi(w[j].y, z);
                            o1.x = widen_lo(w[j].z, z); o1.y = widen_hi(w[j].z, z);
                            o1.z = widen_lo(w[j].w, z); o1.w = widen_hi(w[j].w, z);
                            *reinterpret_cast<uint4*>(out + swz128_offset(r, 2 * c)) = o0;
                            *reinterpret_cast<uint4*>(out + swz128_offset(r, 2 * c + 1)) = o1;
                        }
                    }
                    fence_proxy_async_smem();
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&S.wdone[s]);
                ++it;
                return true;
            };
            uint32_t zA[2][4] = {}, zB[2][4] = {};
            if (!eight) {
                load_z(0, zA);
                if (n_ss > 1) load_z(1, zB);
            }
            for (int sp = 0; sp < n_ss; sp += 2) {
                if (!widen_stage(sp, zA)) goto widen_done;
                if (!eight && sp + 2 < n_ss) load_z(sp + 2, zA);
                if (sp + 1 < n_ss) {
                    if (!widen_stage(sp + 1, zB)) goto widen_done;
                    if (!eight && sp + 3 < n_ss) load_z(sp + 3, zB);
                }
            }
        }
    widen_done:;
    } else if (warp >= 8) {
        // ------------------------------------------------------------ epilogue
        const int q = warp & 3;                      // TMEM lane quarter of this warp
        const int row = q * 32 + lane;               // packed row within the tile
        const int cb = ((warp - 8) >> 2) * 64;       // first of this warp's 64 tokens
        const uint32_t lane_addr = tmem + (uint32_t(q * 32) << 16);
        const float2 nbias = make_float2(-kI2FBias, -kI2FBias);
        uint32_t gc = 0;
        for (int t = blockIdx.x; t < a.n_tiles; t += gridDim.x) {
            const int rt = t / a.n_tt, tt = t % a.n_tt;
            const bool eight = rt < g.t8;
            const int lt = eight ? rt : rt - g.t8;
            const __half* sc = (eight ? g.scales8 : g.scales4) + size_t(lt) * g.G * kTileRows + row;
            const int orig = g.rowmap[rt * kTileRows + row];
            float2 acc[32];
#pragma unroll
            for (int c = 0; c < 32; ++c) acc[c] = make_float2(0.0f, 0.0f);
            // group scales live in a ring of kScaleRing registers, each loaded kScaleRing
            // groups before its use; the group loop is unrolled by kScaleRing so every
            // ring slot is a fixed register and no instruction waits on a young load
            // (the ring holds the raw fp16 values: converting at the load would wait for it)
            __half swr[kScaleRing];
#pragma unroll
            for (int j = 0; j < kScaleRing; ++j)
                swr[j] = j < g.G ? sc[size_t(j) * kTileRows] : __float2half_rn(0.0f);
            for (int gi0 = 0; gi0 < g.G; gi0 += kScaleRing) {
#pragma unroll
                for (int j = 0; j < kScaleRing; ++j) {
                    const int gi = gi0 + j;
                    if (gi >= g.G) break;
                    const float sw = __half2float(swr[j]);
                    if (gi + kScaleRing < g.G) swr[j] = sc[size_t(gi + kScaleRing) * kTileRows];
                    const float2 s2 = make_float2(sw, sw);
                    const uint32_t b = gc % kAccBufs, u = gc / kAccBufs;
                    // every lane waits; the warp leaves together if any lane gave up, because
                    // the TMEM loads below are warp-collective (.sync.aligned)
                    const bool ok = mbar_wait_bounded(&S.acc_full[b], u & 1, abort, a.status, a.timeout_ns);
                    if (!__all_sync(0xffffffffu, ok)) goto epi_done;
                    tc_fence_after();
                    // group-wise activations: refill this warp's window of token scales
                    // every kSatGroups groups (warp-private, so only the warp synchronises)
                    __half (*sat)[BN / 2] = S.sat[warp - 8];
                    if (AG && gi % kSatGroups == 0) {
                        __syncwarp();
                        for (int i = lane; i < kSatGroups * (BN / 2); i += 32) {
                            const int w = i / (BN / 2), t = i % (BN / 2), m = tt * BN + cb + t;
                            sat[w][t] = gi + w < g.G && m < a.M ? a.s_a[int64_t(m) * g.G + gi + w]
                                                                : __float2half_rn(0.0f);
                        }
                        __syncwarp();
                    }
                    // drain the group's 64 columns in eight 8-column chunks, loading chunk
                    // h+1 while chunk h is converted
                    const uint32_t col0 = lane_addr + b * BN + cb;
                    uint32_t va[8], vb[8];
                    tmem_ld_x8(col0, va);
                    tmem_wait_ld();
#pragma unroll
                    for (int h = 0; h < 8; ++h) {
                        uint32_t (&v)[8] = (h & 1) ? vb : va;
                        uint32_t (&vn)[8] = (h & 1) ? va : vb;
                        if (h < 7) tmem_ld_x8(col0 + (h + 1) * 8, vn);
                        // acc += (float(bias + P) - bias) * s_w: the fast int-to-float adds the
                        // bias as an integer, two columns per float instruction
                        if constexpr (AG) {
                            // group-wise activations: column (token) m also takes s_a[m][gi]
                            const uint4 sv = *reinterpret_cast<const uint4*>(&sat[gi % kSatGroups][h * 8]);
                            const __half2* sh = reinterpret_cast<const __half2*>(&sv);
#pragma unroll
                            for (int c = 0; c < 4; ++c) {
                                const float2 sa2 = __half22float2(sh[c]);
                                const float2 f = add2(make_float2(__uint_as_float(v[2 * c] + kI2FBiasBits),
                                                                  __uint_as_float(v[2 * c + 1] + kI2FBiasBits)),
                                                      nbias);
                                acc[h * 4 + c] = fma2(f, make_float2(__fmul_rn(sw, sa2.x), __fmul_rn(sw, sa2.y)),
                                                      acc[h * 4 + c]);
                            }
                        } else {
#pragma unroll
                            for (int c = 0; c < 4; ++c) {
                                const float2 f = add2(make_float2(__uint_as_float(v[2 * c] + kI2FBiasBits),
                                                                  __uint_as_float(v[2 * c + 1] + kI2FBiasBits)),
                                                      nbias);
                                acc[h * 4 + c] = fma2(f, s2, acc[h * 4 + c]);
                            }
                        }
                        if (DEBUG && orig >= 0) {
#pragma unroll
                            for (int c = 0; c < 8; ++c) {
                                const int m = tt * BN + cb + h * 8 + c;
                                if (m < a.M)
                                    a.debug[(size_t(m) * g.N + orig) * g.G + gi] = int32_t(v[c]);
                            }
                        }
                        if (h < 7) tmem_wait_ld();
                    }
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&S.acc_empty[b]);
                    ++gc;
                }
            }
            if (orig >= 0) {
#pragma unroll
                for (int c = 0; c < 32; ++c) {
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const int m = tt * BN + cb + 2 * c + e;
                        if (m < a.M) {
                            const float v = e ? acc[c].y : acc[c].x;
                            // group-wise scales were applied per group
                            a.Y[int64_t(m) * a.ldy + orig] =
                                __float2half_rn(AG ? v : __fmul_rn(v, __half2float(a.s_a[m])));
                        }
                    }
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

}  // namespace

// ---------------------------------------------------------------- host side
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

size_t tc_smem_bytes() { return sizeof(Smem) + 1024; }

cudaError_t launch_gemm_tc(const mx_layout& L, const void* blob, const int8_t* Aq,
                           const uint16_t* s_a, int M, uint16_t* Y, int64_t ldy, int ag,
                           int32_t* debug_partials, int32_t* status, uint64_t timeout_ns,
                           int stall_test, cudaStream_t s) {
    if (M == 0) return cudaSuccess;
    cudaError_t e;
    EncodeTiledFn enc = encode_fn(&e);
    if (e != cudaSuccess) return e;
    // activations as a 3-D tensor [k-block][token][128 bytes]: one box brings one
    // k-block of BN tokens as a swizzled 128-byte-row block
    CUtensorMap map;
    const cuuint64_t dims[3] = {cuuint64_t(kKBlock), cuuint64_t(M), cuuint64_t(L.kblocks)};
    const cuuint64_t strides[2] = {cuuint64_t(L.K), cuuint64_t(kKBlock)};
    const cuuint32_t box[3] = {cuuint32_t(kKBlock), cuuint32_t(BN), 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = enc(&map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<int8_t*>(Aq), dims, strides,
                     box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;

    int dev = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    static int sms[64] = {};
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (sms[dev] == 0) {
        for (auto k : {gemm_tc_kernel<false, false>, gemm_tc_kernel<true, false>, gemm_tc_kernel<false, true>,
                       gemm_tc_kernel<true, true>})
            if ((e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, int(tc_smem_bytes()))) !=
                cudaSuccess)
                return e;
        int n = 0;
        if ((e = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
        sms[dev] = n;
    }
    TcArgs a{};
    a.g = make_geom(L, blob);
    a.s_a = reinterpret_cast<const __half*>(s_a);
    a.ag = ag;
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
    auto k = debug_partials ? (ag ? gemm_tc_kernel<true, true> : gemm_tc_kernel<true, false>)
                            : (ag ? gemm_tc_kernel<false, true> : gemm_tc_kernel<false, false>);
    k<<<grid, kThreads, tc_smem_bytes(), s>>>(map, a);
    return cudaGetLastError();
}

}  // namespace mx
