// gemm_tcd.cu -- tensor-core mixed-precision GEMM for decode-sized M (sm_100a, path 6).
//
// The arithmetic is MixLLM's two-step dequantization (section 3.3): per
// quantization group an exact int32 product P of the 8-bit activations with the
// widened weight codes (q - z), then acc += float(P) * s_w in fp32, and
// Y = fp16(acc * s_a) scattered to the original output columns.
//
// Decode batches (a few to 128 tokens) have every weight used by few tokens: the
// step is bound by streaming the weights, and a pair MMA of N = 256 would mostly
// multiply padding.  Here each CTA works alone (tcgen05.mma.cta_group::1.kind::i8,
// M = 128 weight rows, N = NT tokens: the batch rounded up to 16), which on this
// part costs about half of a pair MMA per K step at small N.  The weights are read
// once: a unit is one row tile and a range of its k-blocks (a K split), and the
// fp32 sums of the splits are added in split order by a second kernel.  With small
// accumulators (NT columns) TMEM holds up to eight, so the epilogue drains them
// while the tensor core fills the next ones.
//
// Roles (16 warps, one CTA per SM, persistent over the units):
//   warp 0       weight copies: per stage one k-block of the tile's codes (uint4
//                raw, or pre-swizzled int8) and its zero points, from rotating lanes
//   warps 1-2    TMEM allocation (warp 1); one thread of each issues the MMAs and
//                commits of every second group (the accumulators of one parity).
//                At small N an MMA executes faster than a thread can issue the
//                next one, so two issuers keep the tensor core fed
//   warp 3       token copies: one TMA box of NT tokens x 128 bytes per stage.
//                Issuing a copy takes a thread long compared with a k-block's work
//                at decode sizes, so weights and tokens come from different warps
//   warps 4-     widening of 4-bit rows (uint4 -> int8 q - z), then an arrival on
//                the stage's "ready" barrier (8 warps; 4 at NT = 128, whose MMAs
//                take longer)
//   last warps   epilogue: warp w reads TMEM lane quarter w % 4, kEpiCols tokens each;
//                the group's partials are converted with cvt.rn.f32.s32 (exact:
//                |P| < 2^22) and scaled in fp32
// Every wait is bounded; on expiry the kernel records MX_ERR_TIMEOUT in the
// status word and every role leaves its loop.
#include <algorithm>

#include "mx_internal.cuh"
#include "sm100.cuh"

namespace mx {
namespace {

using namespace sm100;

constexpr int BM = 128;                         // weight rows per tile (UMMA M)
constexpr int kABytes = BM * kKBlock;           // int8 weight operand of one k-block
constexpr int kRawBytes = BM * kKBlock / 2;     // uint4 codes of one k-block
constexpr int kZBytes = 2 * BM;                 // zero points of up to two groups
constexpr int kWiden0 = 4;                      // first widening warp
constexpr int kScaleRing = 2;

template <int NT>
struct Cfg {
    static constexpr int kWidenWarps = NT <= 64 ? 8 : 4;
    static constexpr int kWidenThreads = kWidenWarps * 32;
    static constexpr int kWidenChunks = BM * 4 / kWidenThreads;   // 16-byte raw chunks per thread and stage
    static constexpr int kEpiWarp0 = kWiden0 + kWidenWarps;      // first epilogue warp (a multiple of 4)
    static constexpr int kEpiWarps = NT <= 64 ? 4 : 8;
    static constexpr int kEpiCols = NT * 4 / kEpiWarps;       // tokens per epilogue warp
    static constexpr int kPiece = kEpiCols >= 32 && NT <= 64 ? 32 : 16;   // TMEM columns per load
    static constexpr int kSlots = NT <= 64 ? 8 : 4;           // group accumulators in TMEM (even: one
                                                              // parity per issuer)
    static constexpr uint32_t kTmemCols = kSlots * NT <= 128 ? 128 : kSlots * NT <= 256 ? 256 : 512;
    static constexpr int kStages = NT <= 64 ? 6 : 5;
    static constexpr int kBBytes = NT * kKBlock;
    static constexpr int kThreads = (kEpiWarp0 + kEpiWarps) * 32;
    static_assert(kThreads == 512, "16 warps: 128 registers per thread");
    static_assert(kSlots * NT <= int(kTmemCols), "accumulators fit in TMEM");
    static_assert(kEpiCols % kPiece == 0, "whole loads");
};

template <int NT>
struct __align__(1024) Smem {
    uint8_t A[Cfg<NT>::kStages][kABytes];        // int8 weight operand (swizzled 128-byte rows)
    uint8_t B[Cfg<NT>::kStages][Cfg<NT>::kBBytes];   // the batch's tokens (swizzled by the copy)
    uint8_t R[Cfg<NT>::kStages][kRawBytes];      // raw uint4 codes of 4-bit rows
    uint8_t Z[Cfg<NT>::kStages][kZBytes];        // zero points of the stage's groups, [group][row]
    uint64_t full_w[Cfg<NT>::kStages];           // the stage's weight codes and zero points landed
    uint64_t full_t[Cfg<NT>::kStages];           // the stage's tokens landed
    uint64_t ready[Cfg<NT>::kStages];            // the stage's operands are in place
    uint64_t empty[Cfg<NT>::kStages];            // the MMAs reading the stage completed (one commit per group)
    uint64_t acc_full[Cfg<NT>::kSlots];          // a group accumulator is complete
    uint64_t acc_empty[Cfg<NT>::kSlots];         // the epilogue drained it
    uint64_t mma_done[2];                        // an issuer's MMAs all completed
    uint32_t tmem_base;
    int abort;
};

struct TcdArgs {
    Geom g;
    const __half* s_a;   // [M], or [M][G] with group-wise activation scales
    __half* Y;
    int64_t ldy;
    int M;
    int S;               // K splits
    int per;             // k-blocks per split (the last may be shorter)
    int n_units;         // row tiles x splits
    float* part;         // S > 1: fp32 split sums [S][M][N] (original column order)
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

__device__ __forceinline__ void tmem_ld_piece(uint32_t taddr, uint32_t (&r)[16]) { tmem_ld_x16(taddr, r); }
__device__ __forceinline__ void tmem_ld_piece(uint32_t taddr, uint32_t (&r)[32]) { tmem_ld_x32(taddr, r); }

struct Unit {
    int t;        // row tile
    int ks;       // K split
    int kb0, kb1; // its k-blocks [kb0, kb1)
    bool eight;
    int lt;       // index among the tiles of its kind
};

__device__ __forceinline__ Unit unit_of(const TcdArgs& a, int u) {
    Unit r;
    r.t = u / a.S;
    r.ks = u % a.S;
    r.kb0 = r.ks * a.per;
    r.kb1 = min(a.g.kblocks, r.kb0 + a.per);
    r.eight = r.t < a.g.t8;
    r.lt = r.eight ? r.t : r.t - a.g.t8;
    return r;
}

template <int NT, bool DEBUG, bool AG>
__global__ void __launch_bounds__(Cfg<NT>::kThreads, 1)
gemm_tcd_kernel(const __grid_constant__ CUtensorMap amap, const __grid_constant__ TcdArgs a) {
    using C = Cfg<NT>;
    extern __shared__ uint8_t smem_raw[];
    Smem<NT>& S = *reinterpret_cast<Smem<NT>*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const Geom& g = a.g;
    const int gpk = kKBlock / g.group;            // groups per k-block (1 or 2)
    const int ksteps = g.group / 32;              // MMA k-steps per group
    volatile int* abort = &S.abort;

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::kStages; ++s) {
            mbar_init(&S.full_w[s], 1);
            mbar_init(&S.full_t[s], 1);
            mbar_init(&S.ready[s], C::kWidenWarps);
            mbar_init(&S.empty[s], gpk);
        }
        for (int b = 0; b < C::kSlots; ++b) {
            mbar_init(&S.acc_full[b], 1);
            mbar_init(&S.acc_empty[b], C::kEpiWarps);
        }
        mbar_init(&S.mma_done[0], 1);
        mbar_init(&S.mma_done[1], 1);
        S.abort = 0;
        fence_mbar_init();
        prefetch_tensormap(&amap);
    }
    if (warp == 1) {
        tmem_alloc(&S.tmem_base, C::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = S.tmem_base;

    if (warp == 0 || warp == 3) {
        // ------------------------------------------------------------ copies
        // warp 0: the weight codes and zero points; warp 3: the tokens
        const bool wts = warp == 0;
        uint64_t* full = wts ? S.full_w : S.full_t;
        int it = 0;
        if (!a.stall_test) {
            for (int u = blockIdx.x; u < a.n_units; u += gridDim.x) {
                const Unit un = unit_of(a, u);
                for (int kb = un.kb0; kb < un.kb1; ++kb, ++it) {
                    const int s = it % C::kStages;
                    const uint32_t ph = (it / C::kStages) & 1;
                    bool ok = true;
                    if (lane == 0) ok = mbar_wait_bounded(&S.empty[s], ph ^ 1, abort, a.status, a.timeout_ns);
                    if (!__shfl_sync(0xffffffffu, ok, 0)) goto load_done;
                    if (wts) {
                        const uint32_t cbytes = uint32_t(un.eight ? kABytes : kRawBytes);
                        const uint32_t zbytes = un.eight ? 0u : uint32_t(gpk * BM);
                        if (lane == 0) mbar_arrive_expect_tx(&full[s], cbytes + zbytes);
                        __syncwarp();
                        const size_t blk = size_t(un.lt) * g.kblocks + kb;
                        if (lane == (it & 15)) {
                            if (un.eight)
                                bulk_g2s(S.A[s], reinterpret_cast<const uint8_t*>(g.codes8) + blk * kABytes, cbytes,
                                         &full[s]);
                            else
                                bulk_g2s(S.R[s], g.codes4 + blk * kRawBytes, cbytes, &full[s]);
                        }
                        if (zbytes != 0 && lane == 16 + (it & 15))
                            bulk_g2s(S.Z[s], g.zeros4 + (size_t(un.lt) * g.G + size_t(kb) * gpk) * kTileRows, zbytes,
                                     &full[s]);
                    } else {
                        // tokens past M read as zeros; the box is always counted whole
                        if (lane == 0) mbar_arrive_expect_tx(&full[s], uint32_t(C::kBBytes));
                        __syncwarp();
                        if (lane == (it & 31)) tma_load_3d(S.B[s], &amap, 0, 0, kb, &full[s]);
                    }
                }
            }
        }
    load_done:
        // no copy may target this CTA's shared memory after it exits
        if (lane == 0)
            for (int j = max(0, it - C::kStages); j < it; ++j) {
                int dummy = 0;
                mbar_wait_bounded(&full[j % C::kStages], (j / C::kStages) & 1, &dummy, nullptr, a.timeout_ns);
            }
    } else if (warp <= 2) {
        // ------------------------------------------------------------ MMAs
        // issuer `mine` takes the groups with gc % 2 == mine (accumulators of that parity)
        const uint32_t mine = uint32_t(warp - 1);
        if (lane == 0) {
            const uint32_t idesc = idesc_i8(BM, NT);
            int it = 0;
            uint32_t gc = 0;
            for (int u = blockIdx.x; u < a.n_units; u += gridDim.x) {
                const Unit un = unit_of(a, u);
                for (int kb = un.kb0; kb < un.kb1; ++kb, ++it) {
                    const int s = it % C::kStages;
                    const uint32_t ph = (it / C::kStages) & 1;
                    // a stage without a group of mine (one group per k-block): skip it
                    if (gpk == 1 && (gc & 1u) != mine) {
                        ++gc;
                        continue;
                    }
                    if (!mbar_wait_bounded(&S.ready[s], ph, abort, a.status, a.timeout_ns)) goto mma_out;
                    tc_fence_after();
                    const uint32_t a0 = smem_u32(S.A[s]), b0 = smem_u32(S.B[s]);
                    for (int j = 0; j < gpk; ++j, ++gc) {
                        if ((gc & 1u) != mine) continue;
                        const uint32_t b = gc % C::kSlots;
                        // use gc / kSlots of accumulator b: phase 0 is the epilogue's first release
                        if (!mbar_wait_bounded(&S.acc_empty[b], (gc / C::kSlots) & 1, abort, a.status, a.timeout_ns))
                            goto mma_out;
                        tc_fence_after();
                        // the group's first k-step overwrites the accumulator
                        for (int kk = 0; kk < ksteps; ++kk) {
                            const uint32_t off = uint32_t(j * g.group + kk * 32);
                            mma_i8(tmem + b * NT, sw128_kmajor_desc(a0 + off), sw128_kmajor_desc(b0 + off), idesc,
                                   kk > 0 ? 1u : 0u);
                        }
                        mma_commit(&S.acc_full[b]);
                        mma_commit(&S.empty[s]);
                    }
                }
            }
        mma_out:
            mma_commit(&S.mma_done[mine]);           // all MMAs issued so far complete before teardown
            int dummy = 0;
            mbar_wait_bounded(&S.mma_done[mine], 0, &dummy, nullptr, a.timeout_ns);
        }
    } else if (warp < C::kEpiWarp0) {
        // ------------------------------------------------------------ widening (4-bit rows)
        constexpr int kWidenThreads = C::kWidenThreads, kWidenChunks = C::kWidenChunks;
        const int wt = threadIdx.x - kWiden0 * 32;
        int it = 0;
        for (int u = blockIdx.x; u < a.n_units; u += gridDim.x) {
            const Unit un = unit_of(a, u);
            for (int kb = un.kb0; kb < un.kb1; ++kb, ++it) {
                const int s = it % C::kStages;
                const uint32_t ph = (it / C::kStages) & 1;
                // the weights to widen, then the tokens: the MMA needs both
                bool ok = mbar_wait_bounded(&S.full_w[s], ph, abort, a.status, a.timeout_ns);
                ok = ok && mbar_wait_bounded(&S.full_t[s], ph, abort, a.status, a.timeout_ns);
                if (!__all_sync(0xffffffffu, ok)) goto widen_done;
                if (!un.eight) {
                    const uint8_t* raw = S.R[s];
                    uint8_t* out = S.A[s];
                    const uint8_t* zs = S.Z[s];
                    uint4 w[kWidenChunks];
#pragma unroll
                    for (int j = 0; j < kWidenChunks; ++j)
                        w[j] = *reinterpret_cast<const uint4*>(raw + (wt + kWidenThreads * j) * 16);
#pragma unroll
                    for (int j = 0; j < kWidenChunks; ++j) {
                        const int i = wt + kWidenThreads * j, r = i >> 2, c = i & 3;
                        // (128 - z) in every byte, z of the group holding this chunk's 32 codes
                        const uint32_t zc = (0x80u - uint32_t(zs[(c * 32 / g.group) * BM + r])) * 0x01010101u;
                        uint4 o0, o1;
                        o0.x = widen_lo(w[j].x, zc); o0.y = widen_hi(w[j].x, zc);
                        o0.z = widen_lo(w[j].y, zc); o0.w = widen_hi(w[j].y, zc);
                        o1.x = widen_lo(w[j].z, zc); o1.y = widen_hi(w[j].z, zc);
                        o1.z = widen_lo(w[j].w, zc); o1.w = widen_hi(w[j].w, zc);
                        *reinterpret_cast<uint4*>(out + swz128_offset(r, 2 * c)) = o0;
                        *reinterpret_cast<uint4*>(out + swz128_offset(r, 2 * c + 1)) = o1;
                    }
                    fence_proxy_async_smem();
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&S.ready[s]);
            }
        }
    widen_done:;
    } else {
        // ------------------------------------------------------------ epilogue
        constexpr int kCols = C::kEpiCols, kPiece = C::kPiece;
        const int e = warp - C::kEpiWarp0;
        const int q = warp & 3;                      // TMEM lane quarter of this warp
        const int row = q * 32 + lane;               // weight row within the tile
        const int m0 = (e >> 2) * kCols;             // this warp's first token
        const uint32_t lane_addr = tmem + (uint32_t(q * 32) << 16) + uint32_t(m0);
        // every accumulator starts free
        if (lane == 0)
            for (int b = 0; b < C::kSlots; ++b) mbar_arrive(&S.acc_empty[b]);
        uint32_t gc = 0;
        for (int u = blockIdx.x; u < a.n_units; u += gridDim.x) {
            const Unit un = unit_of(a, u);
            const int g0 = un.kb0 * gpk, g1 = un.kb1 * gpk;     // this unit's groups
            const __half* sc = (un.eight ? g.scales8 : g.scales4) + size_t(un.lt) * g.G * kTileRows + row;
            const int orig = g.rowmap[un.t * kTileRows + row];
            float acc[kCols];
#pragma unroll
            for (int c = 0; c < kCols; ++c) acc[c] = 0.0f;
            __half swr[kScaleRing];
#pragma unroll
            for (int j = 0; j < kScaleRing; ++j) swr[j] = g0 + j < g1 ? sc[size_t(g0 + j) * kTileRows] : __float2half_rn(0.0f);
            for (int gi0 = g0; gi0 < g1; gi0 += kScaleRing) {
#pragma unroll
                for (int j = 0; j < kScaleRing; ++j) {
                    const int gi = gi0 + j;
                    if (gi >= g1) break;
                    const float sw = __half2float(swr[j]);
                    if (gi + kScaleRing < g1) swr[j] = sc[size_t(gi + kScaleRing) * kTileRows];
                    const uint32_t b = gc % C::kSlots;
                    const bool ok = mbar_wait_bounded(&S.acc_full[b], (gc / C::kSlots) & 1, abort, a.status,
                                                      a.timeout_ns);
                    if (!__all_sync(0xffffffffu, ok)) goto epi_done;
                    tc_fence_after();
                    const uint32_t col0 = lane_addr + b * NT;
                    auto consume = [&](const uint32_t (&v)[kPiece], int piece) {
#pragma unroll
                        for (int c = 0; c < kPiece; ++c) {
                            const int k = piece * kPiece + c;
                            float s2 = sw;
                            if constexpr (AG) {
                                const int m = m0 + k;
                                s2 = __fmul_rn(sw, m < a.M ? __half2float(a.s_a[int64_t(m) * g.G + gi]) : 0.0f);
                            }
                            acc[k] = __fmaf_rn(__int2float_rn(int32_t(v[c])), s2, acc[k]);
                        }
                        if (DEBUG && orig >= 0) {
#pragma unroll
                            for (int c = 0; c < kPiece; ++c) {
                                const int m = m0 + piece * kPiece + c;
                                if (m < a.M) a.debug[(size_t(m) * g.N + orig) * g.G + gi] = int32_t(v[c]);
                            }
                        }
                    };
                    constexpr int kPieces = kCols / kPiece;
                    uint32_t va[kPiece], vb[kPiece];
                    tmem_ld_piece(col0, va);
                    tmem_wait_ld();
#pragma unroll
                    for (int p = 0; p < kPieces; ++p) {
                        uint32_t (&cur)[kPiece] = (p & 1) ? vb : va;
                        uint32_t (&nxt)[kPiece] = (p & 1) ? va : vb;
                        if (p + 1 < kPieces) {
                            tmem_ld_piece(col0 + (p + 1) * kPiece, nxt);
                        } else {
                            // every load of the group landed: release the accumulator
                            tc_fence_before();
                            __syncwarp();
                            if (lane == 0) mbar_arrive(&S.acc_empty[b]);
                        }
                        consume(cur, p);
                        if (p + 1 < kPieces) tmem_wait_ld();
                    }
                    ++gc;
                }
            }
            if (orig >= 0) {
                // one split: Y; several: this split's fp32 sums, added in split order and
                // scaled by the reduction kernel
                float* part = a.S > 1 ? a.part + size_t(un.ks) * a.M * g.N : nullptr;
#pragma unroll
                for (int c = 0; c < kCols; ++c) {
                    const int m = m0 + c;
                    if (m < a.M) {
                        if (part) part[int64_t(m) * g.N + orig] = acc[c];
                        else a.Y[int64_t(m) * a.ldy + orig] =
                                 __float2half_rn(AG ? acc[c] : __fmul_rn(acc[c], __half2float(a.s_a[m])));
                    }
                }
            }
        }
    epi_done:;
    }

    __syncwarp();            // single-thread roles: reconverge before the block barrier
    tc_fence_before();
    __syncthreads();         // no MMA or copy of this CTA is in flight any more
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, C::kTmemCols);
    }
}

template <int NT>
size_t tcd_smem() { return sizeof(Smem<NT>) + 1024; }

template <int NT>
cudaError_t launch_nt(const mx_layout& L, const CUtensorMap& map, const TcdArgs& a, int grid, bool debug, int ag,
                      cudaStream_t s) {
    static bool configured[64] = {};
    int dev = 0;
    cudaError_t e;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!configured[dev]) {
        for (auto k : {gemm_tcd_kernel<NT, false, false>, gemm_tcd_kernel<NT, true, false>,
                       gemm_tcd_kernel<NT, false, true>, gemm_tcd_kernel<NT, true, true>})
            if ((e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, int(tcd_smem<NT>()))) !=
                cudaSuccess)
                return e;
        configured[dev] = true;
    }
    auto k = debug ? (ag ? gemm_tcd_kernel<NT, true, true> : gemm_tcd_kernel<NT, true, false>)
                   : (ag ? gemm_tcd_kernel<NT, false, true> : gemm_tcd_kernel<NT, false, false>);
    k<<<grid, Cfg<NT>::kThreads, tcd_smem<NT>(), s>>>(map, a);
    return cudaGetLastError();
}

}  // namespace

int tcd_tokens(int M) { return M <= 16 ? 16 : M <= 32 ? 32 : M <= 64 ? 64 : 128; }

// The K split with the smallest estimated time: the larger of the streaming time of
// the weights plus the split sums (written, then read back by the reduction) and the
// time of the k-blocks the busiest SM processes, plus a launch for the reduction.
// The estimates assume HBM at about 6 TB/s and about 0.2 us per k-block and SM.
int tcd_auto_split(const mx_layout& L, int M, int sms) {
    const int tiles = L.t8 + L.t4, nkb = L.kblocks;
    if (M <= 0 || sms <= 0) return 1;
    const double bw = 6.0e6, t_kb = 0.2, t_launch = 2.0;          // bytes per us, us, us
    const double wbytes = double(L.n8) * L.K + double(L.n4) * L.K / 2 + 2.5 * double(L.N) * L.G;
    int best = 1;
    double best_t = 1e30;
    for (int S = 1; S <= kTcdMaxSplit && S <= nkb; ++S) {
        const int per = (nkb + S - 1) / S;
        if ((nkb + per - 1) / per != S) continue;            // no empty split
        const double sums = S > 1 ? 8.0 * S * M * double(L.N) : 0.0;
        const double t = std::max(double((tiles * S + sms - 1) / sms) * per * t_kb, (wbytes + sums) / bw) +
                         (S > 1 ? t_launch : 0.0);
        if (t < best_t) {
            best_t = t;
            best = S;
        }
    }
    return best;
}

size_t tcd_split_bytes(const mx_layout& L, int M, int S) {
    return S > 1 ? (size_t(S) * size_t(M) * size_t(L.N) * 4 + 255) & ~size_t(255) : 0;
}

// Decode-sized M (1 .. 128): tokens in one tile of NT (the batch rounded up to 16),
// rows past M zero-filled by the copy and never stored.
cudaError_t launch_gemm_tcd(const mx_layout& L, const void* blob, const int8_t* Aq, const uint16_t* s_a, int M,
                            uint16_t* Y, int64_t ldy, int ag, int S, float* part, int32_t* debug_partials,
                            int32_t* status, uint64_t timeout_ns, int stall_test, int sms, cudaStream_t s) {
    if (M == 0) return cudaSuccess;
    if (M > kTcdMaxM || S < 1 || S > kTcdMaxSplit || (S > 1 && part == nullptr)) return cudaErrorInvalidValue;
    cudaError_t e;
    EncodeTiledFn enc = encode_fn(&e);
    if (e != cudaSuccess) return e;
    const int NT = tcd_tokens(M);
    // activations as a 3-D tensor [k-block][token][128 bytes]: one box brings one
    // k-block of the batch as swizzled 128-byte rows
    CUtensorMap map;
    const cuuint64_t dims[3] = {cuuint64_t(kKBlock), cuuint64_t(M), cuuint64_t(L.kblocks)};
    const cuuint64_t strides[2] = {cuuint64_t(L.K), cuuint64_t(kKBlock)};
    const cuuint32_t box[3] = {cuuint32_t(kKBlock), cuuint32_t(NT), 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = enc(&map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<int8_t*>(Aq), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
    TcdArgs a{};
    a.g = make_geom(L, blob);
    a.s_a = reinterpret_cast<const __half*>(s_a);
    a.Y = reinterpret_cast<__half*>(Y);
    a.ldy = ldy;
    a.M = M;
    S = std::min(S, L.kblocks);
    a.per = (L.kblocks + S - 1) / S;
    a.S = (L.kblocks + a.per - 1) / a.per;
    a.part = a.S > 1 ? part : nullptr;
    a.n_units = (L.t8 + L.t4) * a.S;
    a.debug = debug_partials;
    a.status = status;
    a.timeout_ns = timeout_ns;
    a.stall_test = stall_test;
    const int grid = std::min(a.n_units, sms);
    const bool dbg = debug_partials != nullptr;
    switch (NT) {
        case 16: e = launch_nt<16>(L, map, a, grid, dbg, ag, s); break;
        case 32: e = launch_nt<32>(L, map, a, grid, dbg, ag, s); break;
        case 64: e = launch_nt<64>(L, map, a, grid, dbg, ag, s); break;
        default: e = launch_nt<128>(L, map, a, grid, dbg, ag, s); break;
    }
    if (e != cudaSuccess || a.S == 1) return e;
    return launch_split_reduce(a.part, a.S, M, L.N, s_a, ag, Y, ldy, sms, s);
}

}  // namespace mx
