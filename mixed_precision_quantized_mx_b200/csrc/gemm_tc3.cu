// gemm_tc3.cu -- tensor-core mixed-precision GEMM on CTA pairs with 256-token
// tiles (sm_100a, prefill M).
//
// The arithmetic is MixLLM's two-step dequantization (section 3.3): per
// quantization group an exact int32 product P of the 8-bit activations with the
// widened weight codes (q - z) on the tensor cores, then acc += float(P) * s_w in
// fp32, and Y = fp16(acc * s_a) scattered to the original output columns (the
// 8-bit and 4-bit row sets are independent sub-problems, section 3.1.1).
//
// The tile is 256 weight rows x 256 tokens on two SMs: one
// tcgen05.mma.cta_group::2.kind::i8 of M = 256, N = 256, K = 32 per step, each CTA
// holding 128 weight rows and 128 tokens in shared memory.  Against a 128-token
// tile this halves the widening work and the weight staging per multiply-
// accumulate, and N = 256 is the MMA shape that runs at the full int8 rate.
// Each CTA's TMEM (512 columns) holds two group accumulators of 128 rows x 256
// tokens: the first MMA of a group overwrites one, and while the tensor core
// fills it the epilogue drains the other.
//
// The epilogue converts P with the hardware int-to-float instruction (exact:
// |P| < 2^22).  The paper's fast conversion (section 3.3, Figure 3) preloads the
// accumulator with a bias integer so that a float subtract replaces the
// conversion, because the A100 converts slowly; on this part the conversion
// runs about as fast as an fp32 add, and the preload would write 128 KB of TMEM
// per group and CTA, as much as the epilogue reads.  P and Y are the same either
// way.
//
// Stages are one k-block (128 columns of K): 16 KB of int8 weight operand,
// 16 KB of this CTA's tokens, 8 KB of raw uint4 codes and the zero points, five
// in flight.  The raw codes land in their own buffer, so widening needs no
// barrier between its reads and writes.
//
// Roles (16 warps; registers moved from the copy, MMA and widening warps to the
// epilogue with setmaxnreg):
//   warp 0      weight copies: codes (uint4 raw, or pre-swizzled int8) and the
//               zero points of the stage, from rotating lanes
//   warp 1      token copies: one TMA box of 128 tokens x 128 bytes per stage
//   warps 2-3   TMEM allocation (warp 2, both CTAs); in the even CTA one thread
//               of each issues the pair MMAs of one accumulator (even or odd
//               groups) and commits to barriers in both CTAs.  Issuing a group
//               blocks while the tensor core still runs the one before it, so a
//               single issuer would notice the release of the other accumulator
//               only after that; with one issuer per accumulator each waits on
//               its own.
//   warps 4-7   widening of 4-bit rows (uint4 -> int8 q - z), then an arrival
//               on the even CTA's "stage ready" barrier
//   warps 8-15  epilogue: warp w reads TMEM lane quarter w % 4, accumulator
//               columns 128 * ((w - 8) / 4) .. +127
// Every wait is bounded; on expiry the kernel records MX_ERR_TIMEOUT in the
// status word and every role leaves its loop.
#include <algorithm>

#include "mx_internal.cuh"
#include "sm100.cuh"

namespace mx {
namespace {

using namespace sm100;

constexpr int BM = 128;                         // weight rows per CTA (the pair: 256)
constexpr int BN = 256;                         // tokens per pair tile (MMA N)
constexpr int BNH = BN / 2;                     // tokens staged per CTA
constexpr int kStages = 5;
constexpr int kABytes = BM * kKBlock;           // int8 weight operand of one k-block
constexpr int kBBytes = BNH * kKBlock;          // this CTA's tokens of one k-block
constexpr int kRawBytes = BM * kKBlock / 2;     // uint4 codes of one k-block
constexpr int kZBytes = 2 * BM;                 // zero points of up to two groups
constexpr int kSlots = 2;                       // group accumulators in TMEM
constexpr int kSlotCols = BN;                   // TMEM columns of one accumulator
constexpr uint32_t kTmemCols = 512;
constexpr int kWidenWarps = 4;
constexpr int kWidenThreads = kWidenWarps * 32;
constexpr int kWidenChunks = BM * 4 / kWidenThreads;   // 16-byte raw chunks per thread and stage
constexpr int kEpiWarps = 8;
constexpr int kEpiCols = 128;                   // accumulator columns (tokens) per epilogue warp
constexpr int kThreads = 16 * 32;
constexpr int kScaleRing = 4;
constexpr int kPiece = 32;                      // TMEM columns per epilogue load
constexpr int kSatGroups = 4;
static_assert(kSlots * kSlotCols <= int(kTmemCols), "accumulators fit in TMEM");
static_assert(kEpiWarps * kEpiCols == 4 * BN, "two epilogue warps per TMEM lane quarter");
static_assert(kWidenChunks * kWidenThreads == BM * 4, "every raw chunk widened once");

// registers per thread after the split: 256 threads at kLowRegs, 256 at kEpiRegs,
// together the kLaunchRegs x 512 the block is launched with (a split above the
// launch would leave setmaxnreg.inc waiting for ever, so the launcher checks the
// compiled count)
constexpr uint32_t kLaunchRegs = 128;
constexpr uint32_t kLowRegs = 72;
constexpr uint32_t kEpiRegs = 184;
static_assert(256 * kLowRegs + 256 * kEpiRegs == kLaunchRegs * kThreads, "register split adds up to the launch");

struct __align__(1024) Smem {
    uint8_t A[kStages][kABytes];   // int8 weight operand (swizzled 128-byte rows)
    uint8_t B[kStages][kBBytes];   // this CTA's 128 tokens (swizzled by the copy)
    uint8_t R[kStages][kRawBytes]; // raw uint4 codes of 4-bit rows
    uint8_t Z[kStages][kZBytes];   // zero points of the stage's groups, [group][row]
    uint64_t full_w[kStages];      // this CTA's weight codes and zero points of the stage landed
    uint64_t full_t[kStages];      // this CTA's tokens of the stage landed
    uint64_t ready[kStages];       // (even CTA) both CTAs' operands of the stage are in place
    uint64_t empty[kStages];       // (both) the pair MMAs reading the stage completed (one commit
                                   // per group of the stage)
    uint64_t acc_full[kSlots];     // (both) a group accumulator is complete
    uint64_t acc_empty[kSlots];    // (even CTA) both CTAs drained and re-armed it
    uint64_t mma_done[kSlots];     // (even CTA) an issuer's MMAs all completed
    __align__(16) __half sat[kEpiWarps][kSatGroups][kEpiCols];   // group-wise token scales
    uint32_t tmem_base;
    int abort;
};

struct Tc3Args {
    Geom g;
    const __half* s_a;   // [M], or [M][G] with group-wise activation scales
    __half* Y;
    int64_t ldy;
    int M;
    int n_tt;            // token tiles of BN
    int n_units;         // row-tile pairs x token tiles
    int32_t* debug;
    int32_t* status;
    uint64_t timeout_ns;
    int stall_test;
};

__device__ __forceinline__ void tmem_ld_piece(uint32_t taddr, uint32_t (&r)[16]) { tmem_ld_x16(taddr, r); }
__device__ __forceinline__ void tmem_ld_piece(uint32_t taddr, uint32_t (&r)[32]) { tmem_ld_x32(taddr, r); }

__device__ __forceinline__ uint32_t widen_lo(uint32_t w, uint32_t zc) {
    return ((w & 0x0F0F0F0Fu) + zc) ^ 0x80808080u;   // bytes q + 128 - z, then -128
}
__device__ __forceinline__ uint32_t widen_hi(uint32_t w, uint32_t zc) {
    return (((w >> 4) & 0x0F0F0F0Fu) + zc) ^ 0x80808080u;
}

// Unit u of the persistent walk: a pair of consecutive row tiles and a token
// tile.  Consecutive units share the row-tile pair, so the clusters working at
// one time read each weight block from HBM about once; the tokens stay in L2.
struct Unit {
    int rt;       // this CTA's row tile (may be past the last: then it has no rows)
    int tt;       // token tile
    bool rows;    // this CTA has weight rows in this unit
    bool eight;
    int lt;       // index among the tiles of its kind
};

__device__ __forceinline__ Unit unit_of(const Tc3Args& a, int u, uint32_t rank) {
    Unit r;
    r.rt = 2 * (u / a.n_tt) + int(rank);
    r.tt = u % a.n_tt;
    r.rows = r.rt < a.g.t8 + a.g.t4;
    r.eight = r.rt < a.g.t8;
    r.lt = r.eight ? r.rt : r.rt - a.g.t8;
    return r;
}

// Drain every stage a producer issued (bounded) so that none of its copies
// targets this CTA's shared memory after it exits.
__device__ __forceinline__ void drain_stages(uint64_t* full, int issued, uint64_t timeout_ns) {
    for (int j = max(0, issued - kStages); j < issued; ++j) {
        int dummy = 0;
        mbar_wait_bounded(&full[j % kStages], (j / kStages) & 1, &dummy, nullptr, timeout_ns);
    }
}

template <bool DEBUG, bool AG>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
gemm_tc3_kernel(const __grid_constant__ CUtensorMap amap, const __grid_constant__ Tc3Args a) {
    extern __shared__ uint8_t smem_raw[];
    // the same offset in both CTAs: barriers and the TMEM address are addressed by
    // offset across the pair
    Smem& S = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const Geom& g = a.g;
    const int gpk = kKBlock / g.group;            // groups per k-block (1 or 2)
    const int ksteps = g.group / 32;              // MMA k-steps per group
    const int nkb = g.kblocks;
    const int cid = int(blockIdx.x >> 1), ncl = int(gridDim.x >> 1);
    volatile int* abort = &S.abort;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&S.full_w[s], 1);
            mbar_init(&S.full_t[s], 1);
            mbar_init(&S.ready[s], 2 * kWidenWarps);
            mbar_init(&S.empty[s], kKBlock / g.group);
        }
        for (int b = 0; b < kSlots; ++b) {
            mbar_init(&S.acc_full[b], 1);
            mbar_init(&S.acc_empty[b], 2 * kEpiWarps);
        }
        for (int b = 0; b < kSlots; ++b) mbar_init(&S.mma_done[b], 1);
        S.abort = 0;
        fence_mbar_init();
        prefetch_tensormap(&amap);
    }
    if (warp == 2) {
        tmem_alloc_pair(&S.tmem_base, kTmemCols);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    cluster_sync();                               // both CTAs' barriers initialised, TMEM allocated
    tc_fence_after();
    const uint32_t tmem = S.tmem_base;
    // the even CTA's barriers that the warps of both CTAs arrive on
    const uint32_t ready_c = mapa_shared(&S.ready[0], 0);
    const uint32_t acc_empty_c = mapa_shared(&S.acc_empty[0], 0);

    if (warp < 8) {
    // every warpgroup runs one setmaxnreg; the code of each role follows the one
    // that sets its budget
    regs_dec<kLowRegs>();
    if (warp == 0) {
        // ------------------------------------------------------------ weight copies
        int it = 0;
        if (!a.stall_test) {
            for (int u = cid; u < a.n_units; u += ncl) {
                const Unit un = unit_of(a, u, rank);
                for (int kb = 0; kb < nkb; ++kb, ++it) {
                    const int s = it % kStages;
                    const uint32_t ph = (it / kStages) & 1;
                    bool ok = true;
                    if (lane == 0) ok = mbar_wait_bounded(&S.empty[s], ph ^ 1, abort, a.status, a.timeout_ns);
                    if (!__shfl_sync(0xffffffffu, ok, 0)) goto wload_done;
                    const uint32_t cbytes = un.rows ? uint32_t(un.eight ? kABytes : kRawBytes) : 0u;
                    const uint32_t zbytes = un.rows && !un.eight ? uint32_t(gpk * BM) : 0u;
                    if (lane == 0) mbar_arrive_expect_tx(&S.full_w[s], cbytes + zbytes);
                    __syncwarp();
                    const size_t blk = size_t(un.lt) * nkb + kb;
                    if (cbytes != 0 && lane == (it & 15)) {
                        if (un.eight)
                            bulk_g2s(S.A[s], reinterpret_cast<const uint8_t*>(g.codes8) + blk * kABytes, cbytes,
                                     &S.full_w[s]);
                        else
                            bulk_g2s(S.R[s], g.codes4 + blk * kRawBytes, cbytes, &S.full_w[s]);
                    }
                    // the zero points of the stage's groups: [group][128 rows], contiguous
                    if (zbytes != 0 && lane == 16 + (it & 15))
                        bulk_g2s(S.Z[s], g.zeros4 + (size_t(un.lt) * g.G + size_t(kb) * gpk) * kTileRows, zbytes,
                                 &S.full_w[s]);
                }
            }
        }
    wload_done:
        if (lane == 0) drain_stages(S.full_w, it, a.timeout_ns);
    } else if (warp == 1) {
        // ------------------------------------------------------------ token copies
        int it = 0;
        if (!a.stall_test) {
            for (int u = cid; u < a.n_units; u += ncl) {
                const Unit un = unit_of(a, u, rank);
                for (int kb = 0; kb < nkb; ++kb, ++it) {
                    const int s = it % kStages;
                    const uint32_t ph = (it / kStages) & 1;
                    bool ok = true;
                    if (lane == 0) ok = mbar_wait_bounded(&S.empty[s], ph ^ 1, abort, a.status, a.timeout_ns);
                    if (!__shfl_sync(0xffffffffu, ok, 0)) goto tload_done;
                    // tokens past M read as zeros; the box is always counted whole
                    if (lane == 0) mbar_arrive_expect_tx(&S.full_t[s], uint32_t(kBBytes));
                    __syncwarp();
                    if (lane == (it & 31))
                        tma_load_3d(S.B[s], &amap, 0, un.tt * BN + int(rank) * BNH, kb, &S.full_t[s]);
                }
            }
        }
    tload_done:
        if (lane == 0) drain_stages(S.full_t, it, a.timeout_ns);
    } else if (warp == 2 || warp == 3) {
        // ------------------------------------------------------------ pair MMAs (even CTA)
        // issuer `mine` takes the groups of accumulator `mine`: every second group
        const uint32_t mine = uint32_t(warp - 2);
        if (rank == 0 && lane == 0) {
            const uint32_t idesc = idesc_i8(2 * BM, BN);
            int it = 0;
            uint32_t gc = 0;
            for (int u = cid; u < a.n_units; u += ncl) {
                for (int kb = 0; kb < nkb; ++kb, ++it) {
                    const int s = it % kStages;
                    const uint32_t ph = (it / kStages) & 1;
                    // does this stage hold a group of mine?  (gpk groups from gc on)
                    if (gpk == 1 && (gc & 1u) != mine) {
                        ++gc;
                        continue;
                    }
                    if (!mbar_wait_bounded(&S.ready[s], ph, abort, a.status, a.timeout_ns)) goto mma_out;
                    tc_fence_after();
                    const uint32_t a0 = smem_u32(S.A[s]), b0 = smem_u32(S.B[s]);
                    for (int j = 0; j < gpk; ++j, ++gc) {
                        const uint32_t b = gc % kSlots;
                        if (b != mine) continue;
                        // use gc / kSlots of accumulator b: phase 0 is the epilogue's first release
                        if (!mbar_wait_bounded(&S.acc_empty[b], (gc / kSlots) & 1, abort, a.status, a.timeout_ns))
                            goto mma_out;
                        tc_fence_after();
                        // the group's first k-step overwrites the accumulator
                        for (int kk = 0; kk < ksteps; ++kk) {
                            const uint32_t off = uint32_t(j * g.group + kk * 32);
                            mma_i8_pair(tmem + b * kSlotCols, sw128_kmajor_desc(a0 + off),
                                        sw128_kmajor_desc(b0 + off), idesc, kk > 0 ? 1u : 0u);
                        }
                        mma_commit_pair(&S.acc_full[b]);
                        mma_commit_pair(&S.empty[s]);    // once this group's MMAs are done, its part of
                                                         // the stage may be refilled
                    }
                }
            }
        mma_out:
            mma_commit_pair(&S.mma_done[mine], 0x1);     // all MMAs issued so far complete before teardown
            int dummy = 0;
            mbar_wait_bounded(&S.mma_done[mine], 0, &dummy, nullptr, a.timeout_ns);
        }
    } else {
        // ------------------------------------------------------------ widening (4-bit rows)
        const int wt = threadIdx.x - 4 * 32;
        int it = 0;
        for (int u = cid; u < a.n_units; u += ncl) {
            const Unit un = unit_of(a, u, rank);
            const bool widen = un.rows && !un.eight;
            for (int kb = 0; kb < nkb; ++kb, ++it) {
                const int s = it % kStages;
                const uint32_t ph = (it / kStages) & 1;
                // the weights to widen, then the tokens: the pair MMA needs both CTAs' stages
                bool ok = mbar_wait_bounded(&S.full_w[s], ph, abort, a.status, a.timeout_ns);
                ok = ok && mbar_wait_bounded(&S.full_t[s], ph, abort, a.status, a.timeout_ns);
                if (!__all_sync(0xffffffffu, ok)) goto widen_done;
                if (widen) {
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
                if (lane == 0) mbar_arrive_cluster(ready_c + 8u * uint32_t(s));
            }
        }
    widen_done:;
    }
    } else {
        // ------------------------------------------------------------ epilogue
        regs_inc<kEpiRegs>();
        const int e = warp - 8;                      // 0 .. kEpiWarps-1
        const int q = warp & 3;                      // TMEM lane quarter of this warp
        const int row = q * 32 + lane;               // weight row within this CTA's tile
        const int cb = (e >> 2) * kEpiCols;          // first of this warp's columns (tokens) in the tile
        const uint32_t lane_addr = tmem + (uint32_t(q * 32) << 16) + uint32_t(cb);
        // both accumulators start free
        if (lane == 0)
            for (int b = 0; b < kSlots; ++b) mbar_arrive_cluster(acc_empty_c + 8u * uint32_t(b));
        uint32_t gc = 0;
        for (int u = cid; u < a.n_units; u += ncl) {
            const Unit un = unit_of(a, u, rank);
            const __half* sc = (un.eight ? g.scales8 : g.scales4) + size_t(un.lt) * g.G * kTileRows + row;
            const int orig = un.rows ? g.rowmap[un.rt * kTileRows + row] : -1;
            const int m0 = un.tt * BN + cb;          // this warp's first token
            float2 acc[kEpiCols / 2];
#pragma unroll
            for (int c = 0; c < kEpiCols / 2; ++c) acc[c] = make_float2(0.0f, 0.0f);
            // group scales in a ring of kScaleRing registers, each loaded kScaleRing
            // groups before its use (a tile without rows multiplies by zero)
            __half swr[kScaleRing];
#pragma unroll
            for (int j = 0; j < kScaleRing; ++j)
                swr[j] = un.rows && j < g.G ? sc[size_t(j) * kTileRows] : __float2half_rn(0.0f);
            for (int gi0 = 0; gi0 < g.G; gi0 += kScaleRing) {
#pragma unroll
                for (int j = 0; j < kScaleRing; ++j) {
                    const int gi = gi0 + j;
                    if (gi >= g.G) break;
                    const float sw = __half2float(swr[j]);
                    if (un.rows && gi + kScaleRing < g.G) swr[j] = sc[size_t(gi + kScaleRing) * kTileRows];
                    const uint32_t b = gc % kSlots;
                    // every lane waits; the warp leaves together if any lane gave up (the
                    // TMEM accesses below are warp-collective)
                    const bool ok = mbar_wait_bounded(&S.acc_full[b], (gc / kSlots) & 1, abort, a.status,
                                                      a.timeout_ns);
                    if (!__all_sync(0xffffffffu, ok)) goto epi_done;
                    tc_fence_after();
                    __half (*sat)[kEpiCols] = S.sat[e];
                    if (AG && gi % kSatGroups == 0) {
                        // group-wise activations: this warp's token scales for the next groups
                        __syncwarp();
                        for (int i = lane; i < kSatGroups * kEpiCols; i += 32) {
                            const int w = i / kEpiCols, t = i % kEpiCols, m = m0 + t;
                            sat[w][t] = gi + w < g.G && m < a.M ? a.s_a[int64_t(m) * g.G + gi + w]
                                                                : __float2half_rn(0.0f);
                        }
                        __syncwarp();
                    }
                    const uint32_t col0 = lane_addr + b * kSlotCols;
                    // kPiece columns at a time: the int32 partials P
                    auto consume = [&](const uint32_t (&v)[kPiece], int piece) {
#pragma unroll
                        for (int c = 0; c < kPiece / 2; ++c) {
                            const float2 f = make_float2(__int2float_rn(int32_t(v[2 * c])),
                                                         __int2float_rn(int32_t(v[2 * c + 1])));
                            const int k = piece * (kPiece / 2) + c;
                            if constexpr (AG) {
                                const __half2 sh = *reinterpret_cast<const __half2*>(&sat[gi % kSatGroups][2 * k]);
                                const float2 sa2 = __half22float2(sh);
                                acc[k] = fma2(f, make_float2(__fmul_rn(sw, sa2.x), __fmul_rn(sw, sa2.y)), acc[k]);
                            } else {
                                acc[k] = fma2(f, make_float2(sw, sw), acc[k]);
                            }
                        }
                        if (DEBUG && orig >= 0) {
#pragma unroll
                            for (int c = 0; c < kPiece; ++c) {
                                const int m = m0 + piece * kPiece + c;
                                if (m < a.M) a.debug[(size_t(m) * g.N + orig) * g.G + gi] = int32_t(v[c]);
                            }
                        }
                    };
                    // two buffers: the load of piece p + 1 is in flight while piece p is
                    // multiplied; after the last load the accumulator is released, before
                    // the arithmetic on the last piece
                    constexpr int kPieces = kEpiCols / kPiece;
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
                            tc_fence_before();
                            __syncwarp();
                            if (lane == 0) mbar_arrive_cluster(acc_empty_c + 8u * b);
                        }
                        consume(cur, p);
                        if (p + 1 < kPieces) tmem_wait_ld();
                    }
                    ++gc;
                }
            }
            if (orig >= 0) {
                // one running pointer down the column: a single address stays live
                __half* yp = a.Y + int64_t(m0) * a.ldy + orig;
                const __half* sp = a.s_a + m0;
                const int mt = min(kEpiCols, a.M - m0);
#pragma unroll
                for (int c = 0; c < kEpiCols; ++c) {
                    if (c < mt) {
                        const float v = (c & 1) ? acc[c >> 1].y : acc[c >> 1].x;
                        *yp = __float2half_rn(AG ? v : __fmul_rn(v, __half2float(sp[c])));
                        yp += a.ldy;
                    }
                }
            }
        }
    epi_done:;
    }

    __syncwarp();            // single-thread roles: reconverge before the cluster barrier
    tc_fence_before();
    cluster_sync();          // no MMA, copy or arrival of either CTA touches the other any more
    if (warp == 2) {
        tc_fence_after();
        tmem_dealloc_pair(tmem, kTmemCols);
    }
}

}  // namespace

size_t tc3_smem_bytes() { return sizeof(Smem) + 1024; }

int tc3_units(const mx_layout& L, int M) { return ((L.t8 + L.t4 + 1) / 2) * ((M + BN - 1) / BN); }

// Served by the pair kernel with 256-token tiles: any M >= 1 (token rows past M
// are zero-filled by the copies and never stored).
cudaError_t launch_gemm_tc3(const mx_layout& L, const void* blob, const int8_t* Aq, const uint16_t* s_a, int M,
                            uint16_t* Y, int64_t ldy, int ag, int32_t* debug_partials, int32_t* status,
                            uint64_t timeout_ns, int stall_test, cudaStream_t s) {
    if (M == 0) return cudaSuccess;
    cudaError_t e;
    EncodeTiledFn enc = encode_fn(&e);
    if (e != cudaSuccess) return e;
    // activations as a 3-D tensor [k-block][token][128 bytes]: one box brings one
    // k-block of one CTA's 128 tokens as swizzled 128-byte rows
    CUtensorMap map;
    const cuuint64_t dims[3] = {cuuint64_t(kKBlock), cuuint64_t(M), cuuint64_t(L.kblocks)};
    const cuuint64_t strides[2] = {cuuint64_t(L.K), cuuint64_t(kKBlock)};
    const cuuint32_t box[3] = {cuuint32_t(kKBlock), cuuint32_t(BNH), 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = enc(&map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<int8_t*>(Aq), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;

    int dev = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    static int sms[64] = {};
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (sms[dev] == 0) {
        for (auto k : {gemm_tc3_kernel<false, false>, gemm_tc3_kernel<true, false>, gemm_tc3_kernel<false, true>,
                       gemm_tc3_kernel<true, true>}) {
            if ((e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, int(tc3_smem_bytes()))) !=
                cudaSuccess)
                return e;
            // the register split must match the launch allocation
            cudaFuncAttributes fa;
            if ((e = cudaFuncGetAttributes(&fa, k)) != cudaSuccess) return e;
            if (fa.numRegs != int(kLaunchRegs)) return cudaErrorInvalidConfiguration;
        }
        int n = 0;
        if ((e = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
        sms[dev] = n;
    }
    Tc3Args a{};
    a.g = make_geom(L, blob);
    a.s_a = reinterpret_cast<const __half*>(s_a);
    a.Y = reinterpret_cast<__half*>(Y);
    a.ldy = ldy;
    a.M = M;
    a.n_tt = (M + BN - 1) / BN;
    a.n_units = tc3_units(L, M);
    a.debug = debug_partials;
    a.status = status;
    a.timeout_ns = timeout_ns;
    a.stall_test = stall_test;
    const int pairs = std::min(a.n_units, sms[dev] / 2);
    auto k = debug_partials ? (ag ? gemm_tc3_kernel<true, true> : gemm_tc3_kernel<true, false>)
                            : (ag ? gemm_tc3_kernel<false, true> : gemm_tc3_kernel<false, false>);
    k<<<2 * pairs, kThreads, tc3_smem_bytes(), s>>>(map, a);
    return cudaGetLastError();
}

}  // namespace mx
