// gemm_tc2.cu -- tensor-core mixed-precision GEMM on CTA pairs (sm_100a, prefill M).
//
// The arithmetic is that of the one-CTA kernel (MixLLM section 3.3, two-step
// dequantization): per quantization group an exact int32 product P of the 8-bit
// activations with the (widened) weight codes on the tensor cores, then
// acc += float(P) * s_w[row, group] in fp32, and Y = fp16(acc * s_a[token])
// scattered to the original output columns.
//
// What changes is the tile.  Two CTAs of a cluster share one tcgen05.mma
// (cta_group::2): 256 weight rows (128 in each CTA) times 128 tokens (64 of them
// staged in each CTA).  Per multiply-accumulate this moves fewer operand bytes
// from L2 into shared memory than a 128 x 128 tile on one CTA, and the tensor
// core of each SM reads only its own half of the tokens.  Each CTA's TMEM holds
// four accumulators of 128 rows x 128 tokens, one group's int32 sum each.  They
// are preloaded with the integer of the fast int-to-float bias (section 3.3,
// Figure 3), so the products land in TMEM already offset and the epilogue reads
// fp32 bit patterns.  An epilogue warp releases a finished accumulator as soon as
// it has copied its 64 columns out (16 at a time) and stored the bias back, and
// does the arithmetic on the last 16 after the release, so four accumulators
// cover the round trip between the MMA thread and the epilogue.
//
// Roles (12 warps per CTA: three per SM sub-partition, whose register file then
// gives each thread up to 168 registers):
//   warp 0       copies: per stage two k-blocks of this CTA's weight rows (uint4
//                codes and their zero points, or pre-swizzled int8 codes) and of
//                its 64 tokens, three copies; the issuing lanes rotate with the
//                stage, so consecutive copies overlap
//   warp 1       TMEM allocation (both CTAs); in the even CTA one thread issues
//                the pair MMAs and commits to barriers in both CTAs
//   warps 2-3    widening of 4-bit rows in place (uint4 -> int8 q - z), then an
//                arrival on the even CTA's "stage ready" barrier
//   warps 4-11   epilogue: warp w reads TMEM lane quarter w % 4, tokens
//                64 * ((w - 4) / 4) .. +63 of the tile
// The odd CTA's widening and epilogue warps arrive on the even CTA's barriers
// through their cluster addresses.  Every wait is bounded; on expiry the kernel
// records MX_ERR_TIMEOUT and all roles leave their loops.
#include <algorithm>

#include "mx_internal.cuh"
#include "sm100.cuh"

namespace mx {
namespace {

using namespace sm100;

constexpr int BM = 128;                         // weight rows per CTA (the pair: 256)
constexpr int BN = 128;                         // tokens per pair tile
constexpr int BNH = BN / 2;                     // tokens staged per CTA
constexpr int KPS = 2;                          // k-blocks per pipeline stage
constexpr int kStages = 4;
constexpr int kABytes = BM * kKBlock;           // int8 weight operand of one k-block
constexpr int kBBytes = BNH * kKBlock;          // this CTA's activations of one k-block
constexpr int kRawBytes = BM * kKBlock / 2;     // uint4 codes of one k-block
// the uint4 codes of a stage land at the top of its weight-operand buffer and are
// widened in place, k-block after k-block, into the int8 operand below them
constexpr int kRawBase = KPS * (kABytes - kRawBytes);
constexpr int kZBytes = KPS * 2 * BM;           // zero points of up to two groups per k-block
constexpr int kWidenWarps = 2;
constexpr int kWidenThreads = kWidenWarps * 32;
constexpr int kEpiWarps = 8;
constexpr int kEpiTokens = 64;                  // tokens per epilogue warp
constexpr int kThreads = (2 + kWidenWarps + kEpiWarps) * 32;
constexpr int kWidenChunks = BM * 4 / kWidenThreads;   // 16-byte code chunks per thread and k-block
constexpr int kAccBufs = 4;                     // int32 group accumulators in TMEM
constexpr int kAccCols = BN;                    // TMEM columns of one accumulator
constexpr uint32_t kTmemCols = 512;
constexpr int kWidenBarrier = 1;
constexpr int kScaleRing = 4;
constexpr int kSatGroups = 8;
static_assert(kEpiWarps * kEpiTokens == 4 * BN, "two epilogue warps per TMEM lane quarter");
static_assert(kAccBufs * kAccCols <= int(kTmemCols), "accumulators fit in TMEM");

struct __align__(1024) Smem {
    uint8_t A[kStages][KPS * kABytes];
    uint8_t B[kStages][KPS * kBBytes];
    uint8_t Z[kStages][kZBytes];  // zero points of the stage's groups (4-bit rows), [group][row]
    uint64_t full[kStages];       // this CTA's copies of the stage landed
    uint64_t ready[kStages];      // (even CTA) both CTAs' operands of the stage are in place
    uint64_t empty[kStages];      // (both) the pair MMAs reading the stage completed
    uint64_t acc_full[kAccBufs];  // (both) a group accumulator is complete
    uint64_t acc_empty[kAccBufs]; // (even CTA) both CTAs drained and re-armed it
    uint64_t mma_done;
    __align__(16) __half sat[kEpiWarps][kSatGroups][kEpiTokens];
    uint32_t tmem_base;
    int abort;
};

struct Tc2Args {
    Geom g;
    const __half* s_a;   // [M], or [M][G] with group-wise activation scales
    __half* Y;
    int64_t ldy;
    int M;
    int n_tt;            // token tiles of BN
    int n_units;         // pairs of row tiles x K splits x token tiles
    int S;               // K splits (1: each unit covers the whole K)
    int ss_per;          // stages per split
    float* part;         // S > 1: fp32 partial sums [S][M][N] (original column order)
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

// Unit u of the persistent walk: a pair of consecutive row tiles, a range of K
// (a split) and a token tile.  Consecutive units share the row-tile pair and the
// split, so the pairs working at one time read each weight block from HBM about once.
struct Unit {
    int rt;       // this CTA's row tile (may be past the last: then it has no rows)
    int tt;       // token tile
    int ks;       // K split
    int sp0, sp1; // its stages [sp0, sp1)
    bool rows;    // this CTA has weight rows in this unit
    bool eight;
    int lt;       // index among the tiles of its kind
};

__device__ __forceinline__ Unit unit_of(const Tc2Args& a, int u, uint32_t rank, int n_ss) {
    Unit r;
    const int pk = u / a.n_tt;                    // (pair, split)
    r.rt = 2 * (pk / a.S) + int(rank);
    r.ks = pk % a.S;
    r.tt = u % a.n_tt;
    r.sp0 = r.ks * a.ss_per;
    r.sp1 = min(n_ss, r.sp0 + a.ss_per);
    r.rows = r.rt < a.g.t8 + a.g.t4;
    r.eight = r.rt < a.g.t8;
    r.lt = r.eight ? r.rt : r.rt - a.g.t8;
    return r;
}


// Drain every issued stage (bounded) so that no copy targets this CTA's shared
// memory after it exits.
__device__ __forceinline__ void drain_stages(Smem& S, int issued, uint64_t timeout_ns) {
    for (int j = max(0, issued - kStages); j < issued; ++j) {
        int dummy = 0;
        mbar_wait_bounded(&S.full[j % kStages], (j / kStages) & 1, &dummy, nullptr, timeout_ns);
    }
}

template <bool DEBUG, bool AG>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
gemm_tc2_kernel(const __grid_constant__ CUtensorMap amap, const __grid_constant__ Tc2Args a) {
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
            mbar_init(&S.full[s], 1);
            mbar_init(&S.ready[s], 2 * kWidenWarps);
            mbar_init(&S.empty[s], 1);
        }
        for (int b = 0; b < kAccBufs; ++b) {
            mbar_init(&S.acc_full[b], 1);
            mbar_init(&S.acc_empty[b], 2 * kEpiWarps);
        }
        mbar_init(&S.mma_done, 1);
        S.abort = 0;
        fence_mbar_init();
        prefetch_tensormap(&amap);
    }
    if (warp == 1) {
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

    const int n_ss = (nkb + KPS - 1) / KPS;       // stages per unit
    if (warp == 0) {
        // ------------------------------------------------------------ copies
        // Three copies per stage of KPS k-blocks (issuing a copy costs more than its
        // bytes here, so they are few and large); the issuing lanes rotate with the
        // stage so that consecutive copies overlap.
        int it = 0;
        if (!a.stall_test) {
            for (int u = cid; u < a.n_units; u += ncl) {
                const Unit un = unit_of(a, u, rank, n_ss);
                for (int sp = un.sp0; sp < un.sp1; ++sp, ++it) {
                    const int s = it % kStages;
                    const uint32_t ph = (it / kStages) & 1;
                    bool ok = true;
                    if (lane == 0) ok = mbar_wait_bounded(&S.empty[s], ph ^ 1, abort, a.status, a.timeout_ns);
                    if (!__shfl_sync(0xffffffffu, ok, 0)) goto load_done;
                    const int kb0 = sp * KPS, nk = min(KPS, nkb - kb0);
                    const uint32_t abytes = un.rows ? uint32_t(nk * (un.eight ? kABytes : kRawBytes)) : 0u;
                    const uint32_t zbytes = un.rows && !un.eight ? uint32_t(nk * gpk * BM) : 0u;
                    // the token box always spans KPS k-blocks (past the last it reads zeros)
                    if (lane == 0) mbar_arrive_expect_tx(&S.full[s], abytes + zbytes + uint32_t(KPS * kBBytes));
                    __syncwarp();
                    if (abytes != 0 && lane == (it & 7)) {
                        const size_t blk = size_t(un.lt) * nkb + kb0;
                        if (un.eight)
                            bulk_g2s(S.A[s], reinterpret_cast<const uint8_t*>(g.codes8) + blk * kABytes, abytes, &S.full[s]);
                        else
                            bulk_g2s(S.A[s] + kRawBase, g.codes4 + blk * kRawBytes, abytes, &S.full[s]);
                    }
                    // the zero points of the stage's groups: [group][128 rows], contiguous
                    if (zbytes != 0 && lane == 8 + (it & 7))
                        bulk_g2s(S.Z[s], g.zeros4 + (size_t(un.lt) * g.G + size_t(kb0) * gpk) * kTileRows, zbytes,
                                 &S.full[s]);
                    // this CTA's half of the token tile for the stage's k-blocks (rows past
                    // M read as zeros)
                    if (lane == 16 + (it & 15))
                        tma_load_3d(S.B[s], &amap, 0, un.tt * BN + int(rank) * BNH, kb0, &S.full[s]);
                }
            }
        }
    load_done:
        if (lane == 0) drain_stages(S, it, a.timeout_ns);
    } else if (warp == 1) {
        // ------------------------------------------------------------ pair MMAs (even CTA)
        if (rank == 0 && lane == 0) {
            const uint32_t idesc = idesc_i8(2 * BM, BN);
            int it = 0;
            uint32_t gc = 0;
            for (int u = cid; u < a.n_units; u += ncl) {
                const Unit un = unit_of(a, u, rank, n_ss);
                for (int sp = un.sp0; sp < un.sp1; ++sp, ++it) {
                    const int s = it % kStages;
                    const uint32_t ph = (it / kStages) & 1;
                    if (!mbar_wait_bounded(&S.ready[s], ph, abort, a.status, a.timeout_ns)) goto mma_out;
                    tc_fence_after();
                    const int nk = min(KPS, nkb - sp * KPS);
                    for (int kbi = 0; kbi < nk; ++kbi) {
                        const uint32_t a0 = smem_u32(S.A[s] + kbi * kABytes), b0 = smem_u32(S.B[s] + kbi * kBBytes);
                        for (int j = 0; j < gpk; ++j, ++gc) {
                            const uint32_t b = gc % kAccBufs;
                            // use gc / kAccBufs of accumulator b: phase 0 is the epilogue's first bias preload
                            if (!mbar_wait_bounded(&S.acc_empty[b], (gc / kAccBufs) & 1, abort, a.status, a.timeout_ns))
                                goto mma_out;
                            tc_fence_after();
                            // the accumulator holds the bias: every k-step adds
                            for (int kk = 0; kk < ksteps; ++kk) {
                                const uint32_t off = uint32_t(j * g.group + kk * 32);
                                mma_i8_pair(tmem + b * kAccCols, sw128_kmajor_desc(a0 + off), sw128_kmajor_desc(b0 + off),
                                            idesc, 1u);
                            }
                            mma_commit_pair(&S.acc_full[b]);
                        }
                    }
                    mma_commit_pair(&S.empty[s]);        // both CTAs may refill the stage
                }
            }
        mma_out:
            mma_commit_pair(&S.mma_done, 0x1);           // all MMAs issued so far complete before teardown
            int dummy = 0;
            mbar_wait_bounded(&S.mma_done, 0, &dummy, nullptr, a.timeout_ns);
        }
    } else if (warp < 2 + kWidenWarps) {
        // ------------------------------------------------------------ widening (4-bit rows)
        const int wt = threadIdx.x - 64;
        int it = 0;
        for (int u = cid; u < a.n_units; u += ncl) {
            const Unit un = unit_of(a, u, rank, n_ss);
            const bool widen = un.rows && !un.eight;
            for (int sp = un.sp0; sp < un.sp1; ++sp, ++it) {
                const int s = it % kStages;
                const uint32_t ph = (it / kStages) & 1;
                const bool ok = mbar_wait_bounded(&S.full[s], ph, abort, a.status, a.timeout_ns);
                __syncwarp();   // the named barrier is warp-collective
                // one decision for all widening threads: the in-place conversion needs
                // every one of them at the named barrier
                if (!named_bar_and(kWidenBarrier, kWidenThreads, ok)) goto widen_done;
                if (widen) {
                    const int nk = min(KPS, nkb - sp * KPS);
                    const uint8_t* raw = S.A[s] + kRawBase;
                    for (int kbi = 0; kbi < nk; ++kbi) {
                        uint4 w[kWidenChunks];
#pragma unroll
                        for (int j = 0; j < kWidenChunks; ++j)
                            w[j] = *reinterpret_cast<const uint4*>(raw + kbi * kRawBytes + (wt + kWidenThreads * j) * 16);
                        // once the int8 block reaches the codes, every thread reads before any writes
                        if ((kbi + 1) * kABytes > kRawBase) named_bar_and(kWidenBarrier, kWidenThreads, true);
                        uint8_t* out = S.A[s] + kbi * kABytes;
                        const uint8_t* zs = S.Z[s] + kbi * gpk * BM;
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
                    }
                    fence_proxy_async_smem();
                }
                __syncwarp();
                if (lane == 0) mbar_arrive_cluster(ready_c + 8u * uint32_t(s));
            }
        }
    widen_done:;
    } else {
        // ------------------------------------------------------------ epilogue
        const int e = warp - 2 - kWidenWarps;        // 0 .. kEpiWarps-1
        const int q = warp & 3;                      // TMEM lane quarter of this warp
        const int row = q * 32 + lane;               // weight row within this CTA's tile
        const int cb = (e >> 2) * kEpiTokens;        // first of this warp's tokens in the tile
        const uint32_t lane_addr = tmem + (uint32_t(q * 32) << 16) + uint32_t(cb);
        const float2 nbias = make_float2(-kI2FBias, -kI2FBias);
        // preload every accumulator with the bias, then hand them to the MMA
#pragma unroll
        for (int b = 0; b < kAccBufs; ++b) {
            tmem_st_x32_splat(lane_addr + b * kAccCols, kI2FBiasBits);
            tmem_st_x32_splat(lane_addr + b * kAccCols + 32, kI2FBiasBits);
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0)
            for (int b = 0; b < kAccBufs; ++b) mbar_arrive_cluster(acc_empty_c + 8u * uint32_t(b));
        uint32_t gc = 0;
        for (int u = cid; u < a.n_units; u += ncl) {
            const Unit un = unit_of(a, u, rank, n_ss);
            // this unit's groups [g0, g1)
            const int g0 = un.sp0 * KPS * gpk, g1 = min(g.G, un.sp1 * KPS * gpk);
            const __half* sc = (un.eight ? g.scales8 : g.scales4) + (size_t(un.lt) * g.G + g0) * kTileRows + row;
            const int orig = un.rows ? g.rowmap[un.rt * kTileRows + row] : -1;
            const int m0 = un.tt * BN + cb;          // this warp's first token
            float2 acc[kEpiTokens / 2];
#pragma unroll
            for (int c = 0; c < kEpiTokens / 2; ++c) acc[c] = make_float2(0.0f, 0.0f);
            // group scales in a ring of kScaleRing registers, each loaded kScaleRing
            // groups before its use; the group loop is unrolled by kScaleRing so every
            // ring slot is a fixed register and no instruction waits on a young load
            // (a tile without rows multiplies by zero)
            // (the ring holds the raw fp16 values: converting at the load would wait for it)
            __half swr[kScaleRing];
#pragma unroll
            for (int j = 0; j < kScaleRing; ++j)
                swr[j] = un.rows && g0 + j < g1 ? sc[size_t(j) * kTileRows] : __float2half_rn(0.0f);
            for (int gi0 = g0; gi0 < g1; gi0 += kScaleRing) {
#pragma unroll
                for (int j = 0; j < kScaleRing; ++j) {
                    const int gi = gi0 + j;
                    if (gi >= g1) break;
                    const float sw = __half2float(swr[j]);
                    if (un.rows && gi + kScaleRing < g1) swr[j] = sc[size_t(gi - g0 + kScaleRing) * kTileRows];
                    const uint32_t b = gc % kAccBufs;
                    // every lane waits; the warp leaves together if any lane gave up (the
                    // TMEM accesses below are warp-collective)
                    const bool ok = mbar_wait_bounded(&S.acc_full[b], (gc / kAccBufs) & 1, abort, a.status,
                                                      a.timeout_ns);
                    if (!__all_sync(0xffffffffu, ok)) goto epi_done;
                    tc_fence_after();
                    __half (*sat)[kEpiTokens] = S.sat[e];
                    if (AG && (gi - g0) % kSatGroups == 0) {
                        // group-wise activations: this warp's token scales for the next groups
                        __syncwarp();
                        for (int i = lane; i < kSatGroups * kEpiTokens; i += 32) {
                            const int w = i / kEpiTokens, t = i % kEpiTokens, m = m0 + t;
                            sat[w][t] = gi + w < g.G && m < a.M ? a.s_a[int64_t(m) * g.G + gi + w]
                                                                : __float2half_rn(0.0f);
                        }
                        __syncwarp();
                    }
                    // 16 columns at a time (fp32 bit patterns bias + P); after the last copy
                    // the bias goes back and the accumulator is released, before the
                    // arithmetic on those columns
                    const uint32_t col0 = lane_addr + b * kAccCols;
                    auto consume = [&](const uint32_t (&v)[16], int quarter) {
#pragma unroll
                        for (int hh = 0; hh < 2; ++hh) {
                            const int h = 2 * quarter + hh;                 // 8-column chunk
                            if constexpr (AG) {
                                const uint4 sv = *reinterpret_cast<const uint4*>(&sat[(gi - g0) % kSatGroups][h * 8]);
                                const __half2* sh = reinterpret_cast<const __half2*>(&sv);
#pragma unroll
                                for (int c = 0; c < 4; ++c) {
                                    const float2 sa2 = __half22float2(sh[c]);
                                    const float2 f = add2(make_float2(__uint_as_float(v[hh * 8 + 2 * c]),
                                                                      __uint_as_float(v[hh * 8 + 2 * c + 1])),
                                                          nbias);
                                    acc[h * 4 + c] = fma2(f, make_float2(__fmul_rn(sw, sa2.x), __fmul_rn(sw, sa2.y)),
                                                          acc[h * 4 + c]);
                                }
                            } else {
                                const float2 s2 = make_float2(sw, sw);
#pragma unroll
                                for (int c = 0; c < 4; ++c) {
                                    const float2 f = add2(make_float2(__uint_as_float(v[hh * 8 + 2 * c]),
                                                                      __uint_as_float(v[hh * 8 + 2 * c + 1])),
                                                          nbias);
                                    acc[h * 4 + c] = fma2(f, s2, acc[h * 4 + c]);
                                }
                            }
                        }
                        if (DEBUG && orig >= 0) {
#pragma unroll
                            for (int c = 0; c < 16; ++c) {
                                const int m = m0 + quarter * 16 + c;
                                if (m < a.M) a.debug[(size_t(m) * g.N + orig) * g.G + gi] = int32_t(v[c] - kI2FBiasBits);
                            }
                        }
                    };
                    uint32_t v[16];
#pragma unroll
                    for (int qq = 0; qq < 3; ++qq) {
                        tmem_ld_x16(col0 + qq * 16, v);
                        tmem_wait_ld();
                        consume(v, qq);
                    }
                    tmem_ld_x16(col0 + 48, v);
                    tmem_wait_ld();
                    tmem_st_x32_splat(col0, kI2FBiasBits);
                    tmem_st_x32_splat(col0 + 32, kI2FBiasBits);
                    tmem_wait_st();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive_cluster(acc_empty_c + 8u * b);
                    ++gc;
                    consume(v, 3);
                }
            }
            if (orig >= 0) {
                // one split: Y; several: this split's fp32 sums, added in split order and
                // scaled by the reduction kernel
                float* part = a.S > 1 ? a.part + size_t(un.ks) * a.M * g.N : nullptr;
#pragma unroll
                for (int c = 0; c < kEpiTokens / 2; ++c) {
#pragma unroll
                    for (int x = 0; x < 2; ++x) {
                        const int m = m0 + 2 * c + x;
                        if (m < a.M) {
                            const float v = x ? acc[c].y : acc[c].x;
                            if (part) part[int64_t(m) * g.N + orig] = v;
                            else a.Y[int64_t(m) * a.ldy + orig] =
                                     __float2half_rn(AG ? v : __fmul_rn(v, __half2float(a.s_a[m])));
                        }
                    }
                }
            }
        }
    epi_done:;
    }

    __syncwarp();            // single-thread roles: reconverge before the cluster barrier
    tc_fence_before();
    cluster_sync();          // no MMA, copy or arrival of either CTA touches the other any more
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem, kTmemCols);
    }
}

// Y[m][n] = fp16(the splits' fp32 sums of (m, n), added in split order, x s_a[m]);
// group-wise activation scales were applied per group.  Elementwise over M x N.
__global__ void __launch_bounds__(256) split_reduce_kernel(const float* __restrict__ part, int S, int M, int N,
                                                           const __half* __restrict__ s_a, int ag, __half* Y,
                                                           int64_t ldy) {
    const int64_t total = int64_t(M) * N;
    // launched as a programmatic dependent: resident while the GEMM finishes, it reads
    // the sums only once that kernel completed; its own dependents may start at once
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;");
    for (int64_t i = int64_t(blockIdx.x) * 256 + threadIdx.x; i < total; i += int64_t(gridDim.x) * 256) {
        const int m = int(i / N), n = int(i % N);
        float v = part[i];
        for (int k = 1; k < S; ++k) v = __fadd_rn(v, part[int64_t(k) * total + i]);
        Y[int64_t(m) * ldy + n] = __float2half_rn(ag ? v : __fmul_rn(v, __half2float(s_a[m])));
    }
}

}  // namespace

size_t tc2_smem_bytes() { return sizeof(Smem) + 1024; }

int tc2_stages(const mx_layout& L) { return (L.kblocks + KPS - 1) / KPS; }

int tc2_auto_split(const mx_layout& L, int M, int clusters) {
    const int units1 = ((L.t8 + L.t4 + 1) / 2) * ((M + BN - 1) / BN);
    const int n_ss = tc2_stages(L);
    if (M <= 0 || clusters <= 0 || units1 >= clusters || n_ss < 2) return 1;
    // waves x stages per unit, smallest first; the split adds partial sums to write
    // and read back, so a tie keeps fewer splits
    int best = 1;
    long best_t = long(n_ss);
    for (int S = 2; S <= kTc2MaxSplit && S <= n_ss; ++S) {
        const int per = (n_ss + S - 1) / S;
        if ((n_ss + per - 1) / per != S) continue;            // no empty split
        const long t = (long(units1) * S + clusters - 1) / clusters * per;
        if (t < best_t) {
            best_t = t;
            best = S;
        }
    }
    return best;
}

size_t tc2_split_bytes(const mx_layout& L, int M, int S) {
    return S > 1 ? (size_t(S) * size_t(M) * size_t(L.N) * 4 + 255) & ~size_t(255) : 0;
}

// Served by the pair kernel: any M >= 1 (token tiles of 128; rows past M are
// zero-filled by the copies and never stored).
cudaError_t launch_gemm_tc2(const mx_layout& L, const void* blob, const int8_t* Aq, const uint16_t* s_a, int M,
                            uint16_t* Y, int64_t ldy, int ag, int S, float* part, int32_t* debug_partials,
                            int32_t* status, uint64_t timeout_ns, int stall_test, cudaStream_t s) {
    if (M == 0) return cudaSuccess;
    cudaError_t e;
    EncodeTiledFn enc = encode_fn(&e);
    if (e != cudaSuccess) return e;
    // activations as a 3-D tensor [k-block][token][128 bytes]: one box brings KPS
    // k-blocks of one CTA's 64 tokens as swizzled 128-byte-row blocks
    CUtensorMap map;
    const cuuint64_t dims[3] = {cuuint64_t(kKBlock), cuuint64_t(M), cuuint64_t(L.kblocks)};
    const cuuint64_t strides[2] = {cuuint64_t(L.K), cuuint64_t(kKBlock)};
    const cuuint32_t box[3] = {cuuint32_t(kKBlock), cuuint32_t(BNH), cuuint32_t(KPS)};
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
        for (auto k : {gemm_tc2_kernel<false, false>, gemm_tc2_kernel<true, false>, gemm_tc2_kernel<false, true>,
                       gemm_tc2_kernel<true, true>})
            if ((e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, int(tc2_smem_bytes()))) !=
                cudaSuccess)
                return e;
        int n = 0;
        if ((e = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
        sms[dev] = n;
    }
    Tc2Args a{};
    a.g = make_geom(L, blob);
    a.s_a = reinterpret_cast<const __half*>(s_a);
    a.Y = reinterpret_cast<__half*>(Y);
    a.ldy = ldy;
    a.M = M;
    a.n_tt = (M + BN - 1) / BN;
    // S splits of the stages (the last split may be shorter, none is empty)
    const int n_ss = tc2_stages(L);
    if (S < 1 || S > kTc2MaxSplit || (S > 1 && part == nullptr)) return cudaErrorInvalidValue;
    S = std::min(S, n_ss);
    a.ss_per = (n_ss + S - 1) / S;
    a.S = (n_ss + a.ss_per - 1) / a.ss_per;
    a.part = a.S > 1 ? part : nullptr;
    a.n_units = ((L.t8 + L.t4 + 1) / 2) * a.S * a.n_tt;
    a.debug = debug_partials;
    a.status = status;
    a.timeout_ns = timeout_ns;
    a.stall_test = stall_test;
    const int pairs = std::min(a.n_units, sms[dev] / 2);
    auto k = debug_partials ? (ag ? gemm_tc2_kernel<true, true> : gemm_tc2_kernel<true, false>)
                            : (ag ? gemm_tc2_kernel<false, true> : gemm_tc2_kernel<false, false>);
    k<<<2 * pairs, kThreads, tc2_smem_bytes(), s>>>(map, a);
    if ((e = cudaGetLastError()) != cudaSuccess || a.S == 1) return e;
    return launch_split_reduce(a.part, a.S, M, L.N, s_a, ag, Y, ldy, sms[dev], s);
}

cudaError_t launch_split_reduce(const float* part, int S, int M, int N, const uint16_t* s_a, int ag, uint16_t* Y,
                                int64_t ldy, int sms, cudaStream_t s) {
    const int64_t total = int64_t(M) * N;
    if (total == 0) return cudaSuccess;
    const int blocks = int(std::min<int64_t>((total + 255) / 256, int64_t(sms) * 8));
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(blocks);
    cfg.blockDim = dim3(256);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, split_reduce_kernel, part, S, M, N, reinterpret_cast<const __half*>(s_a), ag,
                              reinterpret_cast<__half*>(Y), ldy);
}

}  // namespace mx
