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
// At these sizes every step of a k-block's way is short, and what sets the pace is
// how many steps wait on one another.  Measured on this part: one thread issues a
// bulk copy only every few hundred ns whatever its size, a copy lands about a
// microsecond after issue, an MMA issue takes about 60 ns, and a barrier hand-over
// about 100 ns.  Hence:
//   R ring   the weights as stored, in 8 KB slots: a 4-bit k-block (uint4 codes)
//            takes one slot, its zero points beside it, an 8-bit k-block (int8
//            codes, stored pre-swizzled) two consecutive ones.  The copies move
//            chunks of four slots (one bulk copy per run of one unit's slots), and
//            a chunk is free once it is widened, so the ring is deep and the copies
//            run far ahead of the tensor core.
//   A ring   the int8 weight operand, written by the widening warps (a stage always
//            by the same group), freed by the MMAs (a commit per group).
//   B ring   the batch's tokens, one TMA box per chunk of four k-blocks (two from
//            NT = 64); a chunk is freed by one commit of each MMA issuer.
//   widening groups of two warps take every fourth k-block each (every second
//            from NT = 64), so that several k-blocks are widened at once.
// Chunks are aligned to the ring (they start at a multiple of the chunk size and may
// hold runs of two units), so they never wrap a ring.  A chunk's bytes are counted
// on the barrier of its first slot.  A barrier's parity names its phase only to a
// waiter at most one phase away, so every waiter of a barrier waits on each of its
// phases in order: every widening group waits on every weight chunk and releases it
// (the copy thread re-arms a chunk once all have), each MMA issuer waits on every
// token chunk (each holds k-blocks of both), and an operand stage always belongs to
// the same widening group.
//
// Roles (16 warps, one CTA per SM, persistent over the units):
//   warp 0       weight copies into the R ring.  The weights do not depend on the
//                kernel before this one in the stream (under programmatic dependent
//                launch), so they stream from the start
//   warps 1-2    TMEM allocation (warp 1); one thread of each waits for the tokens
//                and the operand and issues the MMAs and commits of every second
//                group (the accumulators of one parity).  At small N an MMA executes
//                faster than a thread can issue the next one (about 60 ns), so two
//                issuers keep the tensor core fed
//   warp 3       token copies into the B ring, after griddepcontrol.wait
//   warps 4-     widening: 4-bit codes to int8 q - z, 8-bit codes copied as they
//                are, from the R ring into the group's A stage, then an arrival on
//                the stage's "ready" barrier
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
constexpr int kSlotBytes = BM * kKBlock / 2;    // an R slot: the uint4 codes of one k-block
constexpr int kZBytes = 2 * BM;                 // zero points of up to two groups per slot
constexpr int kCR = 4;                          // R slots per chunk
constexpr int kGW = 2;                          // warps per widening group
constexpr int kWiden0 = 4;                      // first widening warp
constexpr int kScaleRing = 2;

constexpr int token_chunk(int NT) { return NT <= 32 ? 4 : 2; }   // k-blocks per token chunk

template <int NT>
struct Cfg {
    static constexpr int kWidenWarps = NT <= 32 ? 8 : 4;
    static constexpr int kGroups = kWidenWarps / kGW;          // widening groups
    static constexpr int kGT = kGW * 32;                       // threads per widening group
    static constexpr int kEpiWarp0 = kWiden0 + kWidenWarps;    // first epilogue warp (a multiple of 4)
    static constexpr int kEpiWarps = NT <= 32 ? 4 : 8;
    static constexpr int kEpiCols = NT * 4 / kEpiWarps;       // tokens per epilogue warp
    static constexpr int kPiece = kEpiCols >= 32 && NT <= 64 ? 32 : 16;   // TMEM columns per load
    static constexpr int kSlots = NT <= 64 ? 8 : 4;           // group accumulators in TMEM (even: one
                                                              // parity per issuer)
    static constexpr uint32_t kTmemCols = kSlots * NT <= 128 ? 128 : kSlots * NT <= 256 ? 256 : 512;
    static constexpr int kA = 4;                              // int8 operand stages (stage s: group s % kGroups)
    static constexpr int kCB = token_chunk(NT);
    static constexpr int kB = NT <= 32 ? 12 : NT == 64 ? 6 : 4;    // token stages
    static constexpr int kBChunks = kB / kCB;
    static constexpr int kR = NT <= 16 ? 16 : NT <= 64 ? 12 : 8;   // raw weight slots
    static constexpr int kBBytes = NT * kKBlock;
    static constexpr int kThreads = (kEpiWarp0 + kEpiWarps) * 32;
    static_assert(kThreads == 512, "16 warps: 128 registers per thread");
    static_assert(kSlots * NT <= int(kTmemCols), "accumulators fit in TMEM");
    static_assert(kEpiCols % kPiece == 0, "whole loads");
    static_assert(kB % kCB == 0 && kR % kCR == 0, "chunks never wrap a ring");
    static_assert(kBChunks >= 2 && kR >= 2 * kCR, "rings hold two chunks");
    static_assert(kSlotBytes % (16 * kGT) == 0, "whole 16-byte chunks per widening thread");
    static_assert(kA % kGroups == 0, "an operand stage always belongs to the same widening group");
};

template <int NT>
struct __align__(1024) Smem {
    uint8_t A[Cfg<NT>::kA][kABytes];             // int8 weight operand (swizzled 128-byte rows)
    uint8_t B[Cfg<NT>::kB][Cfg<NT>::kBBytes];    // the batch's tokens (swizzled by the copy)
    uint8_t R[Cfg<NT>::kR][kSlotBytes];          // weights as stored (4-bit: one slot, 8-bit: two)
    uint8_t Z[Cfg<NT>::kR][kZBytes];             // zero points: a run's lie contiguously from its first slot
    uint64_t r_full[Cfg<NT>::kR];                // a weight chunk landed (the barrier of its first slot)
    uint64_t r_rel[Cfg<NT>::kR / kCR];           // every widening warp is done with a weight chunk
    uint64_t b_full[Cfg<NT>::kB];                // a token chunk landed (the barrier of its first stage)
    uint64_t b_empty[Cfg<NT>::kBChunks];         // the MMAs reading a token chunk completed (one per issuer)
    uint64_t ready[Cfg<NT>::kA];                 // the operand is written
    uint64_t a_empty[Cfg<NT>::kA];               // the MMAs reading the operand completed (one commit per group)
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

__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

__device__ __forceinline__ void griddep_launch() { asm volatile("griddepcontrol.launch_dependents;"); }

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

// A run: consecutive slots (stages) of one unit inside one chunk, one copy.
struct WRun {
    const uint8_t* src;    // codes
    const uint8_t* zsrc;   // zero points (4-bit units)
    int slot;              // first slot (running count)
    uint32_t bytes, zbytes;
};
struct TRun {
    int kb;                // first k-block
    int n;                 // k-blocks
    int stage;             // first stage (running count)
};

template <int NT, bool DEBUG, bool AG>
__global__ void __launch_bounds__(Cfg<NT>::kThreads, 1)
gemm_tcd_kernel(const __grid_constant__ CUtensorMap amap1, const __grid_constant__ CUtensorMap amapC,
                const __grid_constant__ TcdArgs a) {
    using C = Cfg<NT>;
    extern __shared__ uint8_t smem_raw[];
    Smem<NT>& S = *reinterpret_cast<Smem<NT>*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const Geom& g = a.g;
    const int gpk = kKBlock / g.group;            // groups per k-block (1 or 2)
    const int ksteps = g.group / 32;              // MMA k-steps per group
    volatile int* abort = &S.abort;

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::kR; ++s) mbar_init(&S.r_full[s], 1);
        for (int c = 0; c < C::kR / kCR; ++c) mbar_init(&S.r_rel[c], C::kWidenWarps);
        for (int s = 0; s < C::kB; ++s) mbar_init(&S.b_full[s], 1);
        for (int c = 0; c < C::kBChunks; ++c) mbar_init(&S.b_empty[c], 2);
        for (int s = 0; s < C::kA; ++s) {
            mbar_init(&S.ready[s], kGW);
            mbar_init(&S.a_empty[s], gpk);
        }
        for (int b = 0; b < C::kSlots; ++b) {
            mbar_init(&S.acc_full[b], 1);
            mbar_init(&S.acc_empty[b], C::kEpiWarps);
        }
        mbar_init(&S.mma_done[0], 1);
        mbar_init(&S.mma_done[1], 1);
        S.abort = 0;
        fence_mbar_init();
        prefetch_tensormap(&amap1);
        prefetch_tensormap(&amapC);
    }
    if (warp == 1) {
        tmem_alloc(&S.tmem_base, C::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = S.tmem_base;
    // the next kernel in the stream may be scheduled now; it waits for this one to
    // complete before it touches anything this one reads or writes
    if (threadIdx.x == 0) griddep_launch();

    if (warp == 0) {
        // ------------------------------------------------------------ weight copies (R ring)
        // every lane keeps the same bookkeeping; lane 0 waits and arms, the runs'
        // copies are spread over the lanes
        WRun run[kCR];
        int nrun = 0, ir = 0, armed = 0, nchunk = 0;
        auto flush = [&](int end) -> bool {
            const int base = (end - 1) & ~(kCR - 1);
            uint32_t total = 0;
            for (int j = 0; j < nrun; ++j) total += run[j].bytes + run[j].zbytes;
            bool ok = true;
            if (lane == 0) {
                // the chunk's place released by every widening warp in the previous pass
                ok = mbar_wait_bounded(&S.r_rel[(base % C::kR) / kCR], ((base / C::kR) & 1) ^ 1, abort, a.status,
                                       a.timeout_ns);
                if (ok) mbar_arrive_expect_tx(&S.r_full[base % C::kR], total);
            }
            if (!__shfl_sync(0xffffffffu, ok, 0)) return false;
            uint64_t* bar = &S.r_full[base % C::kR];
            const int l0 = (nchunk * 2 * kCR) & 31;
            for (int j = 0; j < nrun; ++j) {
                if (lane == ((l0 + 2 * j) & 31)) bulk_g2s(S.R[run[j].slot % C::kR], run[j].src, run[j].bytes, bar);
                if (run[j].zbytes != 0 && lane == ((l0 + 2 * j + 1) & 31))
                    bulk_g2s(&S.Z[run[j].slot % C::kR][0], run[j].zsrc, run[j].zbytes, bar);
            }
            nrun = 0;
            ++nchunk;
            armed = end;
            return true;
        };
        if (!a.stall_test) {
            for (int u = blockIdx.x; u < a.n_units; u += gridDim.x) {
                const Unit un = unit_of(a, u);
                const int w = un.eight ? 2 : 1;
                const int ns = (un.kb1 - un.kb0) * w;       // the unit's slots
                const size_t blk = size_t(un.lt) * g.kblocks + un.kb0;
                // slot o of the unit holds bytes [o, o + 1) x 8 KB of its codes
                const uint8_t* src = un.eight ? reinterpret_cast<const uint8_t*>(g.codes8) + blk * kABytes
                                              : g.codes4 + blk * kSlotBytes;
                const uint8_t* zsrc = g.zeros4 + (size_t(un.lt) * g.G + size_t(un.kb0) * gpk) * kTileRows;
                for (int o = 0; o < ns;) {
                    const int take = min(ns - o, kCR - ir % kCR);
                    run[nrun].src = src + size_t(o) * kSlotBytes;
                    run[nrun].zsrc = zsrc + size_t(o) * gpk * kTileRows;
                    run[nrun].slot = ir;
                    run[nrun].bytes = uint32_t(take * kSlotBytes);
                    run[nrun].zbytes = un.eight ? 0u : uint32_t(take * gpk * BM);
                    ++nrun;
                    ir += take;
                    o += take;
                    if (ir % kCR == 0 && !flush(ir)) goto wload_done;
                }
            }
            if (ir % kCR != 0) flush(ir);
        }
    wload_done:
        // no copy may target this CTA's shared memory after it exits: wait for the
        // last use of every chunk place
        if (lane == 0 && armed > 0) {
            const int last = (armed - 1) & ~(kCR - 1);
            for (int b = max(0, last - C::kR + kCR); b <= last; b += kCR) {
                int dummy = 0;
                mbar_wait_bounded(&S.r_full[b % C::kR], (b / C::kR) & 1, &dummy, nullptr, a.timeout_ns);
            }
        }
    } else if (warp == 3) {
        // ------------------------------------------------------------ token copies (B ring)
        griddep_wait();                              // the tokens come from the previous kernel
        constexpr int kCB = C::kCB;
        TRun run[kCB];
        int nrun = 0, ia = 0, armed = 0, nchunk = 0;
        auto flush = [&](int end) -> bool {
            const int base = (end - 1) & ~(kCB - 1);
            const int ci = base / kCB;
            bool ok = true;
            if (lane == 0) {
                // the chunk's place released in the previous pass (one arrival per issuer)
                ok = mbar_wait_bounded(&S.b_empty[ci % C::kBChunks], ((ci / C::kBChunks) & 1) ^ 1, abort, a.status,
                                       a.timeout_ns);
                // tokens past M read as zeros; the boxes are always counted whole
                if (ok) mbar_arrive_expect_tx(&S.b_full[base % C::kB], uint32_t((end - base) * C::kBBytes));
            }
            if (!__shfl_sync(0xffffffffu, ok, 0)) return false;
            uint64_t* bar = &S.b_full[base % C::kB];
            int l = (nchunk * kCB) & 31;
            for (int j = 0; j < nrun; ++j) {
                if (run[j].n == kCB) {
                    if (lane == (l & 31)) tma_load_3d(S.B[run[j].stage % C::kB], &amapC, 0, 0, run[j].kb, bar);
                    ++l;
                } else {
                    for (int t = 0; t < run[j].n; ++t, ++l)
                        if (lane == (l & 31)) tma_load_3d(S.B[(run[j].stage + t) % C::kB], &amap1, 0, 0, run[j].kb + t, bar);
                }
            }
            nrun = 0;
            ++nchunk;
            armed = end;
            return true;
        };
        if (!a.stall_test) {
            for (int u = blockIdx.x; u < a.n_units; u += gridDim.x) {
                const Unit un = unit_of(a, u);
                for (int kb = un.kb0; kb < un.kb1;) {
                    const int take = min(un.kb1 - kb, kCB - ia % kCB);
                    run[nrun].kb = kb;
                    run[nrun].n = take;
                    run[nrun].stage = ia;
                    ++nrun;
                    ia += take;
                    kb += take;
                    if (ia % kCB == 0 && !flush(ia)) goto tload_done;
                }
            }
            if (ia % kCB != 0) flush(ia);
        }
    tload_done:
        if (lane == 0 && armed > 0) {
            const int last = (armed - 1) & ~(kCB - 1);
            for (int b = max(0, last - C::kB + kCB); b <= last; b += kCB) {
                int dummy = 0;
                mbar_wait_bounded(&S.b_full[b % C::kB], (b / C::kB) & 1, &dummy, nullptr, a.timeout_ns);
            }
        }
    } else if (warp <= 2) {
        // ------------------------------------------------------------ MMAs
        // issuer `mine` takes the groups with gc % 2 == mine (accumulators of that parity)
        const uint32_t mine = uint32_t(warp - 1);
        if (lane == 0) {
            const uint32_t idesc = idesc_i8(BM, NT);
            int ia = 0, hb_seen = -1;
            uint32_t gc = 0;
            bool any = false;                        // an MMA of mine reads the current token chunk
            for (int u = blockIdx.x; u < a.n_units; u += gridDim.x) {
                const Unit un = unit_of(a, u);
                const bool last_unit = u + int(gridDim.x) >= a.n_units;
                for (int kb = un.kb0; kb < un.kb1; ++kb, ++ia) {
                    const int sa = ia % C::kA, sb = ia % C::kB;
                    if (gpk == 2 || (gc & 1u) == mine) {
                        // the k-block's tokens: their chunk's barrier, once per chunk (every chunk
                        // but the last holds k-blocks of both issuers, so each issuer waits on
                        // every chunk barrier in the order of its phases)
                        const int hb = ia & ~(C::kCB - 1);
                        if (hb != hb_seen) {
                            if (!mbar_wait_bounded(&S.b_full[hb % C::kB], (hb / C::kB) & 1, abort, a.status,
                                                   a.timeout_ns))
                                goto mma_out;
                            hb_seen = hb;
                        }
                        if (!mbar_wait_bounded(&S.ready[sa], (ia / C::kA) & 1, abort, a.status, a.timeout_ns))
                            goto mma_out;
                        tc_fence_after();
                        const uint32_t a0 = smem_u32(S.A[sa]), b0 = smem_u32(S.B[sb]);
                        for (int j = 0; j < gpk; ++j, ++gc) {
                            if ((gc & 1u) != mine) continue;
                            const uint32_t b = gc % C::kSlots;
                            // use gc / kSlots of accumulator b: phase 0 is the epilogue's first release
                            if (!mbar_wait_bounded(&S.acc_empty[b], (gc / C::kSlots) & 1, abort, a.status,
                                                   a.timeout_ns))
                                goto mma_out;
                            tc_fence_after();
                            // the group's first k-step overwrites the accumulator
                            for (int kk = 0; kk < ksteps; ++kk) {
                                const uint32_t off = uint32_t(j * g.group + kk * 32);
                                mma_i8(tmem + b * NT, sw128_kmajor_desc(a0 + off), sw128_kmajor_desc(b0 + off),
                                       idesc, kk > 0 ? 1u : 0u);
                            }
                            mma_commit(&S.acc_full[b]);
                            mma_commit(&S.a_empty[sa]);
                            any = true;
                        }
                    } else {
                        ++gc;                        // the other issuer's group
                    }
                    // leaving a token chunk: release it (after my MMAs that read it).  Only
                    // the CTA's last chunk can hold no k-block of mine; no copy waits on its
                    // release, and an arrival for it could complete the phase of the chunk
                    // this ring place held before, while the other issuer still reads it
                    if ((ia + 1) % C::kCB == 0 || (last_unit && kb + 1 == un.kb1)) {
                        if (any) mma_commit(&S.b_empty[(ia / C::kCB) % C::kBChunks]);
                        any = false;
                    }
                }
            }
        mma_out:
            mma_commit(&S.mma_done[mine]);           // all MMAs issued so far complete before teardown
            int dummy = 0;
            mbar_wait_bounded(&S.mma_done[mine], 0, &dummy, nullptr, a.timeout_ns);
        }
    } else if (warp >= kWiden0 && warp < C::kEpiWarp0) {
        // ------------------------------------------------------------ widening (R ring -> A ring)
        // group q (kGW warps) widens the k-blocks with ia % kGroups == q into operand
        // stage ia % kA (always its own).  Every group waits on every weight chunk's
        // barrier and releases every chunk, in order: the copy thread re-arms a chunk
        // only after all widening warps released it, so no group can be two phases
        // away from a barrier it waits on
        constexpr int kGT = C::kGT, kPer = kSlotBytes / 16 / kGT;   // 16-byte chunks per thread and slot
        const int q = (warp - kWiden0) / kGW;
        const int gt = threadIdx.x - (kWiden0 + q * kGW) * 32;      // thread within the group
        int ir = 0, ia = 0;
        int entered = -kCR, released = 0;           // last weight chunk waited on, next to release
        for (int u = blockIdx.x; u < a.n_units; u += gridDim.x) {
            const Unit un = unit_of(a, u);
            const int w = un.eight ? 2 : 1;
            const int ufs = ir;                      // the unit's first slot
            for (int kb = un.kb0; kb < un.kb1; ++kb, ++ia, ir += w) {
                // enter the chunks up to the one holding the k-block's last slot
                bool ok = true;
                while (ok && entered + kCR <= ir + w - 1) {
                    entered += kCR;
                    ok = mbar_wait_bounded(&S.r_full[entered % C::kR], (entered / C::kR) & 1, abort, a.status,
                                           a.timeout_ns);
                }
                if (!__all_sync(0xffffffffu, ok)) goto widen_done;
                if (ia % C::kGroups == q) {
                    const int sa = ia % C::kA;
                    ok = mbar_wait_bounded(&S.a_empty[sa], ((ia / C::kA) & 1) ^ 1, abort, a.status, a.timeout_ns);
                    if (!__all_sync(0xffffffffu, ok)) goto widen_done;
                    uint8_t* out = S.A[sa];
                    if (!un.eight) {
                        // the run holding this slot starts at the later of its chunk's and its unit's first slot
                        const int h0 = ir & ~(kCR - 1), rs = max(h0, ufs);
                        const uint8_t* raw = S.R[ir % C::kR];
                        const uint8_t* zs = &S.Z[rs % C::kR][0] + (ir - rs) * gpk * BM;
                        uint4 wv[kPer];
                        uint32_t zb[kPer];
#pragma unroll
                        for (int j = 0; j < kPer; ++j) {
                            const int i = gt + kGT * j, r = i >> 2, c = i & 3;
                            wv[j] = *reinterpret_cast<const uint4*>(raw + i * 16);
                            // z of the group holding this chunk's 32 codes
                            zb[j] = zs[(gpk == 2 ? (c >> 1) : 0) * BM + r];
                        }
#pragma unroll
                        for (int j = 0; j < kPer; ++j) {
                            const int i = gt + kGT * j, r = i >> 2, c = i & 3;
                            const uint32_t zc = (0x80u - zb[j]) * 0x01010101u;   // (128 - z) in every byte
                            uint4 o0, o1;
                            o0.x = widen_lo(wv[j].x, zc); o0.y = widen_hi(wv[j].x, zc);
                            o0.z = widen_lo(wv[j].y, zc); o0.w = widen_hi(wv[j].y, zc);
                            o1.x = widen_lo(wv[j].z, zc); o1.y = widen_hi(wv[j].z, zc);
                            o1.z = widen_lo(wv[j].w, zc); o1.w = widen_hi(wv[j].w, zc);
                            *reinterpret_cast<uint4*>(out + swz128_offset(r, 2 * c)) = o0;
                            *reinterpret_cast<uint4*>(out + swz128_offset(r, 2 * c + 1)) = o1;
                        }
                    } else {
                        // the stored 8-bit operand is already in the MMA's layout: its two
                        // slots (the second may wrap to the ring's start) copied as they are
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            const uint8_t* raw = S.R[(ir + h) % C::kR];
                            uint4 wv[kPer];
#pragma unroll
                            for (int j = 0; j < kPer; ++j) wv[j] = *reinterpret_cast<const uint4*>(raw + (gt + kGT * j) * 16);
#pragma unroll
                            for (int j = 0; j < kPer; ++j)
                                *reinterpret_cast<uint4*>(out + h * kSlotBytes + (gt + kGT * j) * 16) = wv[j];
                        }
                    }
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&S.ready[sa]);
                }
                // release the chunks whose slots all precede the next k-block
                __syncwarp();
                for (; released + kCR <= ir + w; released += kCR)
                    if (lane == 0) mbar_arrive(&S.r_rel[(released % C::kR) / kCR]);
            }
        }
        // the last, partly filled chunk
        __syncwarp();
        for (; released <= entered; released += kCR)
            if (lane == 0) mbar_arrive(&S.r_rel[(released % C::kR) / kCR]);
    widen_done:;
    } else if (warp >= C::kEpiWarp0) {
        // ------------------------------------------------------------ epilogue
        griddep_wait();                              // s_a, Y and part belong to the stream's order
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
size_t tcd_smem() {
    static_assert(sizeof(Smem<NT>) + 1024 <= 227 * 1024, "shared memory of one CTA");
    return sizeof(Smem<NT>) + 1024;
}

template <int NT>
cudaError_t launch_nt(const CUtensorMap& map1, const CUtensorMap& mapC, const TcdArgs& a, int grid, bool debug, int ag,
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
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(Cfg<NT>::kThreads);
    cfg.dynamicSmemBytes = tcd_smem<NT>();
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;   // weights stream before the wait
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, k, map1, mapC, a);
}

}  // namespace

int tcd_tokens(int M) { return M <= 16 ? 16 : M <= 32 ? 32 : M <= 64 ? 64 : 128; }

// The K split with the smallest estimated time: the units the busiest SM processes
// (waves), each costing its k-blocks at the time one k-block takes an SM at this
// token tile plus the fill and drain of the pipeline, as measured on this part
// (about 0.45 us per k-block at 16 tokens to 0.9 us at 128, where the epilogue
// drains larger accumulators, and about 3 us per unit); a split adds the reduction
// kernel and the split sums (written, then read back), and the weights cannot stream
// faster than HBM (about 6 TB/s).
int tcd_auto_split(const mx_layout& L, int M, int sms) {
    const int tiles = L.t8 + L.t4, nkb = L.kblocks;
    if (M <= 0 || sms <= 0) return 1;
    const int NT = tcd_tokens(M);
    const double t_kb = NT <= 16 ? 0.45 : NT <= 32 ? 0.55 : NT <= 64 ? 0.68 : 0.9;   // us per k-block and SM
    const double bw = 6.0e6, t_unit = 3.0, t_split = 4.0;                             // bytes per us, us, us
    const double wbytes = double(L.n8) * L.K + double(L.n4) * L.K / 2 + 2.5 * double(L.N) * L.G;
    int best = 1;
    double best_t = 1e30;
    for (int S = 1; S <= kTcdMaxSplit && S <= nkb; ++S) {
        const int per = (nkb + S - 1) / S;
        if ((nkb + per - 1) / per != S) continue;            // no empty split
        const double waves = double((tiles * S + sms - 1) / sms);
        const double t = std::max(waves * (per * t_kb + t_unit), wbytes / bw) +
                         (S > 1 ? t_split + 8.0 * S * M * double(L.N) / bw : 0.0);
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
    // activations as a 3-D tensor [k-block][token][128 bytes]: one box brings one k-block
    // of the batch as swizzled 128-byte rows (map1), or a chunk of consecutive k-blocks
    // (mapC)
    CUtensorMap map1, mapC;
    const cuuint64_t dims[3] = {cuuint64_t(kKBlock), cuuint64_t(M), cuuint64_t(L.kblocks)};
    const cuuint64_t strides[2] = {cuuint64_t(L.K), cuuint64_t(kKBlock)};
    const cuuint32_t estr[3] = {1, 1, 1};
    for (int z : {1, token_chunk(NT)}) {
        const cuuint32_t box[3] = {cuuint32_t(kKBlock), cuuint32_t(NT), cuuint32_t(z)};
        CUresult r = enc(z == 1 ? &map1 : &mapC, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<int8_t*>(Aq), dims,
                         strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
    }
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
        case 16: e = launch_nt<16>(map1, mapC, a, grid, dbg, ag, s); break;
        case 32: e = launch_nt<32>(map1, mapC, a, grid, dbg, ag, s); break;
        case 64: e = launch_nt<64>(map1, mapC, a, grid, dbg, ag, s); break;
        default: e = launch_nt<128>(map1, mapC, a, grid, dbg, ag, s); break;
    }
    if (e != cudaSuccess || a.S == 1) return e;
    return launch_split_reduce(a.part, a.S, M, L.N, s_a, ag, Y, ldy, sms, s);
}

}  // namespace mx
