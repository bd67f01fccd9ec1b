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
// cluster; S is chosen so that the whole grid is resident at once (one wave).
// Each CTA streams its k-blocks -- codes, group scales and zero points --
// through a ring of shared-memory slots of up to four k-blocks each, filled by
// asynchronous copies that one producer warp issues (one copy per operand per
// slot: a bulk copy for the contiguous 4-bit codes, scales and zero points, a
// 4-D tensor copy for the half-tile rows of 8-bit codes), so the eight consumer
// warps spend their issue slots on shared-memory reads and dp4a only.  Consumers leave per-row partial sums in
// shared memory; rank 0 of the cluster adds the S partials in rank order
// (deterministic) through distributed shared memory, applies s_a and scatters
// the rows to their original columns of Y (section 3.3, fused scatter).  No
// workspace and no second kernel.
//
// The kernel is launched as a programmatic dependent of whatever precedes it on
// the stream: the weight stream starts at once, and only the activation reads
// wait (griddepcontrol.wait).  It lets its own dependents launch at once.
//
// Activations come either quantized (Aq, s_a from the activation quantizer) or
// raw (X in fp16/fp32, up to four tokens): then each CTA stages its own K slice
// of X, the cluster exchanges the slice maxima (the row absmax is their max,
// exactly), and each CTA quantizes its slice with the quantizer's own device
// functions, so the codes are identical to the two-kernel path.
#include <algorithm>
#include <cooperative_groups.h>
#include <cstring>
#include <type_traits>

#include "mx_internal.cuh"
#include "sm100.cuh"

namespace mx {
namespace {

namespace cg = cooperative_groups;
using namespace sm100;

constexpr int kConsumers = 256;               // 8 warps: thread -> (row, 32-byte slice)
constexpr int kThreads = kConsumers + 32;     // + one producer warp
constexpr int kProducerWarp = kConsumers / 32;
// per k-block of a slot: one unit's codes, <= 2 groups x 128 rows of fp16
// scales, <= 2 groups x 128 rows of uint8 zero points
constexpr int kKbCodes = 8192;
constexpr int kKbScales = 2 * kTileRows * 2;
constexpr int kKbZeros = 2 * kTileRows;
constexpr int kKbSlotBytes = kKbCodes + kKbScales + kKbZeros;
constexpr int kMaxKps = 4;                    // k-blocks per slot
constexpr int kMaxSlots = 4;
constexpr int kMaxActSmem = 64 * 1024;        // activation slice staged in shared memory
constexpr int kMaxSmem = 200 * 1024;
constexpr int kMaxCluster = 8;                // portable cluster size
constexpr int kFullRowBytes = 16 * 1024;      // X rows staged whole up to this size
constexpr int kConsumerBar = 1;               // named barrier of the consumer warps
constexpr uint64_t kTimeoutNs = 2000000000ull;

static_assert(kKbSlotBytes % 128 == 0, "tensor copies need 128-byte aligned slots");

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
    int kps;          // k-blocks per slot
    int ns;           // ring slots
    int off_act, off_sa64, off_part, off_raw, off_sag;   // dynamic shared-memory layout
    int xfull;        // in-kernel quantization stages whole X rows (no exchange)
    int ag;           // 0: one activation scale per token; g: one per token and group
    int32_t* debug;
    int32_t* status;  // MX_ERR_TIMEOUT if a bounded wait ran out (never expected)
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

__device__ __forceinline__ void griddep_wait() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

__device__ __forceinline__ void consumer_sync() {
    asm volatile("bar.sync %0, %1;" ::"n"(kConsumerBar), "n"(kConsumers) : "memory");
}

__device__ __forceinline__ void cluster_arrive() {
    asm volatile("barrier.cluster.arrive.release;" ::: "memory");
}

__device__ __forceinline__ void cluster_wait() {
    asm volatile("barrier.cluster.wait.acquire;" ::: "memory");
}

// the same shared-memory address in CTA `rank` of this cluster
__device__ __forceinline__ uint32_t map_rank(uint32_t addr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
    return r;
}

// asynchronous store into another CTA's shared memory that counts its 4 bytes
// on that CTA's mbarrier (complete_tx), so the receiver's wait covers every
// writer thread's data
__device__ __forceinline__ void st_async_f32(uint32_t remote_addr, float v, uint32_t remote_bar) {
    asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.b32 [%0], %1, [%2];"
                 ::"r"(remote_addr), "r"(__float_as_uint(v)), "r"(remote_bar) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait_cluster(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity) : "memory");
    return ok != 0;
}

// bounded wait on a cluster-scope phase (remote arrivals); false after the limit
__device__ __forceinline__ bool cluster_phase_wait(uint64_t* bar, uint32_t parity, int32_t* status) {
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait_cluster(bar, parity)) {
        if (globaltimer_ns() - t0 > kTimeoutNs) {
            if (status) atomicExch(status, MX_ERR_TIMEOUT);
            return false;
        }
    }
    return true;
}

// bounded wait for copies to land, ignoring the abort flag (used before exit)
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(bar, parity))
        if (globaltimer_ns() - t0 > kTimeoutNs) return;
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

// four staged activations from shared memory, widened to fp32
__device__ __forceinline__ void smem4(const __half* p, float (&v)[4]) {
    const uint2 raw = *reinterpret_cast<const uint2*>(p);
    const float2 a = __half22float2(*reinterpret_cast<const __half2*>(&raw.x));
    const float2 b = __half22float2(*reinterpret_cast<const __half2*>(&raw.y));
    v[0] = a.x; v[1] = a.y; v[2] = b.x; v[3] = b.y;
}
__device__ __forceinline__ void smem4(const float* p, float (&v)[4]) {
    const float4 a = *reinterpret_cast<const float4*>(p);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
}

// resident CTAs per SM each variant is compiled for (register budget)
__host__ __device__ constexpr int decode_ctas_per_sm(int mt) {
    return mt <= 2 ? 3 : mt <= 8 ? 2 : 1;
}

// XT: void -- read Aq and s_a produced by the activation quantizer; __half or
// float -- read X and quantize in-kernel (see the file comment).
template <int MT, bool DEBUG, typename XT>
__global__ void __launch_bounds__(kThreads, decode_ctas_per_sm(MT))
gemm_decode_kernel(const __grid_constant__ CUtensorMap codes8_map, const __grid_constant__ DecArgs a) {
    extern __shared__ __align__(128) uint8_t smem_raw[];
    // tensor copies land on 128-byte boundaries: align the base (the plan adds 128 bytes)
    uint8_t* smem = smem_raw + ((128u - (smem_u32(smem_raw) & 127u)) & 127u);
    const Geom& g = a.g;
    const int rank = int(cg::this_cluster().block_rank());
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
    const int warp = tid >> 5, lane = tid & 31;
    const int gpk = kKBlock / g.group;                     // groups per k-block: 1 or 2

    __shared__ uint64_t full[kMaxSlots], empty[kMaxSlots];
    __shared__ uint64_t red_bar, x_bar;
    __shared__ int abort_flag;
    if (tid == 0) {
        for (int i = 0; i < a.ns; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], kConsumers / 32);
        }
        mbar_init(&red_bar, 1);      // completes on rank 0's expect_tx + the peers' stores
        mbar_init(&x_bar, 1);
        abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    // Peers store into this CTA's exchange slots (counted on red_bar / x_bar)
    // only after every CTA of the cluster has initialized its barriers: each
    // thread's arrive here is matched by its wait before its first remote access
    // (or before it exits).
    cluster_arrive();
    asm volatile("griddepcontrol.launch_dependents;");
    uint8_t* ring = smem;

    if (warp == kProducerWarp) {
        // ---- producer: slot use c carries k-blocks kb0 + c*kps .. (codes, scales,
        // zero points). These do not depend on the previous kernel: they start at once.
        const uint8_t* codes4 = g.codes4 + size_t(tile) * g.kblocks * kBlock4Bytes;
        const uint32_t sbytes = uint32_t(gpk) * kTileRows * 2;          // per k-block
        const uint32_t zbytes = eight ? 0u : uint32_t(gpk) * kTileRows;
        const uint8_t* scl = reinterpret_cast<const uint8_t*>(eight ? g.scales8 : g.scales4) +
                             size_t(tile) * g.G * kTileRows * 2;
        const uint8_t* zer = g.zeros4 + size_t(tile) * g.G * kTileRows;   // read for 4-bit units only
        const int kps = a.kps;
        const int uses = (nkb + kps - 1) / kps;
        int issued = 0;
        for (int c = 0; c < uses; ++c) {
            const int s = c % a.ns;
            if (c >= a.ns) {
                bool ok = true;
                if (lane == 0)
                    ok = mbar_wait_bounded(&empty[s], uint32_t((c / a.ns - 1) & 1), &abort_flag, a.status, kTimeoutNs);
                if (!__shfl_sync(0xffffffffu, ok, 0)) break;
            }
            const int kb = kb0 + c * kps;
            const int nk = min(kps, kb1 - kb);
            uint8_t* slot = ring + size_t(s) * kps * kKbSlotBytes;
            // an 8-bit box always spans kps k-blocks (beyond K it is zero-filled)
            const uint32_t cbytes = eight ? uint32_t(kps) * kKbCodes : uint32_t(nk) * kKbCodes;
            const int l0 = (c % 10) * 3;        // consecutive slots from different lanes
            if (lane == l0) mbar_arrive_expect_tx(&full[s], cbytes + nk * (sbytes + zbytes));
            __syncwarp();
            if (lane == l0) {
                if (eight) tma_load_4d(slot, &codes8_map, 0, row0, kb, tile, &full[s]);
                else bulk_g2s(slot, codes4 + size_t(kb) * kBlock4Bytes, cbytes, &full[s]);
            } else if (lane == l0 + 1) {
                bulk_g2s(slot + kps * kKbCodes, scl + size_t(kb) * sbytes, nk * sbytes, &full[s]);
            } else if (lane == l0 + 2 && !eight) {
                bulk_g2s(slot + kps * (kKbCodes + kKbScales), zer + size_t(kb) * zbytes, nk * zbytes, &full[s]);
            }
            issued = c + 1;
        }
        // every copy has landed before the CTA may exit
        if (lane == 0)
            for (int c = max(0, issued - a.ns); c < issued; ++c)
                drain_wait(&full[c % a.ns], uint32_t((c / a.ns) & 1));
        __syncwarp();
        cluster_wait();
        return;
    }

    // ---- consumers (warps 0-7)
    // rank 0 scatters rows tid % rows (rows divides the thread count): their
    // columns of Y come from the row map, which does not depend on the previous kernel
    const int y_slot = eight ? tile * kTileRows + row0 + tid % rows : (g.t8 + tile) * kTileRows + tid % rows;
    const int y_col = rank == 0 ? g.rowmap[y_slot] : -1;
    const int rowb = a.kbu * kKBlock;
    int8_t* act = reinterpret_cast<int8_t*>(smem + a.off_act);
    int32_t* sa64 = reinterpret_cast<int32_t*>(smem + a.off_sa64);
    float* part = reinterpret_cast<float*>(smem + a.off_part);   // [S][MT][128], rank 0's is used
    __shared__ float sa_loc[MT];                                  // token scales quantized in-kernel
    bool cluster_waited = false;                                  // (the wait matching the arrive)
    griddep_wait();
    // group-wise activation scales of this CTA's groups: [MT][kbu * gpk]
    float* sag = reinterpret_cast<float*>(smem + a.off_sag);
    const int ngl = a.kbu * gpk;
    if constexpr (std::is_void_v<XT>) {
        // ---- stage Aq[m0 .. m0+MT)[kb0*128 .. kb1*128) (zero rows beyond M)
        const int chunks = nkb * (kKBlock / 16);
        for (int i = tid; i < MT * chunks; i += kConsumers) {
            const int j = i / chunks, c = i % chunks;
            uint4 v = make_uint4(0, 0, 0, 0);
            if (m0 + j < a.M)
                v = __ldg(reinterpret_cast<const uint4*>(a.Aq + int64_t(m0 + j) * g.K + kb0 * kKBlock) + c);
            *reinterpret_cast<uint4*>(act + j * rowb + c * 16) = v;
        }
        if (a.ag) {
            for (int i = tid; i < MT * nkb * gpk; i += kConsumers) {
                const int j = i / (nkb * gpk), li = i % (nkb * gpk);
                sag[j * ngl + li] =
                    m0 + j < a.M ? __half2float(a.s_a[int64_t(m0 + j) * g.G + kb0 * gpk + li]) : 0.0f;
            }
        }
    } else if (a.ag) {
        // ---- group-wise scales: this CTA's k-blocks hold whole groups, so it stages its
        // slice, takes each group's absmax over its lane segment and quantizes it; no
        // exchange between the CTAs of the cluster
        const XT* X = static_cast<const XT*>(a.X);
        const int xrow = a.kbu * kKBlock;
        XT* xs = reinterpret_cast<XT*>(smem + a.off_raw);
        const int chunks = nkb * kKBlock * int(sizeof(XT)) / 16;
        for (int i = tid; i < MT * chunks; i += kConsumers) {
            const int j = i / chunks, c = i % chunks;
            if (m0 + j < a.M)
                cp_async16(reinterpret_cast<uint8_t*>(xs + size_t(j) * xrow) + size_t(c) * 16,
                           reinterpret_cast<const uint8_t*>(X + int64_t(m0 + j) * a.ldx + kb0 * kKBlock) +
                               size_t(c) * 16);
        }
        cp_async_wait_all();
        consumer_sync();
        const int cpg = a.ag / 8, n8 = nkb * (kKBlock / 8);
#pragma unroll
        for (int j = 0; j < MT; ++j) {
            const bool row = m0 + j < a.M;
            for (int c0 = 0; c0 < n8; c0 += kConsumers) {           // same trip count in every lane
                const int c = c0 + tid;
                const bool live = row && c < n8;
                float v[8];
                if (live) {
                    smem4(xs + size_t(j) * xrow + c * 8, *reinterpret_cast<float(*)[4]>(v));
                    smem4(xs + size_t(j) * xrow + c * 8 + 4, *reinterpret_cast<float(*)[4]>(v + 4));
                } else {
#pragma unroll
                    for (int e = 0; e < 8; ++e) v[e] = 0.0f;
                }
                float am = 0.0f;
#pragma unroll
                for (int e = 0; e < 8; ++e) am = fmaxf(am, fabsf(v[e]));
                for (int o = cpg / 2; o > 0; o >>= 1) am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, o));
                const float sg = __half2float(act_scale(am)), rg = __frcp_rn(sg);
                if (c < n8) {
                    uint2 o = make_uint2(0, 0);
                    if (live) {
                        o.x = quant4(v, sg, rg);
                        o.y = quant4(v + 4, sg, rg);
                    }
                    *reinterpret_cast<uint2*>(act + j * rowb + c * 8) = o;
                    if (c % cpg == 0) sag[j * ngl + c / cpg] = live ? sg : 0.0f;
                }
            }
        }
    } else {
        // ---- in-kernel quantization of X.  Short rows (xfull): every CTA stages the
        // whole rows and takes the absmax itself.  Long rows: every CTA stages its own
        // K slice and the cluster exchanges the slice maxima (their max is the row
        // absmax, exactly).  Either way the CTA then quantizes its own slice with the
        // quantizer's device functions.
        const XT* X = static_cast<const XT*>(a.X);
        const int xrow = a.xfull ? g.K : a.kbu * kKBlock;   // elements per staged row
        const int xoff = a.xfull ? 0 : kb0 * kKBlock;       // first staged column
        const int ncols = a.xfull ? g.K : nkb * kKBlock;    // columns staged per row
        uint8_t* raw = smem + a.off_raw;
        const int chunks = ncols * int(sizeof(XT)) / 16;
        for (int i = tid; i < MT * chunks; i += kConsumers) {
            const int j = i / chunks, c = i % chunks;
            if (m0 + j < a.M)
                cp_async16(raw + (size_t(j) * xrow) * sizeof(XT) + size_t(c) * 16,
                           reinterpret_cast<const uint8_t*>(X + int64_t(m0 + j) * a.ldx + xoff) + size_t(c) * 16);
        }
        cp_async_wait_all();
        consumer_sync();
        const XT* xs = reinterpret_cast<const XT*>(raw);
        const int units8 = ncols / 8;
        __shared__ float red[kConsumers / 32][MT];
        __shared__ float xmax[kMaxCluster][MT];
#pragma unroll
        for (int j = 0; j < MT; ++j) {
            float am = 0.0f;
            if (m0 + j < a.M) {
                for (int c = tid; c < units8; c += kConsumers) am = absmax8(xs + size_t(j) * xrow + c * 8, am);
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, o));
            if (lane == 0) red[warp][j] = am;
        }
        consumer_sync();
        const bool exchange = !a.xfull && a.S > 1;
        if (exchange) {
            cluster_wait();
            cluster_waited = true;
        }
        if (tid < MT) {
            float m = red[0][tid];
#pragma unroll
            for (int w = 1; w < kConsumers / 32; ++w) m = fmaxf(m, red[w][tid]);
            xmax[rank][tid] = m;
            if (exchange) {
                const uint32_t slot = smem_u32(&xmax[rank][tid]), bar = smem_u32(&x_bar);
                for (int q = 0; q < a.S; ++q)
                    if (q != rank) st_async_f32(map_rank(slot, q), m, map_rank(bar, q));
            }
        }
        if (exchange && tid == 0) {
            mbar_arrive_expect_tx(&x_bar, uint32_t(a.S - 1) * MT * 4);
            cluster_phase_wait(&x_bar, 0, a.status);
        }
        consumer_sync();
        float sc[MT], rsc[MT];
#pragma unroll
        for (int j = 0; j < MT; ++j) {
            float m = xmax[rank][j];
            if (exchange)
                for (int q = 0; q < a.S; ++q) m = fmaxf(m, xmax[q][j]);
            sc[j] = __half2float(act_scale(m));
            rsc[j] = __frcp_rn(sc[j]);
            if (tid == j) sa_loc[j] = sc[j];
        }
        // the slice, four values to one word of codes per item, over all threads
        const int sbase = a.xfull ? kb0 * kKBlock : 0;       // slice start in the staged row
        const int words = nkb * (kKBlock / 4);
        for (int i = tid; i < MT * words; i += kConsumers) {
            const int j = i / words, c = i % words;
            float sj = sc[0], rj = rsc[0];
#pragma unroll
            for (int t = 1; t < MT; ++t)
                if (j == t) {
                    sj = sc[t];
                    rj = rsc[t];
                }
            uint32_t o = 0;
            if (m0 + j < a.M) {
                float f[4];
                smem4(xs + size_t(j) * xrow + sbase + c * 4, f);
                o = quant4(f, sj, rj);
            }
            *reinterpret_cast<uint32_t*>(act + j * rowb + c * 4) = o;
        }
    }
    consumer_sync();
    if (!eight) {
        for (int i = tid; i < MT * nkb * 2; i += kConsumers) {
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
        consumer_sync();
    }

    // thread -> (row, 32-byte slice of a k-block row)
    int r, sub;
    if (eight) { r = row0 + (tid >> 2); sub = tid & 3; }   // 4 slices of 32 B per 128-B row
    else { r = tid >> 1; sub = tid & 1; }                   // 2 slices of 32 B per 64-B row
    const int coff = eight ? (r - row0) * kKBlock + sub * 32 : r * 64 + sub * 32;
    // logical 16-column chunks held by this thread (the 8-bit rows are stored swizzled)
    const int lc0 = eight ? (2 * sub) ^ (r & 7) : 4 * sub;
    const int lc1 = eight ? (2 * sub + 1) ^ (r & 7) : 4 * sub + 2;   // 4-bit: second 32 codes
    const int gl = lc0 * 16 / g.group;                    // this thread's group within a k-block
    const int slot_row = eight ? tile * kTileRows + r : (g.t8 + tile) * kTileRows + r;
    const int orig = DEBUG ? g.rowmap[slot_row] : 0;
    float out[MT];
#pragma unroll
    for (int j = 0; j < MT; ++j) out[j] = 0.0f;

    bool ok = true;
    const int kps = a.kps;
    // one k-block of a landed slot: codes, scale and zero point from the slot,
    // activations and their 64-column sums from shared memory
    auto kblock = [&](const uint8_t* sl, int u, int kl) {
        const uint8_t* cw = sl + u * kKbCodes + coff;
        const uint4 w[2] = {*reinterpret_cast<const uint4*>(cw), *reinterpret_cast<const uint4*>(cw + 16)};
        const int gs = (u * gpk + gl) * kTileRows + r;     // (group, row) within the slot
        const float sw = __half2float(reinterpret_cast<const __half*>(sl + kps * kKbCodes)[gs]);
        const int kb = kb0 + kl;
        const int gi = kb * gpk + gl;
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
                    acc[j] = dp4a(w[i].x, av.x, acc[j]);
                    acc[j] = dp4a(w[i].y, av.y, acc[j]);
                    acc[j] = dp4a(w[i].z, av.z, acc[j]);
                    acc[j] = dp4a(w[i].w, av.w, acc[j]);
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
            const int z = sl[kps * (kKbCodes + kKbScales) + gs];
            // word q of the thread's 32 bytes holds k = 8q .. 8q+7 of its 64 columns: the
            // low nibbles pair with k = 8q .. 8q+3 and the high nibbles, left in place
            // (16 x code, an unsigned byte), with k = 8q+4 .. 8q+7
            const uint32_t wd[8] = {w[0].x, w[0].y, w[0].z, w[0].w, w[1].x, w[1].y, w[1].z, w[1].w};
#pragma unroll
            for (int j = 0; j < MT; ++j) {
                const uint4* ap = reinterpret_cast<const uint4*>(act + j * rowb + kl * kKBlock + sub * 64);
                int lo = 0, hi16 = 0;
#pragma unroll
                for (int h = 0; h < 4; ++h) {
                    const uint4 av = ap[h];                  // k = 16h .. 16h+15
                    lo = dp4a(wd[2 * h] & 0x0F0F0F0Fu, av.x, lo);
                    hi16 = dp4a_us(wd[2 * h] & 0xF0F0F0F0u, av.y, hi16);
                    lo = dp4a(wd[2 * h + 1] & 0x0F0F0F0Fu, av.z, lo);
                    hi16 = dp4a_us(wd[2 * h + 1] & 0xF0F0F0F0u, av.w, hi16);
                }
                acc[j] = lo + (hi16 >> 4);                   // exact: hi16 is 16 x the sum
            }
#pragma unroll
            for (int j = 0; j < MT; ++j) {
                acc[j] -= z * sa64[j * 2 * a.kbu + kl * 2 + sub];
                if (g.group == 128) acc[j] += __shfl_xor_sync(0xffffffffu, acc[j], 1);
            }
        }
#pragma unroll
        for (int j = 0; j < MT; ++j) {
            // group-wise activations: the token's scale of this group joins the weight's
            const float s = a.ag ? __fmul_rn(sw, sag[j * ngl + kl * gpk + gl]) : sw;
            out[j] = __fmaf_rn(i2f_biased(acc[j]), s, out[j]);
        }
        if (DEBUG && orig >= 0) {                       // padding rows have no column
            const bool writer = eight ? (g.group == 128 ? sub == 0 : (sub & 1) == 0)
                                      : (g.group == 128 ? sub == 0 : true);
            if (writer) {
#pragma unroll
                for (int j = 0; j < MT; ++j)
                    if (m0 + j < a.M) a.debug[(size_t(m0 + j) * g.N + orig) * g.G + gi] = acc[j];
            }
        }
    };
    const int uses = (nkb + kps - 1) / kps;
    for (int c = 0; c < uses; ++c) {
        const int s = c % a.ns;
        if (ok) ok = mbar_wait_bounded(&full[s], uint32_t((c / a.ns) & 1), &abort_flag, a.status, kTimeoutNs);
        ok = __all_sync(0xffffffffu, ok);
        if (ok) {
            const uint8_t* sl = ring + size_t(s) * kps * kKbSlotBytes;
            const int nk = min(kps, nkb - c * kps);
            // the slot's k-blocks are independent dot products: unrolled, their loads
            // and dp4a chains interleave
#pragma unroll
            for (int u = 0; u < kMaxKps; ++u)
                if (u < nk) kblock(sl, u, c * kps + u);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);     // this warp is done with the slot
    }
    // with g = 64 the slices of a row hold different groups: add them up
    if (g.group == 64) {
#pragma unroll
        for (int j = 0; j < MT; ++j)
            out[j] = __fadd_rn(out[j], __shfl_xor_sync(0xffffffffu, out[j], eight ? 2 : 1));
    }
    const bool lead = sub == 0;
    const int rl = r - row0;                       // row within the unit
    if (!cluster_waited) cluster_wait();
    if (rank != 0) {
        // push this CTA's partials into rank 0's slot `rank`, counted on its red_bar
        if (lead) {
            const uint32_t dst = map_rank(smem_u32(part + (size_t(rank) * MT) * 128 + rl), 0);
            const uint32_t bar = map_rank(smem_u32(&red_bar), 0);
#pragma unroll
            for (int j = 0; j < MT; ++j) st_async_f32(dst + j * 128 * 4, out[j], bar);
        }
        return;
    }
    if (lead) {
#pragma unroll
        for (int j = 0; j < MT; ++j) part[j * 128 + rl] = out[j];
    }
    // rank 0: wait (bounded) for the S-1 other partials, then add them in rank order
    bool okr = true;
    if (a.S > 1 && tid == 0) {
        mbar_arrive_expect_tx(&red_bar, uint32_t(a.S - 1) * MT * rows * 4);
        okr = cluster_phase_wait(&red_bar, 0, a.status);
    }
    okr = named_bar_and(kConsumerBar, kConsumers, okr);
    if (!okr) return;
    for (int i = tid; i < MT * rows; i += kConsumers) {
        const int j = i / rows, rr = i % rows;
        if (m0 + j >= a.M) continue;
        float sum = 0.0f;
        for (int q = 0; q < a.S; ++q) sum = __fadd_rn(sum, part[(size_t(q) * MT + j) * 128 + rr]);
        const int o = y_col;                      // rr == tid % rows
        float sa;
        if (a.ag) sa = 1.0f;                  // group-wise scales were applied per group
        else if constexpr (std::is_void_v<XT>) sa = __half2float(a.s_a[m0 + j]);
        else sa = sa_loc[j];
        if (o >= 0) a.Y[int64_t(m0 + j) * a.ldy + o] = __float2half_rn(__fmul_rn(sum, sa));
    }
}

int ceil_div(int a, int b) { return (a + b - 1) / b; }
size_t align16(size_t v) { return (v + 15) & ~size_t(15); }

template <int MT, bool DEBUG, typename XT>
cudaError_t launch_t(const CUtensorMap& map, const DecArgs& args, int units, int m_tiles, size_t smem,
                     cudaStream_t s) {
    auto k = gemm_decode_kernel<MT, DEBUG, XT>;
    static bool configured[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!configured[dev]) {
        e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxSmem);
        if (e != cudaSuccess) return e;
        // the ring of every resident CTA must fit: ask for the largest shared-memory carveout
        e = cudaFuncSetAttribute(k, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
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
    return cudaLaunchKernelEx(&cfg, k, map, args);
}

template <bool DEBUG>
cudaError_t launch_mt(const CUtensorMap& m, const DecArgs& a, int mt, int units, int m_tiles, size_t smem,
                      cudaStream_t s) {
    switch (mt) {
        case 1: return launch_t<1, DEBUG, void>(m, a, units, m_tiles, smem, s);
        case 2: return launch_t<2, DEBUG, void>(m, a, units, m_tiles, smem, s);
        case 4: return launch_t<4, DEBUG, void>(m, a, units, m_tiles, smem, s);
        case 8: return launch_t<8, DEBUG, void>(m, a, units, m_tiles, smem, s);
        default: return launch_t<16, DEBUG, void>(m, a, units, m_tiles, smem, s);
    }
}

// in-kernel quantization of X: up to four tokens per CTA
template <bool DEBUG, typename XT>
cudaError_t launch_mt_fused(const CUtensorMap& m, const DecArgs& a, int mt, int units, int m_tiles, size_t smem,
                            cudaStream_t s) {
    switch (mt) {
        case 1: return launch_t<1, DEBUG, XT>(m, a, units, m_tiles, smem, s);
        case 2: return launch_t<2, DEBUG, XT>(m, a, units, m_tiles, smem, s);
        case 4: return launch_t<4, DEBUG, XT>(m, a, units, m_tiles, smem, s);
        default: return cudaErrorInvalidValue;
    }
}

// 8-bit codes as a 4-D tensor [tile][k-block][row][128 bytes]: one box brings
// kps k-blocks of one 64-row half tile, k-block after k-block, into a slot
cudaError_t codes8_map(const mx_layout& L, const void* blob, int kps, CUtensorMap* map) {
    memset(map, 0, sizeof *map);
    if (L.t8 == 0) return cudaSuccess;                 // no 8-bit units: never read
    cudaError_t e;
    EncodeTiledFn enc = encode_fn(&e);
    if (e != cudaSuccess) return e;
    const cuuint64_t dims[4] = {cuuint64_t(kKBlock), cuuint64_t(kTileRows), cuuint64_t(L.kblocks), cuuint64_t(L.t8)};
    const cuuint64_t strides[3] = {cuuint64_t(kKBlock), cuuint64_t(kBlock8Bytes),
                                   cuuint64_t(kBlock8Bytes) * uint64_t(L.kblocks)};
    const cuuint32_t box[4] = {cuuint32_t(kKBlock), cuuint32_t(kTileRows / 2), cuuint32_t(kps), 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    void* base = const_cast<uint8_t*>(static_cast<const uint8_t*>(blob) + L.off_codes8);
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, base, dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

DecArgs base_args(const mx_layout& L, const void* blob, int M, uint16_t* Y, int64_t ldy, const DecodePlan& p,
                  int32_t* debug_partials, int32_t* status) {
    DecArgs a{};
    a.g = make_geom(L, blob);
    a.Y = reinterpret_cast<__half*>(Y);
    a.ldy = ldy;
    a.M = M;
    a.S = p.S;
    a.kbu = p.kbu;
    a.kps = p.kps;
    a.ns = p.ns;
    a.off_act = p.off_act;
    a.off_sa64 = p.off_sa64;
    a.off_part = p.off_part;
    a.off_raw = p.off_raw;
    a.xfull = p.xfull;
    a.off_sag = p.off_sag;
    a.debug = debug_partials;
    a.status = status;
    return a;
}

}  // namespace

DecodePlan plan_decode(const mx_layout& L, int M, int split_hint, int x_bytes) {
    DecodePlan p{};
    p.mt = M <= 1 ? 1 : M <= 2 ? 2 : M <= 4 ? 4 : M <= 8 ? 8 : 16;
    p.m_tiles = std::max(1, ceil_div(M, p.mt));
    p.units = 2 * L.t8 + L.t4;
    const int kb = L.kblocks;
    const int cps = decode_ctas_per_sm(p.mt);
    // at least as many CTAs per unit as the activation slice needs to fit in shared memory
    const int s_min = ceil_div(kb * p.mt * kKBlock, kMaxActSmem);
    int S = split_hint;
    if (S <= 0) {
        // the whole grid resident at once on a 148-SM B200 (clusters of up to 8
        // CTAs must also pack into GPCs, so aim a little below the capacity)
        const int work = std::max(1, p.units * p.m_tiles);
        S = std::max(1, cps * 148 * 7 / 8 / work);
    }
    S = std::max(S, s_min);
    S = std::min(S, std::min(kMaxCluster, kb));
    p.S = S;
    p.kbu = ceil_div(kb, S);
    // shared memory: ring | staged activations | 64-column activation sums |
    // partial sums of every rank | raw X slice (in-kernel quantization)
    const size_t act = align16(size_t(p.mt) * p.kbu * kKBlock);
    const size_t sa64 = align16(size_t(p.mt) * 2 * p.kbu * 4);
    const size_t part = size_t(S) * p.mt * kTileRows * 4;
    // in-kernel quantization: whole rows when they are short (no cluster exchange of
    // the row maxima), else this CTA's slice
    p.xfull = x_bytes > 0 && S > 1 && size_t(p.mt) * L.K * x_bytes <= size_t(kFullRowBytes);
    const size_t raw = align16(size_t(p.mt) * (p.xfull ? L.K : p.kbu * kKBlock) * x_bytes);
    const size_t rest = act + sa64 + part + raw;
    // resident CTAs per SM the grid needs (at most what the registers allow)
    const int ctas = p.units * p.m_tiles * S;
    const int need = std::max(1, std::min(cps, ceil_div(ctas, 148 * 7 / 8)));
    // per-SM shared memory / resident CTAs, less the 1 KB the hardware reserves per
    // CTA, the static shared memory and the alignment pad
    const size_t budget = size_t(233472) / need - 2560;
    // the largest slots (fewest copies) that leave room for two of them, or one
    // when a single slot holds the whole K range
    int kps = 1, ns = 1;
    for (int k = std::min(kMaxKps, p.kbu); k >= 1; k = k > 2 ? 2 : k - 1) {
        const int uses = ceil_div(p.kbu, k);
        int n = std::min(uses, kMaxSlots);
        while (n > std::min(uses, 2) && size_t(n) * k * kKbSlotBytes + rest > budget) --n;
        kps = k;
        ns = n;
        if (size_t(n) * k * kKbSlotBytes + rest <= budget) break;
    }
    p.kps = kps;
    p.ns = ns;
    p.off_act = ns * kps * kKbSlotBytes;
    p.off_sa64 = int(p.off_act + act);
    p.off_part = int(p.off_sa64 + sa64);
    p.off_raw = int(p.off_part + part);
    p.off_sag = int(p.off_raw + raw);
    p.smem = size_t(p.off_sag) + align16(size_t(p.mt) * p.kbu * 2 * 4) + 128;   // + room to align the base
    p.ok = S >= s_min && size_t(p.kbu) * p.mt * kKBlock <= size_t(kMaxActSmem) && p.smem <= size_t(kMaxSmem);
    return p;
}

cudaError_t launch_gemm_decode(const mx_layout& L, const void* blob, const int8_t* Aq,
                               const uint16_t* s_a, int M, uint16_t* Y, int64_t ldy,
                               const DecodePlan& plan, int ag, int32_t* debug_partials, int32_t* status,
                               cudaStream_t s) {
    if (M == 0) return cudaSuccess;
    DecArgs a = base_args(L, blob, M, Y, ldy, plan, debug_partials, status);
    a.ag = ag;
    a.Aq = Aq;
    a.s_a = reinterpret_cast<const __half*>(s_a);
    CUtensorMap map;
    cudaError_t e = codes8_map(L, blob, plan.kps, &map);
    if (e != cudaSuccess) return e;
    return debug_partials ? launch_mt<true>(map, a, plan.mt, plan.units, plan.m_tiles, plan.smem, s)
                          : launch_mt<false>(map, a, plan.mt, plan.units, plan.m_tiles, plan.smem, s);
}

bool decode_can_fuse(const mx_layout& L, int M, mx_dtype xdt) {
    // each CTA stages its slice of the X rows: keep whole rows to 64 KB
    return M >= 1 && M <= kMaxFusedTokens &&
           size_t(M) * L.K * (xdt == MX_F16 ? 2 : 4) <= size_t(64) * 1024;
}

cudaError_t launch_gemm_decode_fused(const mx_layout& L, const void* blob, const void* X, mx_dtype xdt,
                                     int64_t ldx, int M, uint16_t* Y, int64_t ldy, const DecodePlan& plan,
                                     int ag, int32_t* debug_partials, int32_t* status, cudaStream_t s) {
    if (M == 0) return cudaSuccess;
    if (plan.mt > kMaxFusedTokens || !plan.ok) return cudaErrorInvalidValue;
    // the plan must have room for the raw slice of this input type
    const size_t cols = plan.xfull ? size_t(L.K) : size_t(plan.kbu) * kKBlock;
    if (size_t(plan.smem) < size_t(plan.off_raw) + 128 + size_t(plan.mt) * cols * (xdt == MX_F16 ? 2 : 4))
        return cudaErrorInvalidValue;
    DecArgs a = base_args(L, blob, M, Y, ldy, plan, debug_partials, status);
    a.ag = ag;
    a.X = X;
    a.ldx = ldx;
    CUtensorMap m;
    cudaError_t e = codes8_map(L, blob, plan.kps, &m);
    if (e != cudaSuccess) return e;
    const int u = plan.units, t = plan.m_tiles;
    if (xdt == MX_F16)
        return debug_partials ? launch_mt_fused<true, __half>(m, a, plan.mt, u, t, plan.smem, s)
                              : launch_mt_fused<false, __half>(m, a, plan.mt, u, t, plan.smem, s);
    return debug_partials ? launch_mt_fused<true, float>(m, a, plan.mt, u, t, plan.smem, s)
                          : launch_mt_fused<false, float>(m, a, plan.mt, u, t, plan.smem, s);
}

}  // namespace mx
