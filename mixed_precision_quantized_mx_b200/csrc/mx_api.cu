// mx_api.cu -- the extern "C" boundary: argument validation, packed-layout
// geometry, workspace sizing and dispatch between the two GEMM paths.
// Nothing here computes on the host beyond sizes; every step of the method
// runs in the kernels of the other translation units.
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>
#include <algorithm>

#include "mx_internal.cuh"
#include "mx_blockwise.h"

namespace {

thread_local std::string g_err;

mx_status fail(mx_status st, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_err = buf;
    return st;
}

mx_status cuda_fail(cudaError_t e, const char* what) {
    return fail(MX_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

uint64_t align256(uint64_t v) { return (v + 255) & ~uint64_t(255); }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

// Device (or managed) memory that kernels may dereference; host pointers are
// rejected so that nothing ever runs through a host-side data path.
mx_status check_device_ptr(const void* p, const char* name) {
    if (p == nullptr) return fail(MX_ERR_INVALID_ARG, "%s is NULL", name);
    cudaPointerAttributes at;
    cudaError_t e = cudaPointerGetAttributes(&at, p);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return fail(MX_ERR_INVALID_ARG, "%s: not a CUDA pointer (%s)", name, cudaGetErrorString(e));
    }
    if (at.type != cudaMemoryTypeDevice && at.type != cudaMemoryTypeManaged)
        return fail(MX_ERR_INVALID_ARG, "%s is not device memory", name);
    return MX_OK;
}

// Device memory of the current device, or pinned host memory with a device
// mapping: *devp is the address kernels use, *host says which.  Pageable host
// memory is rejected (a kernel must never dereference it).
mx_status mapped_ptr(const void* p, const char* name, const void** devp, bool* host) {
    if (p == nullptr) return fail(MX_ERR_INVALID_ARG, "%s is NULL", name);
    cudaPointerAttributes at;
    cudaError_t e = cudaPointerGetAttributes(&at, p);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return fail(MX_ERR_INVALID_ARG, "%s: not a CUDA pointer (%s)", name, cudaGetErrorString(e));
    }
    int dev = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (at.type == cudaMemoryTypeHost) {
        if (at.devicePointer == nullptr) return fail(MX_ERR_INVALID_ARG, "%s: host memory without a device mapping", name);
        *devp = at.devicePointer;
        *host = true;
        return MX_OK;
    }
    if (at.type == cudaMemoryTypeManaged || (at.type == cudaMemoryTypeDevice && at.device == dev)) {
        *devp = p;
        *host = false;
        return MX_OK;
    }
    if (at.type == cudaMemoryTypeDevice) return fail(MX_ERR_INVALID_ARG, "%s is another device's memory", name);
    return fail(MX_ERR_INVALID_ARG, "%s is pageable host memory (pin it first)", name);
}

mx_status check_layout(const mx_layout* L) {
    if (L == nullptr) return fail(MX_ERR_INVALID_ARG, "layout is NULL");
    mx_layout ref;
    mx_status st = mx_layout_init(L->N, L->K, L->group, L->n8, &ref);
    if (st != MX_OK) return st;
    if (memcmp(&ref, L, sizeof ref) != 0)
        return fail(MX_ERR_INVALID_ARG, "layout was modified after mx_layout_init");
    return MX_OK;
}

// act_group: 0 (one activation scale per token) or the layer's weight group
mx_status check_act_group(const mx_layout* L, const mx_gemm_opts* opts) {
    const int ag = opts ? opts->act_group : 0;
    if (ag != 0 && ag != L->group)
        return fail(MX_ERR_UNSUPPORTED, "act_group=%d: 0 or the weight group %d", ag, L->group);
    return MX_OK;
}

int act_group_of(const mx_gemm_opts* opts) { return opts ? opts->act_group : 0; }

// activation scales per token: 1, or one per group
size_t scales_per_token(const mx_layout* L, const mx_gemm_opts* opts) {
    return act_group_of(opts) ? size_t(L->G) : 1;
}

}  // namespace

namespace mx {

// the precision search (saliency.cu)
cudaError_t launch_saliency(const void* W, mx_dtype wdt, int64_t ldw, const void* G, mx_dtype gdt, int64_t ldg,
                            int N, int K, int group, float* S, cudaStream_t s);
size_t select_workspace_bytes();
cudaError_t launch_select_top(const float* S, int64_t n, int64_t n_top, uint8_t* is8, void* workspace,
                              cudaStream_t s);

// block-wise bit widths (blockwise.cu)
cudaError_t launch_bw_pack(const mx_bw_layout& L, const void* W, mx_dtype wdt, int64_t ldw, uint8_t* blob,
                           cudaStream_t s);
cudaError_t launch_bw_gemm(const mx_bw_layout& L, const uint8_t* blob, const int8_t* Aq, const __half* s_a, int M,
                           __half* Y, int64_t ldy, int32_t* P, cudaStream_t s);

Geom make_geom(const mx_layout& L, const void* blob) {
    const uint8_t* b = static_cast<const uint8_t*>(blob);
    Geom g;
    g.blob = b;
    g.rowmap = reinterpret_cast<const int32_t*>(b + L.off_rowmap);
    g.scales8 = reinterpret_cast<const __half*>(b + L.off_scales8);
    g.codes8 = reinterpret_cast<const int8_t*>(b + L.off_codes8);
    g.scales4 = reinterpret_cast<const __half*>(b + L.off_scales4);
    g.zeros4 = b + L.off_zeros4;
    g.codes4 = b + L.off_codes4;
    g.N = L.N; g.K = L.K; g.group = L.group; g.G = L.G; g.n8 = L.n8;
    g.t8 = L.t8; g.t4 = L.t4; g.kblocks = L.kblocks;
    return g;
}

}  // namespace mx

extern "C" {

int mx_version(void) { return MX_ABI_VERSION; }

const char* mx_last_error(void) { return g_err.c_str(); }

mx_status mx_layout_init(int N, int K, int group, int n8, mx_layout* out) {
    if (out == nullptr) return fail(MX_ERR_INVALID_ARG, "out is NULL");
    if (N < 1 || K < 1) return fail(MX_ERR_INVALID_ARG, "N=%d K=%d must be positive", N, K);
    if (n8 < 0 || n8 > N) return fail(MX_ERR_INVALID_ARG, "n8=%d outside [0, N=%d]", n8, N);
    if (group != 64 && group != 128)
        return fail(MX_ERR_UNSUPPORTED, "group=%d: supported group sizes are 64 and 128", group);
    if (K % MX_KBLOCK != 0)
        return fail(MX_ERR_UNSUPPORTED, "K=%d must be a multiple of %d", K, MX_KBLOCK);
    mx_layout L;
    memset(&L, 0, sizeof L);
    L.N = N; L.K = K; L.group = group; L.n8 = n8;
    L.n4 = N - n8;
    L.G = K / group;
    L.t8 = (n8 + MX_TILE_ROWS - 1) / MX_TILE_ROWS;
    L.t4 = (L.n4 + MX_TILE_ROWS - 1) / MX_TILE_ROWS;
    L.kblocks = K / MX_KBLOCK;
    const uint64_t rows8 = uint64_t(L.t8) * MX_TILE_ROWS, rows4 = uint64_t(L.t4) * MX_TILE_ROWS;
    uint64_t off = MX_HEADER_BYTES;
    L.off_rowmap = off;  off = align256(off + (rows8 + rows4) * 4);
    L.off_scales8 = off; off = align256(off + rows8 * L.G * 2);
    L.off_codes8 = off;  off = align256(off + rows8 * K);
    L.off_scales4 = off; off = align256(off + rows4 * L.G * 2);
    L.off_zeros4 = off;  off = align256(off + rows4 * L.G);
    L.off_codes4 = off;  off = align256(off + rows4 * K / 2);
    L.total_bytes = off;
    *out = L;
    return MX_OK;
}

mx_status mx_layout_from_header(const void* host_header, size_t bytes, mx_layout* out) {
    if (host_header == nullptr || out == nullptr)
        return fail(MX_ERR_INVALID_ARG, "header or out is NULL");
    if (bytes < MX_HEADER_BYTES) return fail(MX_ERR_BAD_BLOB, "header shorter than %d bytes", MX_HEADER_BYTES);
    uint32_t h[6];
    memcpy(h, host_header, sizeof h);
    if (h[0] != MX_BLOB_MAGIC) return fail(MX_ERR_BAD_BLOB, "bad magic 0x%08x", h[0]);
    if (h[1] != MX_BLOB_VERSION) return fail(MX_ERR_BAD_BLOB, "blob version %u != %d", h[1], MX_BLOB_VERSION);
    mx_status st = mx_layout_init(int(h[2]), int(h[3]), int(h[4]), int(h[5]), out);
    if (st != MX_OK) return fail(MX_ERR_BAD_BLOB, "header geometry invalid: %s", g_err.c_str());
    return MX_OK;
}

mx_status mx_pack_weights(const mx_layout* L, const void* W, mx_dtype wdtype, int64_t ldw,
                          const uint8_t* is8, void* blob, int32_t* status, void* stream) {
    mx_status st = check_layout(L);
    if (st != MX_OK) return st;
    if (wdtype != MX_F32 && wdtype != MX_F16) return fail(MX_ERR_INVALID_ARG, "bad wdtype %d", int(wdtype));
    if (ldw < L->K) return fail(MX_ERR_INVALID_ARG, "ldw=%lld < K=%d", (long long)ldw, L->K);
    if ((st = check_device_ptr(W, "W")) != MX_OK) return st;
    if ((st = check_device_ptr(is8, "is8")) != MX_OK) return st;
    if ((st = check_device_ptr(blob, "blob")) != MX_OK) return st;
    if (status && (st = check_device_ptr(status, "status")) != MX_OK) return st;
    if (!aligned16(blob)) return fail(MX_ERR_ALIGNMENT, "blob must be 16-byte aligned");
    cudaError_t e = mx::launch_pack(*L, W, wdtype, ldw, is8, blob, status,
                                    static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "pack launch");
    return MX_OK;
}

mx_status mx_quant_act(const void* X, mx_dtype xdtype, int M, int K, int64_t ldx,
                       int8_t* Aq, uint16_t* s_a, void* stream) {
    if (xdtype != MX_F32 && xdtype != MX_F16) return fail(MX_ERR_INVALID_ARG, "bad xdtype %d", int(xdtype));
    if (M < 0 || K < 1) return fail(MX_ERR_INVALID_ARG, "M=%d K=%d", M, K);
    if (K % 8 != 0) return fail(MX_ERR_UNSUPPORTED, "K=%d must be a multiple of 8", K);
    if (ldx < K) return fail(MX_ERR_INVALID_ARG, "ldx=%lld < K=%d", (long long)ldx, K);
    if (M == 0) return MX_OK;
    mx_status st;
    if ((st = check_device_ptr(X, "X")) != MX_OK) return st;
    if ((st = check_device_ptr(Aq, "Aq")) != MX_OK) return st;
    if ((st = check_device_ptr(s_a, "s_a")) != MX_OK) return st;
    const int esz = xdtype == MX_F16 ? 2 : 4;
    if (!aligned16(X) || (ldx * esz) % 16 != 0 || !aligned16(Aq))
        return fail(MX_ERR_ALIGNMENT, "X, Aq and every X row must be 16-byte aligned");
    cudaError_t e = mx::launch_quant_act(X, xdtype, M, K, ldx, Aq, s_a, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "quant_act launch");
    return MX_OK;
}

mx_status mx_quant_act_grouped(const void* X, mx_dtype xdtype, int M, int K, int64_t ldx, int act_group,
                               int8_t* Aq, uint16_t* s_a, void* stream) {
    if (act_group == 0) return mx_quant_act(X, xdtype, M, K, ldx, Aq, s_a, stream);
    if (act_group != 64 && act_group != 128) return fail(MX_ERR_UNSUPPORTED, "act_group=%d (0, 64 or 128)", act_group);
    if (xdtype != MX_F32 && xdtype != MX_F16) return fail(MX_ERR_INVALID_ARG, "bad xdtype %d", int(xdtype));
    if (M < 0 || K < 1) return fail(MX_ERR_INVALID_ARG, "M=%d K=%d", M, K);
    if (K % act_group != 0) return fail(MX_ERR_UNSUPPORTED, "K=%d is not a multiple of act_group=%d", K, act_group);
    if (ldx < K) return fail(MX_ERR_INVALID_ARG, "ldx=%lld < K=%d", (long long)ldx, K);
    if (M == 0) return MX_OK;
    mx_status st;
    if ((st = check_device_ptr(X, "X")) != MX_OK) return st;
    if ((st = check_device_ptr(Aq, "Aq")) != MX_OK) return st;
    if ((st = check_device_ptr(s_a, "s_a")) != MX_OK) return st;
    const int esz = xdtype == MX_F16 ? 2 : 4;
    if (!aligned16(X) || (ldx * esz) % 16 != 0 || !aligned16(Aq))
        return fail(MX_ERR_ALIGNMENT, "X, Aq and every X row must be 16-byte aligned");
    cudaError_t e = mx::launch_quant_act_grouped(X, xdtype, M, K, ldx, act_group, Aq, s_a,
                                                 static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "grouped quant_act launch");
    return MX_OK;
}

// Decode-sized M is bound by HBM: up to 8 tokens the split-K CUDA-core path
// streams the weights with enough CTAs (16 when a cluster split is asked for);
// from 9 to 128 tokens the decode tensor-core path, which measured faster on
// the Llama shapes from about 8 tokens on.
constexpr int kDecodeMaxM = 16;
constexpr int kSplitKAutoMaxM = 8;

// Short K and M <= 4 take the row kernel (whole rows per CTA) unless a cluster
// split is asked for; larger M the tensor cores on CTA pairs, which measured at
// least as fast as the one-CTA tensor-core kernel from 32 tokens up on the
// Llama shapes (path 2 stays available when asked for).
static int pair_count();

// Prefill M: the 256-token pair kernel once its tiles give every CTA pair a unit.
static int choose_path(const mx_layout* L, int M, const mx_gemm_opts* opts) {
    if (opts && opts->path) return opts->path;
    const bool split_asked = opts && opts->split > 0;
    if (!split_asked && mx::plan_rows(*L, M).ok) return 3;
    if (M <= (split_asked ? kDecodeMaxM : kSplitKAutoMaxM) && mx::plan_decode(*L, M, 0).ok) return 1;
    if (M <= mx::kTcdMaxM) return 6;
    if (M >= MX_PATH5_MIN_M && !(opts && opts->split > 1) && mx::tc3_units(*L, M) >= pair_count()) return 5;
    return 4;
}

// CTA pairs the device holds (148 SMs on a B200; that figure when no device answers)
static int pair_count() {
    static int pairs[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
        cudaGetLastError();
        return 74;
    }
    if (pairs[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 2) {
            cudaGetLastError();
            return 74;
        }
        pairs[dev] = n / 2;
    }
    return pairs[dev];
}

// K splits path 4 takes: the caller's, or the automatic choice (1 when the grid is full)
static int pair_split(const mx_layout* L, int M, const mx_gemm_opts* opts) {
    return opts && opts->split > 0 ? opts->split : mx::tc2_auto_split(*L, M, pair_count());
}

// K splits path 6 takes: the caller's, or the automatic choice
static int tcd_split(const mx_layout* L, int M, const mx_gemm_opts* opts) {
    return opts && opts->split > 0 ? opts->split : mx::tcd_auto_split(*L, M, 2 * pair_count());
}

// scratch mx_gemm uses at M tokens: the fp32 split sums of paths 4 and 6, else nothing
static size_t gemm_ws_bytes(const mx_layout* L, int M, const mx_gemm_opts* opts) {
    if (M <= 0) return 0;
    const int path = choose_path(L, M, opts);
    if (path == 4) return mx::tc2_split_bytes(*L, M, pair_split(L, M, opts));
    if (path == 6 && M <= mx::kTcdMaxM) return mx::tcd_split_bytes(*L, M, tcd_split(L, M, opts));
    return 0;
}

int mx_gemm_select_path(const mx_layout* L, int M, const mx_gemm_opts* opts) {
    mx_status st = check_layout(L);
    if (st != MX_OK) return -int(st);
    if (M < 0) return -int(fail(MX_ERR_INVALID_ARG, "M=%d", M));
    return choose_path(L, M, opts);
}

mx_status mx_gemm_workspace_size(const mx_layout* L, int M, const mx_gemm_opts* opts, size_t* bytes) {
    mx_status st = check_layout(L);
    if (st != MX_OK) return st;
    if (bytes == nullptr) return fail(MX_ERR_INVALID_ARG, "bytes is NULL");
    if (M < 0) return fail(MX_ERR_INVALID_ARG, "M=%d", M);
    if (opts && opts->split < 0) return fail(MX_ERR_INVALID_ARG, "split=%d", opts->split);
    *bytes = gemm_ws_bytes(L, M, opts);   // only split tensor-core runs use scratch
    return MX_OK;
}

mx_status mx_gemm(const mx_layout* L, const void* blob, const int8_t* Aq, const uint16_t* s_a,
                  int M, uint16_t* Y, int64_t ldy, void* workspace, size_t ws_bytes,
                  const mx_gemm_opts* opts, void* stream) {
    mx_status st = check_layout(L);
    if (st != MX_OK) return st;
    if (M < 0) return fail(MX_ERR_INVALID_ARG, "M=%d", M);
    if (ldy < L->N) return fail(MX_ERR_INVALID_ARG, "ldy=%lld < N=%d", (long long)ldy, L->N);
    if (M == 0) return MX_OK;
    if (M > 65535) return fail(MX_ERR_UNSUPPORTED, "M=%d above 65535", M);
    if ((st = check_act_group(L, opts)) != MX_OK) return st;
    if ((st = check_device_ptr(blob, "blob")) != MX_OK) return st;
    if ((st = check_device_ptr(Aq, "Aq")) != MX_OK) return st;
    if ((st = check_device_ptr(s_a, "s_a")) != MX_OK) return st;
    if ((st = check_device_ptr(Y, "Y")) != MX_OK) return st;
    if (!aligned16(blob) || !aligned16(Aq)) return fail(MX_ERR_ALIGNMENT, "blob and Aq must be 16-byte aligned");
    if (opts && opts->debug_partials && (st = check_device_ptr(opts->debug_partials, "debug_partials")) != MX_OK)
        return st;
    if (opts && opts->status && (st = check_device_ptr(opts->status, "status")) != MX_OK) return st;
    const int ag = act_group_of(opts);
    const int path = choose_path(L, M, opts);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (path == 3) {
        const mx::RowsPlan rp = mx::plan_rows(*L, M);
        if (!rp.ok) return fail(MX_ERR_UNSUPPORTED, "M=%d K=%d: beyond the row path (M <= 4, K <= 4096, one wave)", M, L->K);
        cudaError_t e = mx::launch_gemm_rows(*L, blob, Aq, s_a, nullptr, MX_F16, 0, M, Y, ldy, rp, ag,
                                             opts ? opts->debug_partials : nullptr, opts ? opts->status : nullptr, s);
        if (e != cudaSuccess) return cuda_fail(e, "row decode GEMM launch");
        return MX_OK;
    }
    if (path == 1) {
        if (opts && opts->split > 8) return fail(MX_ERR_UNSUPPORTED, "split=%d above the cluster limit 8", opts->split);
        mx::DecodePlan plan = mx::plan_decode(*L, M, opts ? opts->split : 0);
        if (!plan.ok)
            return fail(MX_ERR_UNSUPPORTED, "M=%d K=%d: activation slice too large for the decode path", M, L->K);
        cudaError_t e = mx::launch_gemm_decode(*L, blob, Aq, s_a, M, Y, ldy, plan, ag,
                                               opts ? opts->debug_partials : nullptr,
                                               opts ? opts->status : nullptr, s);
        if (e != cudaSuccess) return cuda_fail(e, "decode GEMM launch");
        return MX_OK;
    }
    if (path == 2 || path == 4 || path == 5 || path == 6) {
        if (opts && opts->test_stall && !opts->status)
            return fail(MX_ERR_INVALID_ARG, "test_stall needs a status word");
        if (opts && opts->wait_timeout_us < 0) return fail(MX_ERR_INVALID_ARG, "wait_timeout_us < 0");
        const uint64_t timeout_ns =
            (opts && opts->wait_timeout_us > 0) ? uint64_t(opts->wait_timeout_us) * 1000u : 2000000000ull;
        cudaError_t e;
        if (path == 2) {
            e = mx::launch_gemm_tc(*L, blob, Aq, s_a, M, Y, ldy, ag, opts ? opts->debug_partials : nullptr,
                                   opts ? opts->status : nullptr, timeout_ns, opts ? opts->test_stall : 0, s);
            if (e != cudaSuccess) return cuda_fail(e, "tensor-core GEMM launch");
            return MX_OK;
        }
        if (path == 6) {
            if (M > mx::kTcdMaxM) return fail(MX_ERR_UNSUPPORTED, "M=%d: path 6 serves at most %d tokens", M, mx::kTcdMaxM);
            if (opts && (opts->split < 0 || opts->split > mx::kTcdMaxSplit))
                return fail(MX_ERR_UNSUPPORTED, "split=%d: 1..%d on path 6", opts->split, mx::kTcdMaxSplit);
            // K splits: the caller's (needs the workspace) or automatic (taken only when the
            // workspace holds the split sums)
            const bool asked = opts && opts->split > 0;
            int S = tcd_split(L, M, opts);
            const size_t need = mx::tcd_split_bytes(*L, M, S);
            if (S > 1 && (workspace == nullptr || ws_bytes < need)) {
                if (asked)
                    return fail(MX_ERR_WORKSPACE, "split %d needs a workspace of %zu bytes, %zu given", S, need,
                                workspace ? ws_bytes : size_t(0));
                S = 1;
            }
            if (S > 1) {
                if ((st = check_device_ptr(workspace, "workspace")) != MX_OK) return st;
                if (!aligned16(workspace)) return fail(MX_ERR_ALIGNMENT, "workspace must be 16-byte aligned");
            }
            e = mx::launch_gemm_tcd(*L, blob, Aq, s_a, M, Y, ldy, ag, S, S > 1 ? static_cast<float*>(workspace) : nullptr,
                                    opts ? opts->debug_partials : nullptr, opts ? opts->status : nullptr, timeout_ns,
                                    opts ? opts->test_stall : 0, 2 * pair_count(), s);
            if (e != cudaSuccess) return cuda_fail(e, "decode tensor-core GEMM launch");
            return MX_OK;
        }
        if (path == 5) {
            if (opts && opts->split > 1) return fail(MX_ERR_UNSUPPORTED, "split=%d: path 5 does not split K", opts->split);
            e = mx::launch_gemm_tc3(*L, blob, Aq, s_a, M, Y, ldy, ag, opts ? opts->debug_partials : nullptr,
                                    opts ? opts->status : nullptr, timeout_ns, opts ? opts->test_stall : 0, s);
            if (e != cudaSuccess) return cuda_fail(e, "256-token pair tensor-core GEMM launch");
            return MX_OK;
        }
        // K splits: the caller's (needs the workspace) or automatic (taken only when the
        // workspace holds the split sums)
        const bool asked = opts && opts->split > 0;
        if (opts && (opts->split < 0 || opts->split > mx::kTc2MaxSplit))
            return fail(MX_ERR_UNSUPPORTED, "split=%d: 1..%d on path 4", opts->split, mx::kTc2MaxSplit);
        int S = pair_split(L, M, opts);
        const size_t need = mx::tc2_split_bytes(*L, M, S);
        if (S > 1 && (workspace == nullptr || ws_bytes < need)) {
            if (asked)
                return fail(MX_ERR_WORKSPACE, "split %d needs a workspace of %zu bytes, %zu given", S, need,
                            workspace ? ws_bytes : size_t(0));
            S = 1;
        }
        if (S > 1) {
            if ((st = check_device_ptr(workspace, "workspace")) != MX_OK) return st;
            if (!aligned16(workspace)) return fail(MX_ERR_ALIGNMENT, "workspace must be 16-byte aligned");
        }
        e = mx::launch_gemm_tc2(*L, blob, Aq, s_a, M, Y, ldy, ag, S, S > 1 ? static_cast<float*>(workspace) : nullptr,
                                opts ? opts->debug_partials : nullptr, opts ? opts->status : nullptr, timeout_ns,
                                opts ? opts->test_stall : 0, s);
        if (e != cudaSuccess) return cuda_fail(e, "pair tensor-core GEMM launch");
        return MX_OK;
    }
    return fail(MX_ERR_INVALID_ARG, "unknown GEMM path %d", path);
}

namespace {

size_t align16(size_t v) { return (v + 15) & ~size_t(15); }

int x_bytes(mx_dtype xdt) { return xdt == MX_F16 ? 2 : 4; }

bool linear_fused(const mx_layout* L, int M, mx_dtype xdt, const mx_gemm_opts* opts);

// mx_linear's scratch: Aq | s_a | (256-byte aligned) the GEMM's own scratch when
// with_gemm; 0 when one kernel does the whole step
size_t linear_aq_sa_bytes(const mx_layout* L, int M, const mx_gemm_opts* opts) {
    return align16(size_t(M) * L->K) + align16(size_t(2) * M * scales_per_token(L, opts));
}
size_t linear_ws_bytes(const mx_layout* L, int M, mx_dtype xdt, const mx_gemm_opts* opts, bool with_gemm) {
    if (M == 0 || linear_fused(L, M, xdt, opts)) return 0;
    const size_t base = linear_aq_sa_bytes(L, M, opts);
    const size_t g = with_gemm ? gemm_ws_bytes(L, M, opts) : 0;
    return g ? ((base + 255) & ~size_t(255)) + g : base;
}

bool linear_fused(const mx_layout* L, int M, mx_dtype xdt, const mx_gemm_opts* opts) {
    const int path = choose_path(L, M, opts);
    if (path == 3) return mx::plan_rows(*L, M).ok;
    if (path != 1 || !mx::decode_can_fuse(*L, M, xdt)) return false;
    const mx::DecodePlan p = mx::plan_decode(*L, M, opts ? opts->split : 0, x_bytes(xdt));
    return p.ok && p.mt <= mx::kMaxFusedTokens;
}

}  // namespace

mx_status mx_saliency(const void* W, mx_dtype wdtype, int64_t ldw, const void* G, mx_dtype gdtype, int64_t ldg,
                      int N, int K, int group, float* S, void* stream) {
    if (N < 0 || K <= 0) return fail(MX_ERR_INVALID_ARG, "N=%d K=%d", N, K);
    if (group != 64 && group != 128) return fail(MX_ERR_UNSUPPORTED, "group=%d: 64 or 128", group);
    if (K % group != 0) return fail(MX_ERR_INVALID_ARG, "K=%d is not a multiple of the group %d", K, group);
    if (ldw < K || ldg < K) return fail(MX_ERR_INVALID_ARG, "ldw=%lld ldg=%lld < K=%d", (long long)ldw,
                                        (long long)ldg, K);
    for (mx_dtype t : {wdtype, gdtype})
        if (t != MX_F32 && t != MX_F16) return fail(MX_ERR_INVALID_ARG, "bad dtype %d", int(t));
    if (N == 0) return MX_OK;
    mx_status st;
    if ((st = check_device_ptr(W, "W")) != MX_OK) return st;
    if ((st = check_device_ptr(G, "G")) != MX_OK) return st;
    if ((st = check_device_ptr(S, "S")) != MX_OK) return st;
    cudaError_t e = mx::launch_saliency(W, wdtype, ldw, G, gdtype, ldg, N, K, group, S, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? MX_OK : cuda_fail(e, "saliency launch");
}

mx_status mx_select_top_workspace_size(int64_t n, size_t* bytes) {
    if (bytes == nullptr) return fail(MX_ERR_INVALID_ARG, "bytes is NULL");
    if (n < 0 || n > int64_t(0xFFFFFFFFu)) return fail(MX_ERR_INVALID_ARG, "n=%lld", (long long)n);
    *bytes = mx::select_workspace_bytes();
    return MX_OK;
}

mx_status mx_select_top(const float* S, int64_t n, int64_t n_top, uint8_t* is8, void* workspace, size_t ws_bytes,
                        void* stream) {
    if (n < 0 || n > int64_t(0xFFFFFFFFu)) return fail(MX_ERR_INVALID_ARG, "n=%lld", (long long)n);
    if (n_top < 0 || n_top > n) return fail(MX_ERR_INVALID_ARG, "n_top=%lld of %lld", (long long)n_top, (long long)n);
    if (n == 0) return MX_OK;
    mx_status st;
    if ((st = check_device_ptr(S, "S")) != MX_OK) return st;
    if ((st = check_device_ptr(is8, "is8")) != MX_OK) return st;
    if (workspace == nullptr || ws_bytes < mx::select_workspace_bytes())
        return fail(MX_ERR_WORKSPACE, "workspace of %zu bytes needed", mx::select_workspace_bytes());
    if ((st = check_device_ptr(workspace, "workspace")) != MX_OK) return st;
    if (!aligned16(workspace)) return fail(MX_ERR_ALIGNMENT, "workspace must be 16-byte aligned");
    cudaError_t e = mx::launch_select_top(S, n, n_top, is8, workspace, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? MX_OK : cuda_fail(e, "select_top launch");
}

// ---------------------------------------------------------------- block-wise bit widths
namespace {

constexpr uint32_t kBwMagic = 0x5742584Du;    // "MXBW"
constexpr uint32_t kBwVersion = 1;
constexpr uint64_t kBwHeaderBytes = 64;

// the block offsets (16-byte units from the codes) of a layer, and their end
mx_status bw_geometry(int N, int K, const uint8_t table[4], const uint8_t* meta, mx_bw_layout* L,
                      std::vector<uint32_t>* offsets) {
    if (N < 1 || K < MX_BW_BLOCK_COLS || K % MX_BW_BLOCK_COLS)
        return fail(MX_ERR_INVALID_ARG, "N=%d K=%d: N >= 1, K a positive multiple of 128", N, K);
    if (table == nullptr || meta == nullptr) return fail(MX_ERR_INVALID_ARG, "table or meta is NULL");
    for (int c = 0; c < 4; ++c)
        if (table[c] < 1 || table[c] > 8) return fail(MX_ERR_INVALID_ARG, "width table[%d]=%d outside 1..8", c, table[c]);
    mx_bw_layout l;
    memset(&l, 0, sizeof l);
    l.N = N;
    l.K = K;
    l.NB = (N + MX_BW_BLOCK_ROWS - 1) / MX_BW_BLOCK_ROWS;
    l.KB = K / MX_BW_BLOCK_COLS;
    memcpy(l.table, table, 4);
    const int64_t nblk = int64_t(l.NB) * l.KB;
    if (offsets) offsets->assign(size_t(nblk) + 1, 0u);
    uint64_t units = 0;                          // 16-byte units
    for (int64_t bi = 0; bi < nblk; ++bi) {
        if (offsets) (*offsets)[size_t(bi)] = uint32_t(units);
        const int rb = int(bi / l.KB);
        const int rows = std::min(MX_BW_BLOCK_ROWS, N - rb * MX_BW_BLOCK_ROWS);
        const int b = table[(meta[bi >> 2] >> (2 * (bi & 3))) & 3];
        units += uint64_t(rows) * uint64_t(b);   // 16 b bytes per row
        if (units > 0xFFFFFFFFull) return fail(MX_ERR_UNSUPPORTED, "codes larger than 64 GiB");
    }
    if (offsets) (*offsets)[size_t(nblk)] = uint32_t(units);
    l.code_bytes = units * 16;
    l.off_meta = kBwHeaderBytes;
    l.off_offsets = align16(l.off_meta + uint64_t((nblk + 3) / 4));
    l.off_scales = align16(l.off_offsets + 4 * uint64_t(nblk + 1));
    l.off_zeros = align16(l.off_scales + 2 * uint64_t(N) * l.KB);
    l.off_codes = align16(l.off_zeros + uint64_t(N) * l.KB);
    l.total_bytes = l.off_codes + l.code_bytes;
    *L = l;
    return MX_OK;
}

// a layout's fields agree with one another (as mx_bw_layout_init made them)
mx_status bw_check(const mx_bw_layout* L) {
    if (L == nullptr) return fail(MX_ERR_INVALID_ARG, "layout is NULL");
    if (L->N < 1 || L->K < MX_BW_BLOCK_COLS || L->K % MX_BW_BLOCK_COLS ||
        L->NB != (L->N + MX_BW_BLOCK_ROWS - 1) / MX_BW_BLOCK_ROWS || L->KB != L->K / MX_BW_BLOCK_COLS)
        return fail(MX_ERR_INVALID_ARG, "layout geometry is inconsistent");
    for (int c = 0; c < 4; ++c)
        if (L->table[c] < 1 || L->table[c] > 8) return fail(MX_ERR_INVALID_ARG, "layout width table is invalid");
    const uint64_t nblk = uint64_t(L->NB) * L->KB;
    if (L->off_meta != kBwHeaderBytes || L->off_offsets != align16(L->off_meta + (nblk + 3) / 4) ||
        L->off_scales != align16(L->off_offsets + 4 * (nblk + 1)) ||
        L->off_zeros != align16(L->off_scales + 2 * uint64_t(L->N) * L->KB) ||
        L->off_codes != align16(L->off_zeros + uint64_t(L->N) * L->KB) ||
        L->total_bytes != L->off_codes + L->code_bytes || L->code_bytes % 16 ||
        L->code_bytes < uint64_t(L->N) * L->K / 8 || L->code_bytes > uint64_t(L->N) * L->K)
        return fail(MX_ERR_INVALID_ARG, "layout offsets are inconsistent");
    return MX_OK;
}

}  // namespace

mx_status mx_bw_layout_init(int N, int K, const uint8_t table[4], const uint8_t* meta, mx_bw_layout* out) {
    if (out == nullptr) return fail(MX_ERR_INVALID_ARG, "out is NULL");
    return bw_geometry(N, K, table, meta, out, nullptr);
}

mx_status mx_bw_pack(const mx_bw_layout* L, const uint8_t* meta, const void* W, mx_dtype wdtype, int64_t ldw,
                     void* blob, void* stream) {
    mx_status st;
    if ((st = bw_check(L)) != MX_OK) return st;
    mx_bw_layout ref;
    std::vector<uint32_t> offsets;
    if ((st = bw_geometry(L->N, L->K, L->table, meta, &ref, &offsets)) != MX_OK) return st;
    if (memcmp(&ref, L, sizeof ref) != 0) return fail(MX_ERR_INVALID_ARG, "layout was not made from this meta");
    if (wdtype != MX_F32 && wdtype != MX_F16) return fail(MX_ERR_INVALID_ARG, "bad dtype %d", int(wdtype));
    if (ldw < L->K) return fail(MX_ERR_INVALID_ARG, "ldw=%lld < K=%d", (long long)ldw, L->K);
    if ((st = check_device_ptr(W, "W")) != MX_OK) return st;
    if ((st = check_device_ptr(blob, "blob")) != MX_OK) return st;
    if (!aligned16(blob)) return fail(MX_ERR_ALIGNMENT, "blob must be 16-byte aligned");
    // header, block codes and offsets, staged on the host and copied in the stream
    std::vector<uint8_t> head(size_t(L->off_scales), 0);
    const uint32_t h[6] = {kBwMagic, kBwVersion, uint32_t(L->N), uint32_t(L->K),
                           uint32_t(L->table[0]) | uint32_t(L->table[1]) << 8 | uint32_t(L->table[2]) << 16 |
                               uint32_t(L->table[3]) << 24,
                           uint32_t(L->code_bytes >> 4)};
    memcpy(head.data(), h, sizeof h);
    const uint64_t nblk = uint64_t(L->NB) * L->KB;
    memcpy(head.data() + L->off_meta, meta, size_t((nblk + 3) / 4));
    memcpy(head.data() + L->off_offsets, offsets.data(), offsets.size() * sizeof(uint32_t));
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemsetAsync(blob, 0, size_t(L->total_bytes), s);
    if (e == cudaSuccess) e = cudaMemcpyAsync(blob, head.data(), head.size(), cudaMemcpyHostToDevice, s);
    // a pageable source: the call returns once the bytes are staged, so `head` may go
    if (e == cudaSuccess) e = mx::launch_bw_pack(*L, W, wdtype, ldw, static_cast<uint8_t*>(blob), s);
    return e == cudaSuccess ? MX_OK : cuda_fail(e, "bw pack");
}

mx_status mx_bw_gemm(const mx_bw_layout* L, const void* blob, const int8_t* Aq, const void* s_a, int M, void* Y,
                     int64_t ldy, int32_t* partials, void* stream) {
    mx_status st;
    if ((st = bw_check(L)) != MX_OK) return st;
    if (M < 0) return fail(MX_ERR_INVALID_ARG, "M=%d", M);
    if (M > 65535 * 8) return fail(MX_ERR_UNSUPPORTED, "M=%d: at most %d tokens per call", M, 65535 * 8);
    if (ldy < L->N) return fail(MX_ERR_INVALID_ARG, "ldy=%lld < N=%d", (long long)ldy, L->N);
    if (M == 0) return MX_OK;
    if ((st = check_device_ptr(blob, "blob")) != MX_OK) return st;
    if ((st = check_device_ptr(Aq, "Aq")) != MX_OK) return st;
    if ((st = check_device_ptr(s_a, "s_a")) != MX_OK) return st;
    if ((st = check_device_ptr(Y, "Y")) != MX_OK) return st;
    if (partials && (st = check_device_ptr(partials, "partials")) != MX_OK) return st;
    if (!aligned16(blob) || !aligned16(Aq)) return fail(MX_ERR_ALIGNMENT, "blob and Aq must be 16-byte aligned");
    if (reinterpret_cast<uintptr_t>(s_a) % 2 || reinterpret_cast<uintptr_t>(Y) % 2)
        return fail(MX_ERR_ALIGNMENT, "s_a and Y must be 2-byte aligned");
    cudaError_t e = mx::launch_bw_gemm(*L, static_cast<const uint8_t*>(blob), Aq, static_cast<const __half*>(s_a), M,
                                       static_cast<__half*>(Y), ldy, partials, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? MX_OK : cuda_fail(e, "bw gemm");
}

mx_status mx_copy_mapped(void* dst, const void* src, size_t bytes, void* stream) {
    const void *d = nullptr, *s = nullptr;
    bool dh = false, sh = false;
    mx_status st = mapped_ptr(dst, "dst", &d, &dh);
    if (st != MX_OK) return st;
    if ((st = mapped_ptr(src, "src", &s, &sh)) != MX_OK) return st;
    const uintptr_t a0 = reinterpret_cast<uintptr_t>(d), b0 = reinterpret_cast<uintptr_t>(s);
    if (bytes && a0 < b0 + bytes && b0 < a0 + bytes) return fail(MX_ERR_INVALID_ARG, "dst and src overlap");
    cudaError_t e = mx::launch_copy_mapped(const_cast<void*>(d), s, bytes, sh, dh, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? MX_OK : cuda_fail(e, "copy_mapped launch");
}

mx_status mx_linear_workspace_size(const mx_layout* L, int M, mx_dtype xdtype, const mx_gemm_opts* opts,
                                   size_t* bytes) {
    mx_status st = check_layout(L);
    if (st != MX_OK) return st;
    if (bytes == nullptr) return fail(MX_ERR_INVALID_ARG, "bytes is NULL");
    if (M < 0) return fail(MX_ERR_INVALID_ARG, "M=%d", M);
    if (xdtype != MX_F32 && xdtype != MX_F16) return fail(MX_ERR_INVALID_ARG, "bad xdtype %d", int(xdtype));
    if ((st = check_act_group(L, opts)) != MX_OK) return st;
    *bytes = linear_ws_bytes(L, M, xdtype, opts, true);
    return MX_OK;
}

mx_status mx_linear(const mx_layout* L, const void* blob, const void* X, mx_dtype xdtype, int M,
                    int64_t ldx, uint16_t* Y, int64_t ldy, void* workspace, size_t ws_bytes,
                    const mx_gemm_opts* opts, void* stream) {
    mx_status st = check_layout(L);
    if (st != MX_OK) return st;
    if (xdtype != MX_F32 && xdtype != MX_F16) return fail(MX_ERR_INVALID_ARG, "bad xdtype %d", int(xdtype));
    if (M < 0) return fail(MX_ERR_INVALID_ARG, "M=%d", M);
    if (ldx < L->K) return fail(MX_ERR_INVALID_ARG, "ldx=%lld < K=%d", (long long)ldx, L->K);
    if (ldy < L->N) return fail(MX_ERR_INVALID_ARG, "ldy=%lld < N=%d", (long long)ldy, L->N);
    if (M == 0) return MX_OK;
    if (M > 65535) return fail(MX_ERR_UNSUPPORTED, "M=%d above 65535", M);
    const int esz = xdtype == MX_F16 ? 2 : 4;
    if ((st = check_act_group(L, opts)) != MX_OK) return st;
    if ((st = check_device_ptr(X, "X")) != MX_OK) return st;
    if (!aligned16(X) || (ldx * esz) % 16 != 0) return fail(MX_ERR_ALIGNMENT, "X and every X row must be 16-byte aligned");
    const int ag = act_group_of(opts);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (linear_fused(L, M, xdtype, opts)) {
        if ((st = check_device_ptr(blob, "blob")) != MX_OK) return st;
        if ((st = check_device_ptr(Y, "Y")) != MX_OK) return st;
        if (!aligned16(blob)) return fail(MX_ERR_ALIGNMENT, "blob must be 16-byte aligned");
        if (opts && opts->debug_partials && (st = check_device_ptr(opts->debug_partials, "debug_partials")) != MX_OK)
            return st;
        if (opts && opts->status && (st = check_device_ptr(opts->status, "status")) != MX_OK) return st;
        if (choose_path(L, M, opts) == 3) {
            cudaError_t e = mx::launch_gemm_rows(*L, blob, nullptr, nullptr, X, xdtype, ldx, M, Y, ldy,
                                                 mx::plan_rows(*L, M), ag,
                                                 opts ? opts->debug_partials : nullptr,
                                                 opts ? opts->status : nullptr, s);
            if (e != cudaSuccess) return cuda_fail(e, "row decode GEMM launch");
            return MX_OK;
        }
        if (opts && opts->split > 8) return fail(MX_ERR_UNSUPPORTED, "split=%d above the cluster limit 8", opts->split);
        mx::DecodePlan plan = mx::plan_decode(*L, M, opts ? opts->split : 0, x_bytes(xdtype));
        cudaError_t e = mx::launch_gemm_decode_fused(*L, blob, X, xdtype, ldx, M, Y, ldy, plan, ag,
                                                     opts ? opts->debug_partials : nullptr,
                                                     opts ? opts->status : nullptr, s);
        if (e != cudaSuccess) return cuda_fail(e, "fused decode GEMM launch");
        return MX_OK;
    }
    const size_t need = linear_aq_sa_bytes(L, M, opts);
    if (workspace == nullptr || ws_bytes < need)
        return fail(MX_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", need, workspace ? ws_bytes : size_t(0));
    if ((st = check_device_ptr(workspace, "workspace")) != MX_OK) return st;
    if (!aligned16(workspace)) return fail(MX_ERR_ALIGNMENT, "workspace must be 16-byte aligned");
    int8_t* Aq = static_cast<int8_t*>(workspace);
    uint16_t* s_a = reinterpret_cast<uint16_t*>(static_cast<uint8_t*>(workspace) + align16(size_t(M) * L->K));
    if ((st = mx_quant_act_grouped(X, xdtype, M, L->K, ldx, ag, Aq, s_a, stream)) != MX_OK) return st;
    // the rest of the workspace (from a 256-byte boundary) is the GEMM's scratch
    const size_t off = (need + 255) & ~size_t(255);
    void* gws = ws_bytes > off ? static_cast<uint8_t*>(workspace) + off : nullptr;
    return mx_gemm(L, blob, Aq, s_a, M, Y, ldy, gws, gws ? ws_bytes - off : 0, opts, stream);
}

// ---------------------------------------------------------------------------
// mx_linear_noalloc: the scratch of mx_linear's two-kernel path in a fixed
// device array instead of a caller workspace.

}  // extern "C"

static __device__ __align__(256) uint8_t g_noalloc_scratch[MX_NOALLOC_SCRATCH_BYTES];

namespace {

constexpr int kNoAllocDevices = 64;
struct NoAllocSlot {
    CUcontext ctx;     // the context the address belongs to
    void* addr;
};
NoAllocSlot g_noalloc[kNoAllocDevices] = {};
std::mutex g_noalloc_mu;

using CtxGetCurrentFn = CUresult (*)(CUcontext*);

// the driver's cuCtxGetCurrent, found once through the runtime
CtxGetCurrentFn ctx_get_current_fn() {
    static CtxGetCurrentFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<CtxGetCurrentFn>(p);
        cudaGetLastError();
    });
    return fn;
}

// The array's address in the current device's context.  It is looked up once per
// device and context: the first call on a device (and the first after that device's
// primary context was torn down and made again, by cudaDeviceReset for example)
// does the lookup; later calls reuse it.
mx_status noalloc_scratch(void** addr) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev < 0 || dev >= kNoAllocDevices)
        return fail(MX_ERR_UNSUPPORTED, "device %d beyond the %d this call tracks", dev, kNoAllocDevices);
    // cudaSetDevice makes the device's primary context current (creating it if needed)
    if ((e = cudaSetDevice(dev)) != cudaSuccess) return cuda_fail(e, "cudaSetDevice");
    CUcontext ctx = nullptr;
    CtxGetCurrentFn get = ctx_get_current_fn();
    if (get == nullptr || get(&ctx) != CUDA_SUCCESS || ctx == nullptr)
        return fail(MX_ERR_CUDA, "no current CUDA context on device %d", dev);
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    NoAllocSlot& slot = g_noalloc[dev];
    if (slot.addr == nullptr || slot.ctx != ctx) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) {
            cudaGetLastError();
            return cuda_fail(e, "cudaGetSymbolAddress of the scratch array");
        }
        slot.ctx = ctx;
        slot.addr = p;
    }
    *addr = slot.addr;
    return MX_OK;
}

}  // namespace

extern "C" {

mx_status mx_linear_noalloc(const mx_layout* L, const void* blob, const void* X, mx_dtype xdtype, int M,
                            int64_t ldx, uint16_t* Y, int64_t ldy, const mx_gemm_opts* opts,
                            void* stream) {
    size_t need = 0;
    mx_status st = mx_linear_workspace_size(L, M, xdtype, opts, &need);
    if (st != MX_OK) return st;
    // the limit holds for Aq and s_a; split sums of the tensor-core path use the rest of
    // the array when they fit, else the GEMM runs unsplit
    need = linear_ws_bytes(L, M, xdtype, opts, false);
    if (need > MX_NOALLOC_SCRATCH_BYTES)
        return fail(MX_ERR_WORKSPACE, "%zu bytes of scratch needed, the fixed array holds %u", need,
                    MX_NOALLOC_SCRATCH_BYTES);
    void* ws = nullptr;
    if (need > 0 && (st = noalloc_scratch(&ws)) != MX_OK) return st;
    return mx_linear(L, blob, X, xdtype, M, ldx, Y, ldy, ws, need > 0 ? size_t(MX_NOALLOC_SCRATCH_BYTES) : 0,
                     opts, stream);
}

}  // extern "C"
