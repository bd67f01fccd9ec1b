"""The C-ABI library loads and exports every declared entry point; host-only logic.

None of these tests launches a kernel or needs a GPU: they exercise the packed
layout geometry, header validation and the argument checks that fail before any
CUDA call is made.
"""
import ctypes
import os
import re
import struct

import pytest

from mixed_precision_quantized_mx_b200 import binding as mx

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    text = "".join(open(os.path.join(ROOT, "include", f)).read()
                   for f in sorted(os.listdir(os.path.join(ROOT, "include"))) if f.endswith(".h"))
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:mx_status|int|const char\*)\s+(mx_\w+)\s*\(", text, flags=re.M)))


@pytest.fixture(scope="module")
def lib():
    from mixed_precision_quantized_mx_b200 import build
    build.build()
    return mx.lib()


def test_every_declared_symbol_is_exported(lib):
    syms = declared_symbols()
    assert len(syms) >= 8
    for s in syms:
        assert hasattr(lib, s), s
    assert sorted(mx.EXPORTED) == syms          # the binding mirrors the header names


def test_version(lib):
    assert mx.mx_version() == 2


def _expected_total(N, K, g, n8):
    a = lambda v: (v + 255) // 256 * 256
    t8, t4 = -(-n8 // 128), -(-(N - n8) // 128)
    G = K // g
    off = 256
    off = a(off + (t8 + t4) * 128 * 4)
    off = a(off + t8 * 128 * G * 2)
    off = a(off + t8 * 128 * K)
    off = a(off + t4 * 128 * G * 2)
    off = a(off + t4 * 128 * G)
    off = a(off + t4 * 128 * K // 2)
    return off


@pytest.mark.parametrize("N,K,g,n8", [(512, 512, 128, 51), (4096, 4096, 128, 410),
                                      (300, 256, 64, 37), (128, 128, 128, 0), (128, 128, 128, 128),
                                      (28672, 8192, 128, 2867)])
def test_layout_geometry(lib, N, K, g, n8):
    L = mx.mx_layout_init(N, K, g, n8)
    assert (L.N, L.K, L.group, L.n8, L.n4, L.G) == (N, K, g, n8, N - n8, K // g)
    assert (L.t8, L.t4, L.kblocks) == (-(-n8 // 128), -(-(N - n8) // 128), K // 128)
    assert L.total_bytes == _expected_total(N, K, g, n8)
    offs = [L.off_rowmap, L.off_scales8, L.off_codes8, L.off_scales4, L.off_zeros4, L.off_codes4]
    assert offs == sorted(offs) and all(o % 256 == 0 for o in offs)
    assert L.off_codes4 + L.t4 * 128 * K // 2 <= L.total_bytes


@pytest.mark.parametrize("args,status", [
    ((0, 128, 128, 0), 1), ((16, 128, 128, 17), 1), ((16, 128, 128, -1), 1),
    ((16, 128, 32, 0), 2), ((16, 192, 64, 0), 2), ((16, 100, 128, 0), 2)])
def test_layout_rejects(lib, args, status):
    with pytest.raises(mx.MXError) as e:
        mx.mx_layout_init(*args)
    assert e.value.status == status
    assert mx.lib().mx_last_error().decode()


def test_header_round_trip_and_corruption(lib):
    hdr = struct.pack("<6I", 0x4B50584D, 1, 4096, 4096, 128, 410) + bytes(256 - 24)
    L = mx.mx_layout_from_header(hdr)
    ref = mx.mx_layout_init(4096, 4096, 128, 410)
    assert bytes(L) == bytes(ref)
    bad = [struct.pack("<6I", 0x12345678, 1, 4096, 4096, 128, 410),
           struct.pack("<6I", 0x4B50584D, 9, 4096, 4096, 128, 410),
           struct.pack("<6I", 0x4B50584D, 1, 4096, 4096, 96, 410),
           struct.pack("<6I", 0x4B50584D, 1, 4096, 4096, 128, 5000)]
    for h in bad:
        with pytest.raises(mx.MXError) as e:
            mx.mx_layout_from_header(h + bytes(256 - 24))
        assert e.value.status == 6
    with pytest.raises(mx.MXError) as e:
        mx.mx_layout_from_header(hdr[:100])
    assert e.value.status == 6


def test_host_argument_checks_before_any_launch(lib):
    P = ctypes.c_void_p
    # quant_act: K not a multiple of 8 / bad dtype / negative M
    assert lib.mx_quant_act(None, 1, 4, 12, 12, None, None, None) == 2
    assert lib.mx_quant_act(None, 7, 4, 16, 16, None, None, None) == 1
    assert lib.mx_quant_act(None, 1, -1, 16, 16, None, None, None) == 1
    assert lib.mx_quant_act(None, 1, 0, 16, 16, None, None, None) == 0      # M = 0: no-op
    L = mx.mx_layout_init(256, 256, 128, 10)
    # a layout edited after init is refused
    L2 = mx.mx_layout_init(256, 256, 128, 10)
    L2.t8 = 7
    o = mx.GemmOpts(0, 0, None, None)
    assert lib.mx_gemm(ctypes.byref(L2), None, None, None, 1, None, 256, None, 0, ctypes.byref(o), None) == 1
    # ldy < N, NULL layout
    assert lib.mx_gemm(ctypes.byref(L), None, None, None, 1, None, 100, None, 0, ctypes.byref(o), None) == 1
    assert lib.mx_gemm(None, None, None, None, 1, None, 256, None, 0, ctypes.byref(o), None) == 1
    # M = 0 is a no-op that touches nothing
    assert lib.mx_gemm(ctypes.byref(L), None, None, None, 0, None, 256, None, 0, ctypes.byref(o), None) == 0
    n = ctypes.c_size_t(123)
    assert lib.mx_gemm_workspace_size(ctypes.byref(L), 0, ctypes.byref(o), ctypes.byref(n)) == 0
    assert n.value == 0


def test_gemm_workspace_and_dispatch_on_m(lib):
    L = mx.mx_layout_init(4096, 4096, 128, 410)
    for M in (1, 8, 2048):
        assert mx.mx_gemm_workspace_size(L, M) == 0
    # 33 row tiles of 128 rows: at 9..128 tokens the decode tensor-core path splits K
    # four ways (132 units for 148 SMs) and sums the splits in a workspace
    a256 = lambda v: (v + 255) // 256 * 256
    for M, S in ((16, 4), (17, 4), (100, 4)):
        assert mx.mx_gemm_workspace_size(L, M) == a256(S * M * 4096 * 4)
    assert mx.mx_gemm_workspace_size(L, 17, split=3) == a256(3 * 17 * 4096 * 4)
    assert mx.mx_gemm_workspace_size(L, 17, path=mx.PATH_TENSOR) == 0     # the one-CTA kernel
    assert mx.mx_gemm_workspace_size(L, 17, split=1) == 0
    # 17 CTA pairs at 129 tokens: one token tile leaves pairs idle, so path 4 splits K
    n129 = mx.mx_gemm_workspace_size(L, 129)
    assert n129 > 0 and n129 % (129 * 4096 * 4) == 0 and n129 // (129 * 4096 * 4) in range(2, 9)
    assert mx.mx_gemm_select_path(L, 1) == mx.PATH_ROWS          # short K, M <= 4, one wave
    assert mx.mx_gemm_select_path(L, 4) == mx.PATH_ROWS
    assert mx.mx_gemm_select_path(L, 5) == mx.PATH_SPLITK
    assert mx.mx_gemm_select_path(L, 8) == mx.PATH_SPLITK
    assert mx.mx_gemm_select_path(L, 1, split=2) == mx.PATH_SPLITK   # a split asks for clusters
    assert mx.mx_gemm_select_path(L, 16, split=2) == mx.PATH_SPLITK
    assert mx.mx_gemm_select_path(L, 9) == mx.PATH_TC_DECODE       # decode tensor cores, one CTA per tile
    assert mx.mx_gemm_select_path(L, 16) == mx.PATH_TC_DECODE
    assert mx.mx_gemm_select_path(L, 128) == mx.PATH_TC_DECODE
    assert mx.mx_gemm_select_path(L, 129) == mx.PATH_PAIR          # tensor cores on CTA pairs
    # prefill M: 256-token pair tiles once they give every one of the 74 pairs a unit
    # (17 row-tile pairs x 5 token tiles of 256 = 85 units at M = 1280)
    assert mx.mx_gemm_select_path(L, 1024) == mx.PATH_PAIR
    assert mx.mx_gemm_select_path(L, 1280) == mx.PATH_PAIR256
    assert mx.mx_gemm_select_path(L, 2048) == mx.PATH_PAIR256
    assert mx.mx_gemm_select_path(L, 2048, split=2) == mx.PATH_PAIR      # a K split is path 4's
    assert mx.mx_gemm_workspace_size(L, 2048, path=mx.PATH_PAIR256) == 0
    assert mx.mx_gemm_select_path(L, 1, path=mx.PATH_TENSOR) == mx.PATH_TENSOR   # asked for
    # 16 tokens of a 64K-column activation slice cannot be staged per cluster: tensor cores
    Lbig = mx.mx_layout_init(1024, 65536, 128, 102)
    assert mx.mx_gemm_select_path(Lbig, 16) == mx.PATH_TC_DECODE
    # the row path needs K <= 4096 and one wave of CTAs
    assert mx.mx_gemm_select_path(mx.mx_layout_init(4096, 8192, 128, 410), 1) == mx.PATH_SPLITK
    assert mx.mx_gemm_select_path(mx.mx_layout_init(14336, 4096, 128, 1434), 1) == mx.PATH_SPLITK


@pytest.mark.parametrize("K,N,splits", [
    # the fastest K split measured on a B200 for each shape at 16, 64 and 128 tokens (path 6,
    # splits 1..16 swept, 10 % 8-bit rows, group 128): the cost model must pick it
    (4096, 4096, (4, 4, 4)),        # Llama-3-8B q/o
    (4096, 14336, (1, 1, 1)),       # 8B up
    (14336, 4096, (4, 4, 4)),       # 8B down
    (8192, 28672, (1, 1, 1)),       # 70B up
    (28672, 8192, (2, 2, 2)),       # 70B down
])
def test_decode_split_model_picks_the_measured_fastest_split(lib, K, N, splits):
    L = mx.mx_layout_init(N, K, 128, int(0.1 * N + 0.5))
    for M, S in zip((16, 64, 128), splits):
        assert mx.mx_gemm_select_path(L, M) == mx.PATH_TC_DECODE
        ws = mx.mx_gemm_workspace_size(L, M)
        got = ws // (M * N * 4) if ws else 1
        assert got == S, (K, N, M, got, S)


def test_linear_workspace_follows_the_fused_decode_rule(lib):
    L = mx.mx_layout_init(4096, 4096, 128, 410)
    import torch
    # decode-sized M with a small activation row: one fused kernel, no scratch
    for M in (1, 2, 3, 4):
        assert mx.mx_linear_workspace_size(L, M, torch.float16) == 0
        assert mx.mx_linear_workspace_size(L, M, torch.float32) == 0
    assert mx.mx_linear_workspace_size(L, 0, torch.float16) == 0
    # more tokens, the tensor-core path, or a forced path: Aq + s_a, 16-byte rounded, then
    # (from a 256-byte boundary) the GEMM's own workspace when it splits K
    a16 = lambda v: (v + 15) // 16 * 16
    a256 = lambda v: (v + 255) // 256 * 256
    for M in (5, 16, 17, 2048):
        g = mx.mx_gemm_workspace_size(L, M)
        base = a16(M * 4096) + a16(2 * M)
        assert mx.mx_linear_workspace_size(L, M, torch.float16) == (a256(base) + g if g else base)
    assert mx.mx_linear_workspace_size(L, 1, torch.float16, path=mx.PATH_TENSOR) == 4096 + 16
    # 4 fp32 rows of 8192 columns exceed the 64 KB the fused kernel stages
    Lw = mx.mx_layout_init(1024, 8192, 128, 102)
    assert mx.mx_linear_workspace_size(Lw, 2, torch.float32) == 0
    assert mx.mx_linear_workspace_size(Lw, 4, torch.float32) == a16(4 * 8192) + 16


def test_linear_host_argument_checks(lib):
    L = mx.mx_layout_init(256, 256, 128, 10)
    o = mx.GemmOpts(0, 0, None, None)
    n = ctypes.c_size_t(0)
    assert lib.mx_linear_workspace_size(ctypes.byref(L), 1, 5, ctypes.byref(o), ctypes.byref(n)) == 1
    assert lib.mx_linear_workspace_size(ctypes.byref(L), -1, 1, ctypes.byref(o), ctypes.byref(n)) == 1
    assert lib.mx_linear_workspace_size(ctypes.byref(L), 1, 1, ctypes.byref(o), None) == 1
    args = lambda M, ldx, ldy, xdt=1: (ctypes.byref(L), None, None, xdt, M, ldx, None, ldy, None, 0,
                                       ctypes.byref(o), None)
    assert lib.mx_linear(*args(1, 100, 256)) == 1           # ldx < K
    assert lib.mx_linear(*args(1, 256, 100)) == 1           # ldy < N
    assert lib.mx_linear(*args(1, 256, 256, xdt=9)) == 1    # bad dtype
    assert lib.mx_linear(*args(-2, 256, 256)) == 1
    assert lib.mx_linear(*args(0, 256, 256)) == 0           # M = 0: no-op


def test_noalloc_scratch_limit_is_checked_before_any_launch(lib):
    text = open(os.path.join(ROOT, "include", "mx.h")).read()
    m = re.search(r"#define MX_NOALLOC_SCRATCH_BYTES \((\d+)u << (\d+)\)", text)
    assert m and int(m.group(1)) << int(m.group(2)) == mx.NOALLOC_SCRATCH_BYTES
    L = mx.mx_layout_init(4096, 4096, 128, 410)
    o = mx.GemmOpts(0, 0, None, None)
    # 1025 tokens of 4096 codes need 4 MiB + 16 B + 2064 B: refused with no pointer touched
    M = mx.NOALLOC_SCRATCH_BYTES // 4096 + 1
    assert mx.mx_linear_workspace_size(L, M) > mx.NOALLOC_SCRATCH_BYTES
    assert lib.mx_linear_noalloc(ctypes.byref(L), None, None, 1, M, 4096, None, 4096,
                                 ctypes.byref(o), None) == 7
    assert "fixed array" in lib.mx_last_error().decode()
    assert lib.mx_linear_noalloc(ctypes.byref(L), None, None, 1, 0, 4096, None, 4096,
                                 ctypes.byref(o), None) == 0          # M = 0: no-op


def test_group_wise_activation_options_checked_on_the_host(lib):
    L = mx.mx_layout_init(512, 1024, 128, 51)
    o = mx.GemmOpts(0, 0, None, None, 0, 0, 64)                      # act_group != weight group
    assert lib.mx_gemm(ctypes.byref(L), None, None, None, 2, None, 512, None, 0, ctypes.byref(o), None) == 2
    assert lib.mx_linear(ctypes.byref(L), None, None, 1, 2, 1024, None, 512, None, 0, ctypes.byref(o), None) == 2
    n = ctypes.c_size_t(0)
    assert lib.mx_linear_workspace_size(ctypes.byref(L), 8, 1, ctypes.byref(o), ctypes.byref(n)) == 2
    # the grouped quantizer: act_group 0, 64 or 128, dividing K
    assert lib.mx_quant_act_grouped(None, 1, 4, 1024, 1024, 32, None, None, None) == 2
    assert lib.mx_quant_act_grouped(None, 1, 4, 192, 192, 128, None, None, None) == 2
    assert lib.mx_quant_act_grouped(None, 1, 0, 1024, 1024, 128, None, None, None) == 0   # M = 0
    # a workspace for grouped scales holds [M][G] of them
    a16 = lambda v: (v + 15) // 16 * 16
    assert mx.mx_linear_workspace_size(L, 8, act_group=128) == a16(8 * 1024) + a16(2 * 8 * 8)
    assert mx.mx_linear_workspace_size(L, 8) == a16(8 * 1024) + a16(2 * 8)
    assert mx.mx_linear_workspace_size(L, 2, act_group=128) == 0                 # fused


def test_precision_search_argument_checks_before_any_launch(lib):
    # mx_saliency: group, divisibility, leading dimensions and dtypes are refused on the
    # host; no rows is a no-op.  None of these reaches a CUDA call.
    P = ctypes.c_void_p(16)
    S = ctypes.c_void_p(32)
    assert lib.mx_saliency(P, 0, 256, P, 0, 256, 4, 256, 96, S, None) == 2     # group 96
    assert lib.mx_saliency(P, 0, 256, P, 0, 256, 4, 200, 128, S, None) == 1    # K % group
    assert lib.mx_saliency(P, 0, 100, P, 0, 256, 4, 256, 128, S, None) == 1    # ldw < K
    assert lib.mx_saliency(P, 0, 256, P, 0, 255, 4, 256, 128, S, None) == 1    # ldg < K
    assert lib.mx_saliency(P, 7, 256, P, 0, 256, 4, 256, 128, S, None) == 1    # W dtype
    assert lib.mx_saliency(P, 0, 256, P, 2, 256, 4, 256, 128, S, None) == 1    # G dtype
    assert lib.mx_saliency(P, 0, 256, P, 0, 256, -1, 256, 128, S, None) == 1   # N < 0
    assert lib.mx_saliency(P, 0, 256, P, 0, 256, 0, 256, 128, S, None) == 0    # nothing to do
    # mx_select_top: the workspace is a fixed small size; counts are checked first
    nb = ctypes.c_size_t(0)
    assert lib.mx_select_top_workspace_size(1 << 20, ctypes.byref(nb)) == 0
    assert 0 < nb.value <= 4096 and nb.value % 16 == 0
    assert lib.mx_select_top_workspace_size(-1, ctypes.byref(nb)) == 1
    assert lib.mx_select_top_workspace_size(1 << 32, ctypes.byref(nb)) == 1
    assert lib.mx_select_top_workspace_size(5, None) == 1
    assert lib.mx_select_top(S, 10, 11, P, P, 4096, None) == 1                # n_top > n
    assert lib.mx_select_top(S, 10, -1, P, P, 4096, None) == 1
    assert lib.mx_select_top(S, -1, 0, P, P, 4096, None) == 1
    assert lib.mx_select_top(S, 1 << 32, 0, P, P, 4096, None) == 1            # index must fit 32 bits
    assert lib.mx_select_top(S, 0, 0, P, None, 0, None) == 0                  # nothing to do
