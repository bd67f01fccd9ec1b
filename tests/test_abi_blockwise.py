"""Host-only logic of the block-wise bit-width entry points (mx_blockwise.h): the
packed geometry against the oracle's count of code bits, and the argument checks
that fail before any CUDA call.  No kernel runs here.
"""
import ctypes

import numpy as np
import pytest

from mixed_precision_quantized_mx_b200 import binding as mx
from mixed_precision_quantized_mx_b200 import inputs


@pytest.fixture(scope="module")
def lib():
    from mixed_precision_quantized_mx_b200 import build
    build.build()
    return mx.lib()


@pytest.mark.parametrize("N,K,table", [(64, 128, [2, 3, 4, 8]), (200, 512, [1, 2, 6, 8]),
                                       (4096, 4096, [3, 4, 6, 8]), (1, 256, [8, 8, 8, 8])])
def test_geometry_matches_the_oracle_code_bits(lib, orc, N, K, table):
    rng = np.random.default_rng(N + K)
    codes = inputs.block_codes(rng, N, K)
    meta = orc.pack_block_codes(codes)
    L = mx.mx_bw_layout_init(N, K, table, meta)
    NB, KB = codes.shape
    assert (L.N, L.K, L.NB, L.KB) == (N, K, NB, KB) and list(L.table) == table
    # the codes hold exactly the blocks' bits: bits per weight minus the 2-bit metadata
    b = orc.pack_blockwise(np.zeros((N, K), np.float32), codes, table)
    assert L.code_bytes * 8 == round(orc.bits_per_weight(b) * N * K - 2 * NB * KB)
    # sections in order, 16-byte aligned, sized as documented
    offs = [L.off_meta, L.off_offsets, L.off_scales, L.off_zeros, L.off_codes]
    assert L.off_meta == 64 and all(o % 16 == 0 for o in offs) and offs == sorted(offs)
    assert L.off_offsets - L.off_meta >= (NB * KB + 3) // 4
    assert L.off_scales - L.off_offsets >= 4 * (NB * KB + 1)
    assert L.off_zeros - L.off_scales >= 2 * N * KB
    assert L.off_codes - L.off_zeros >= N * KB
    assert L.total_bytes == L.off_codes + L.code_bytes


def test_layout_rejects(lib):
    meta = (ctypes.c_uint8 * 64)()
    out = mx.BwLayout()
    tab = (ctypes.c_uint8 * 4)(2, 3, 4, 8)
    assert lib.mx_bw_layout_init(64, 200, tab, meta, ctypes.byref(out)) == 1       # K % 128
    assert lib.mx_bw_layout_init(0, 128, tab, meta, ctypes.byref(out)) == 1        # N < 1
    assert lib.mx_bw_layout_init(64, 128, (ctypes.c_uint8 * 4)(0, 3, 4, 8), meta, ctypes.byref(out)) == 1
    assert lib.mx_bw_layout_init(64, 128, (ctypes.c_uint8 * 4)(2, 3, 4, 9), meta, ctypes.byref(out)) == 1
    assert lib.mx_bw_layout_init(64, 128, tab, None, ctypes.byref(out)) == 1
    assert lib.mx_bw_layout_init(64, 128, tab, meta, None) == 1
    assert lib.mx_bw_layout_init(64, 128, tab, meta, ctypes.byref(out)) == 0


def test_pack_and_gemm_host_checks_before_any_launch(lib, orc):
    codes = np.array([[0, 1], [2, 3]], np.uint8)
    meta = orc.pack_block_codes(codes)
    L = mx.mx_bw_layout_init(100, 256, [2, 3, 4, 8], meta)
    P = ctypes.c_void_p(256)
    # pack: a meta that is not the layout's, a bad dtype, ldw < K
    other = orc.pack_block_codes(np.array([[3, 1], [2, 3]], np.uint8))
    assert lib.mx_bw_pack(ctypes.byref(L), mx._host_bytes(other), P, 0, 256, P, None) == 1
    assert b"meta" in lib.mx_last_error()
    assert lib.mx_bw_pack(ctypes.byref(L), mx._host_bytes(meta), P, 5, 256, P, None) == 1
    assert lib.mx_bw_pack(ctypes.byref(L), mx._host_bytes(meta), P, 0, 255, P, None) == 1
    # gemm: negative M, ldy < N, too many tokens; M = 0 is a no-op
    assert lib.mx_bw_gemm(ctypes.byref(L), P, P, P, -1, P, 100, None, None) == 1
    assert lib.mx_bw_gemm(ctypes.byref(L), P, P, P, 4, P, 99, None, None) == 1
    assert lib.mx_bw_gemm(ctypes.byref(L), P, P, P, 65535 * 8 + 1, P, 100, None, None) == 2
    assert lib.mx_bw_gemm(ctypes.byref(L), P, P, P, 0, P, 100, None, None) == 0
    # a layout whose fields disagree is refused by both
    for field, value in (("off_codes", L.off_codes + 16), ("NB", 3), ("code_bytes", L.code_bytes + 16)):
        bad = mx.BwLayout.from_buffer_copy(L)
        setattr(bad, field, value)
        assert lib.mx_bw_gemm(ctypes.byref(bad), P, P, P, 0, P, 100, None, None) == 1, field
        assert lib.mx_bw_pack(ctypes.byref(bad), mx._host_bytes(meta), P, 0, 256, P, None) == 1, field


def test_byte_model_counts_every_section_of_the_blob(lib, orc):
    # the algorithmic weight bytes are the blob without its 64-byte header and alignment
    from mixed_precision_quantized_mx_b200 import model
    rng = np.random.default_rng(9)
    for N, K in ((4096, 4096), (14336, 4096), (130, 640)):
        codes = inputs.block_codes(rng, N, K, (0.25, 0.25, 0.4, 0.1))
        L = mx.mx_bw_layout_init(N, K, [2, 3, 4, 8], orc.pack_block_codes(codes))
        wb = model.bw_weight_bytes(N, K, L.code_bytes)
        assert 64 <= L.total_bytes - wb <= 64 + 4 * 15
        assert model.bw_gemm_bytes(3, N, K, L.code_bytes) == wb + 3 * K + 6 + 6 * N
