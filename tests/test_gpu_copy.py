"""mx_copy_mapped: kernel copies between device memory and pinned host memory.

Not part of the method: the graph-captured layer runner moves its input in and
its output out with it.  Every byte must arrive unchanged, whatever the size
and alignment, and a host buffer rewritten between two calls is read afresh.
"""
import numpy as np
import pytest
import torch

from mixed_precision_quantized_mx_b200 import binding as mx

from gpu_helpers import dev

pytestmark = pytest.mark.gpu

SIZES = [1, 15, 16, 17, 8192, 8192 + 7, 1 << 20, (3 << 20) + 5]


def _bytes(n, seed):
    return torch.from_numpy(np.random.default_rng(seed).integers(0, 256, n, dtype=np.uint8))


@pytest.mark.parametrize("n", SIZES)
def test_host_to_device_and_back(n):
    src = _bytes(n, n).pin_memory()
    mid = torch.empty(n, dtype=torch.uint8, device=dev())
    back = torch.zeros(n, dtype=torch.uint8).pin_memory()
    mx.mx_copy_mapped(mid, src)
    mx.mx_copy_mapped(back, mid)
    torch.cuda.synchronize()
    assert torch.equal(mid.cpu(), src)
    assert torch.equal(back, src)


@pytest.mark.parametrize("off_dst,off_src", [(1, 0), (0, 3), (5, 9), (8, 8)])
def test_unaligned_ranges(off_dst, off_src):
    n = 4099
    host = _bytes(n + 16, 5).pin_memory()
    d = torch.zeros(n + 16, dtype=torch.uint8, device=dev())
    mx.mx_copy_mapped(d[off_dst:off_dst + n], host[off_src:off_src + n])
    torch.cuda.synchronize()
    got = d.cpu()
    assert torch.equal(got[off_dst:off_dst + n], host[off_src:off_src + n])
    assert not got[:off_dst].any() and not got[off_dst + n:].any()   # nothing outside the range


def test_device_to_device():
    a = _bytes(65536 + 3, 11).to(dev())
    b = torch.empty_like(a)
    mx.mx_copy_mapped(b, a)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


def test_host_rewrite_between_calls_is_read_afresh():
    n = 8192
    host = _bytes(n, 1).pin_memory()
    d = torch.empty(n, dtype=torch.uint8, device=dev())
    for seed in range(2, 6):
        host.copy_(_bytes(n, seed))
        mx.mx_copy_mapped(d, host)
        torch.cuda.synchronize()
        assert torch.equal(d.cpu(), host)


def test_half_tensors_in_a_stream():
    s = torch.cuda.Stream(dev())
    x = torch.randn(3, 4096).half().pin_memory()
    y = torch.empty(3, 4096, dtype=torch.float16, device=dev())
    with torch.cuda.stream(s):
        mx.mx_copy_mapped(y, x)
    s.synchronize()
    assert torch.equal(y.cpu(), x)


def test_rejections_before_any_launch():
    lib = mx.lib()
    pageable = torch.zeros(4096, dtype=torch.uint8)
    d = torch.zeros(4096, dtype=torch.uint8, device=dev())
    st = lib.mx_copy_mapped(d.data_ptr(), pageable.data_ptr(), 4096, None)
    assert st == 1 and b"pageable" in lib.mx_last_error()
    st = lib.mx_copy_mapped(pageable.data_ptr(), d.data_ptr(), 4096, None)
    assert st == 1
    assert lib.mx_copy_mapped(None, d.data_ptr(), 16, None) == 1
    # overlapping device ranges
    assert lib.mx_copy_mapped(d.data_ptr() + 8, d.data_ptr(), 64, None) == 1
    assert b"overlap" in lib.mx_last_error()
    # zero bytes: nothing to do
    assert lib.mx_copy_mapped(d.data_ptr(), d.data_ptr() + 64, 0, None) == 0
    with pytest.raises(ValueError):
        mx.mx_copy_mapped(d, pageable)
    with pytest.raises(ValueError):
        mx.mx_copy_mapped(d[:16], pageable.pin_memory())
    torch.cuda.synchronize()
    assert not d.any()                                  # nothing was written
