"""soup_nf4_quantize_static, the quantiser entry point that allocates nothing.

It exists for callers that cannot call cudaMalloc and therefore cannot hand the regular
soup_nf4_quantize its absmax scratch buffer; it uses a fixed array inside the library
instead.  Its outputs must be the bytes the regular entry point produces (the quantiser's
outputs are integers and exactly defined floats, so the comparison is exact), on calls made
back to back through the C-ABI, including a second call that is smaller than the first and so
leaves old contents in the shared array."""
import ctypes

import numpy as np
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu


def _quantise(w: torch.Tensor, static: bool) -> dict:
    from layer_streamed_nf4_lut_b200._lib import lib
    n = w.numel()
    nb = (n + 63) // 64
    ng = (nb + 255) // 256
    out = dict(codes=torch.empty((n + 1) // 2, dtype=torch.uint8, device="cuda"),
               q8=torch.empty(nb, dtype=torch.int8, device="cuda"),
               scales=torch.empty(ng, dtype=torch.float32, device="cuda"),
               mean=torch.empty(1, dtype=torch.float32, device="cuda"))
    ptr = lambda t: ctypes.c_void_p(t.data_ptr())
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if static:
        st = lib.soup_nf4_quantize_static(ptr(w), n, ptr(out["codes"]), ptr(out["q8"]), ptr(out["scales"]),
                                          ptr(out["mean"]), stream)
    else:
        scratch = torch.empty(nb, dtype=torch.float32, device="cuda")
        st = lib.soup_nf4_quantize(ptr(w), n, ptr(out["codes"]), ptr(out["q8"]), ptr(out["scales"]),
                                   ptr(out["mean"]), ptr(scratch), stream)
    assert st == 0, st
    torch.cuda.synchronize()
    return {k: v.cpu().numpy() for k, v in out.items()}


def _same(a: dict, b: dict):
    for k in ("codes", "q8"):
        assert np.array_equal(a[k], b[k]), k
    for k in ("scales", "mean"):
        assert np.array_equal(a[k].view(np.uint32), b[k].view(np.uint32)), k


def test_static_matches_allocating_entry_point_on_consecutive_calls():
    big = torch.from_numpy(synth.normal(41, 1, (4096, 1024), 0.02)).cuda()
    small = torch.from_numpy(synth.normal(42, 2, (3, 64 * 300 + 40), 0.05)).cuda()
    for w in (big, small):  # the second, smaller call runs over the first call's leftovers
        _same(_quantise(w, static=True), _quantise(w, static=False))
    _same(_quantise(big, static=True), _quantise(big, static=False))


def test_static_rejects_sizes_beyond_its_array():
    from layer_streamed_nf4_lut_b200._lib import lib
    t = torch.zeros(64, dtype=torch.float32, device="cuda")
    p = ctypes.c_void_p(t.data_ptr())
    too_big = (64 << 20) + 1
    assert lib.soup_nf4_quantize_static(p, too_big, p, p, p, p, None) == -1
