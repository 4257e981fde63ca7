"""The library's host quantiser (soup_nf4_quantize_host, behind soup_model_load_layer) against
the float64 oracle, byte for byte.  Pure host code: runs without a GPU."""
import numpy as np
import pytest

import synth
from layer_streamed_nf4_lut_b200 import model as M
from oracle import nf4


def _same(h, o):
    assert np.array_equal(h["codes"], o["codes"])
    assert np.array_equal(h["q8"], o["q8"])
    assert np.array_equal(h["scales"].view(np.uint32), o["scales"].view(np.uint32))
    assert h["mean"].view(np.uint32)[0] == np.float32(o["mean"]).view(np.uint32)


@pytest.mark.parametrize("shape,std", [((3, 64 * 300 + 40), 0.05), ((256, 688), 0.02), ((7,), 1.0),
                                       ((1024, 512), 0.02), ((5, 64 * 257), 3.0)])
@pytest.mark.parametrize("threads", [1, 0, 5])
def test_host_quantiser_bytes_equal_oracle(shape, std, threads):
    w = synth.normal(61, len(shape) * 7 + shape[0], shape, std).astype(np.float32)
    if w.ndim == 2 and w.shape[0] >= 3:
        w[1, :64] = 0.0          # an all-zero block: every code is the code of 0.0
        w[2, 64:128] *= 1e-30    # a tiny absmax (subnormal-range ratios in float64)
        w[0, 5] = -w[0, :64].__abs__().max() * 2  # a block whose absmax is a negative element
    _same(M.nf4_quantize_host(w, threads), nf4.quantise(w))


def test_host_quantiser_exact_codebook_values():
    # elements equal to absmax * c_j (exactly representable here) must get code j
    c = nf4.codebook()
    w = np.tile(c.astype(np.float32), 4 * 8)[:64 * 8] * np.float32(0.5)
    h = M.nf4_quantize_host(w)
    assert np.array_equal(nf4.unpack_codes(h["codes"], w.size), np.tile(np.arange(16, dtype=np.uint8), 32))
    _same(h, nf4.quantise(w))


def test_host_quantiser_rejects_bad_arguments():
    from layer_streamed_nf4_lut_b200._lib import lib
    assert lib.soup_nf4_quantize_host(None, 64, None, None, None, None, 0) == -1
