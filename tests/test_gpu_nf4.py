"""GPU parity of the NF4 kernels: quantiser bytes and dequantised values bit-exact against
the oracle; the fused dequant GEMM (forward and transposed) against float64."""
import numpy as np
import pytest
import torch

import synth
from oracle import nf4
from tests.gpu_util import rel_err, to64

pytestmark = pytest.mark.gpu


def _gpu_quant(w32):
    from layer_streamed_nf4_lut_b200 import model as M
    q = M.nf4_quantize(torch.from_numpy(w32).cuda())
    torch.cuda.synchronize()
    return q


SHAPES = [(256, 688), (688, 256), (128, 256), (1, 197), (3, 64 * 300 + 40), (4096, 1024)]


@pytest.mark.parametrize("shape", SHAPES)
def test_quantiser_bytes_bit_exact(shape):
    w = synth.normal(7, 100 + shape[1], shape, 0.02)
    if shape == (128, 256):
        w[3, :128] = 0.0  # two all-zero blocks
        w[5, 64:128] = np.float32(1e-30)  # tiny absmax block
    q = _gpu_quant(w)
    o = nf4.quantise(w)
    assert np.array_equal(q["codes"].cpu().numpy(), o["codes"])
    assert np.array_equal(q["q8"].cpu().numpy(), o["q8"])
    assert np.array_equal(q["scales"].cpu().numpy().view(np.uint32), o["scales"].view(np.uint32))
    assert q["mean"].cpu().numpy().view(np.uint32)[0] == np.float32(o["mean"]).view(np.uint32)


@pytest.mark.parametrize("shape", SHAPES)
def test_dequant_bit_exact(shape):
    from layer_streamed_nf4_lut_b200 import model as M
    w = synth.normal(8, 200 + shape[0], shape, 0.02)
    q = _gpu_quant(w)
    d = M.nf4_dequantize(q)
    torch.cuda.synchronize()
    got = d.view(torch.int16).cpu().numpy().view(np.uint16)
    want = nf4.dequant_bits(nf4.quantise(w))
    assert np.array_equal(got, want)


# The last two run the stream-K schedule in one orientation each (forward of the first,
# transposed of the second: k-blocks spread over one CTA per SM, partial tiles summed through
# the workspace), with ragged M and N tiles
@pytest.mark.parametrize("M_,N,K", [(64, 1376, 256), (200, 256, 688), (128, 512, 4096), (37, 128, 128),
                                    (512, 6144, 4096), (300, 768, 1024), (256, 1280, 2048), (300, 3208, 8192),
                                    (300, 12800, 3208)])
@pytest.mark.parametrize("transpose", [False, True])
def test_nf4_matmul_vs_float64(M_, N, K, transpose):
    from layer_streamed_nf4_lut_b200 import model as M
    w = synth.normal(9, N + K, (N, K), 0.02)
    q = _gpu_quant(w)
    Wd = nf4.dequant(nf4.quantise(w)).astype(np.float64)
    kin = N if transpose else K
    xb = synth.bf16_bits_from_f32(synth.normal(10, M_, (M_, kin), 1.0))
    from tests.gpu_util import bf16_tensor
    x = bf16_tensor(xb)
    x64 = to64(x)
    res = None
    if not transpose:
        res = bf16_tensor(synth.bf16_bits_from_f32(synth.normal(11, M_, (M_, N), 1.0)))
    y = M.nf4_matmul(x, q, transpose_w=transpose, residual=res)
    torch.cuda.synchronize()
    want = x64 @ Wd if transpose else x64 @ Wd.T + to64(res)
    got = to64(y)
    # bf16 output rounding (2^-9 relative) dominates: fp32 accumulation of exact bf16 products
    assert rel_err(got, want) < 4e-3
    assert np.max(np.abs(got - want)) <= 2.0 ** -7 * np.max(np.abs(want)) + 1e-3



# Forward GEMMs without a residual and with at least 96 output tiles of 128 weight rows x 256
# tokens take the kernel whose dequantised weight tile lives in tensor memory (the MMA's A
# operand); the second shape has a ragged last weight tile and a ragged last token tile.
@pytest.mark.parametrize("M_,N,K", [(512, 6144, 4096), (300, 12352, 1024)])
def test_nf4_matmul_tmem_weight_form_vs_float64(M_, N, K, monkeypatch):
    from layer_streamed_nf4_lut_b200 import model as M
    from tests.gpu_util import bf16_tensor
    w = synth.normal(19, N + K, (N, K), 0.02)
    q = _gpu_quant(w)
    Wd = nf4.dequant(nf4.quantise(w)).astype(np.float64)
    x = bf16_tensor(synth.bf16_bits_from_f32(synth.normal(20, M_, (M_, K), 1.0)))
    want = to64(x) @ Wd.T
    outs = {}
    for flag in ("1", "0"):  # the tensor-memory form, then the shared-memory kernel
        monkeypatch.setenv("SOUP_GEMM_TS", flag)
        y = M.nf4_matmul(x, q)
        torch.cuda.synchronize()
        got = to64(y)
        assert rel_err(got, want) < 4e-3
        assert np.max(np.abs(got - want)) <= 2.0 ** -7 * np.max(np.abs(want)) + 1e-3
        outs[flag] = y
    if M_ % 256 == 0 and N % 128 == 0:
        # whole tiles on both sides: the same products summed in the same k order
        assert torch.equal(outs["1"], outs["0"])
