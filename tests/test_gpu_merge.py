"""GPU parity of soup_model_merge_lora (the merged bf16 weight W + s B A) against the oracle."""
import numpy as np
import pytest
import torch

import synth
from oracle import model as om
from oracle import nf4
from tests.gpu_util import Pair, to64

pytestmark = pytest.mark.gpu

PROJ = synth.PROJ_NAMES


def _compare(got: np.ndarray, want: np.ndarray, terms: np.ndarray):
    """The GPU sums s B A in fp32 before its one bf16 rounding; the oracle sums exactly.  The
    two may differ by one bf16 step where the exact sum sits next to a rounding boundary, plus,
    where the terms cancel, the fp32 error of the sum: r = 64 accumulated products (bounded by
    r * 2^-24 = 2^-18 of s |B| |A|, taken as 2^-16 for the tensor core's accumulation order)
    and the final add (2^-22 of |W|)."""
    ulp = np.exp2(np.floor(np.log2(np.maximum(np.abs(want), 1e-30))) - 7)
    diff = np.abs(got - want)
    w_abs, ba_abs = terms
    bound = ulp * 1.0001 + w_abs * 2.0 ** -22 + ba_abs * 2.0 ** -16
    assert np.all(diff <= bound), float((diff / bound).max())
    assert np.mean(diff > 0) < 1e-3, float(np.mean(diff > 0))


def _terms(W, A, B, s):
    Ab = nf4.bf16_round(np.asarray(A, np.float32)).astype(np.float64)
    Bb = nf4.bf16_round(np.asarray(B, np.float32)).astype(np.float64)
    return np.abs(W), s * (np.abs(Bb) @ np.abs(Ab))


@pytest.mark.parametrize("mode", ["streamed", "resident"])
def test_merge_matches_oracle_tiny(mode):
    cfg = dict(synth.TINY)
    p = Pair(cfg, seed=21, modes=(mode,))
    try:
        gm = p.models[mode]
        s = cfg["lora_alpha"] / cfg["lora_r"]
        for layer in range(cfg["n_layers"]):
            for proj in PROJ:
                got = to64(gm.merge_lora(layer, proj))
                A, B = p.olora[(layer, proj)]
                want = om.merge_lora(p.olayers[layer][proj], A, B, s)
                _compare(got, want, _terms(p.olayers[layer][proj], A, B, s))
        # zero adapters: the merged weight is the dequantised base, bit for bit
        zero = torch.zeros_like(p.params_t)
        gm.set_lora(zero)
        got = to64(gm.merge_lora(1, "down"))
        assert np.array_equal(got, p.olayers[1]["down"])
    finally:
        p.close()


@pytest.mark.slow
def test_merge_full_size_o_projection():
    """8B shape (hidden 4096, r 64): the o projection, every element against the oracle."""
    from layer_streamed_nf4_lut_b200.model import SoupModel, lora_offset
    cfg = dict(synth.L8B, n_layers=1)
    gm = SoupModel(cfg, mode="streamed", n_layer_buffers=2, max_tokens=64)
    try:
        w = {p: synth.normal_device(synth.proj_shape(cfg, p), 300 + j, 0.02) for j, p in enumerate(PROJ)}
        ones = torch.ones(cfg["hidden"], dtype=torch.bfloat16, device="cuda")
        gm.quantize_layer(0, w, ones, ones)
        w_o = w["o"].cpu().numpy()
        del w
        lora = synth.lora_weights(dict(cfg, n_layers=1), 31)
        flat = np.zeros(gm.lora_n, np.float32)
        for (layer, p), (A, B) in lora.items():
            j = PROJ.index(p)
            oa, _, _ = lora_offset(cfg, layer, j, 0)
            ob, _, _ = lora_offset(cfg, layer, j, 1)
            flat[oa:oa + A.size] = A.ravel()
            flat[ob:ob + B.size] = B.ravel()
        gm.set_lora(torch.from_numpy(flat).cuda())
        got = to64(gm.merge_lora(0, "o"))
        A, B = lora[(0, "o")]
        W = nf4.dequant(nf4.quantise(w_o)).astype(np.float64)
        s = cfg["lora_alpha"] / cfg["lora_r"]
        want = om.merge_lora(W, A.astype(np.float64), B.astype(np.float64), s)
        _compare(got, want, _terms(W, A, B, s))
    finally:
        gm.close()
