"""GPU parity of one decoder layer (forward and backward with LoRA) against the float64
oracle, on the small Llama-style shape (hidden 256, 4/2 heads, head_dim 64, intermediate
688: ragged K and N tiles) and a ragged token count."""
import numpy as np
import pytest
import torch

import synth
from oracle import model as om
from tests.gpu_util import Pair, bf16_tensor, cosine, rel_err, to64

pytestmark = pytest.mark.gpu

PROJ = synth.PROJ_NAMES


@pytest.fixture(scope="module")
def pair():
    cfg = dict(synth.TINY)
    # larger weights than the workload's 0.02 so that the layer's update is of the same size
    # as its residual input and the comparison below is not dominated by bf16 output rounding
    p = Pair(cfg, seed=3, modes=("resident",), max_tokens=2 * 64, w_std=0.08)
    yield p
    p.close()


@pytest.mark.parametrize("B,S", [(1, 64), (2, 37)])
@pytest.mark.parametrize("lora_on", [True, False])
def test_layer_forward_backward(pair, B, S, lora_on):
    cfg = pair.cfg
    gm = pair.models["resident"]
    gm.set_lora_enabled(lora_on)
    T, h = B * S, cfg["hidden"]
    xb = synth.bf16_bits_from_f32(synth.normal(21, T, (T, h), 1.0))
    dyb = synth.bf16_bits_from_f32(synth.normal(22, T, (T, h), 1.0))
    x, dy = bf16_tensor(xb), bf16_tensor(dyb)
    gm.lora_grads.zero_()
    y = gm.layer_fwd(1, x, B, S)
    dx = gm.layer_bwd(1, dy, B, S)
    torch.cuda.synchronize()
    gm.set_lora_enabled(True)
    lo = {p: pair.olora[(1, p)] for p in PROJ}
    y_o, cache = om.layer_forward(cfg, pair.olayers[1], lo, to64(x), B, S, enabled=lora_on)
    dx_o, g_o = om.layer_backward(cfg, pair.olayers[1], lo, cache, to64(dy), B, S, enabled=lora_on)
    # the layer's update y - x and dx - dy (bf16 activations throughout: ~2^-8 relative per
    # rounding, a few roundings deep)
    assert rel_err(to64(y), y_o) < 1e-2
    assert rel_err(to64(y) - to64(x), y_o - to64(x)) < 2e-2
    assert rel_err(to64(dx), dx_o) < 1e-2
    assert rel_err(to64(dx) - to64(dy), dx_o - to64(dy)) < 3e-2
    # element by element: the bf16 output itself is rounded (2^-9 relative) after a few bf16
    # roundings of its operands, so each element may be off by 2^-7 of its own size plus a tenth
    # of the layer's typical update; a wrong tile (a ragged edge of N = 688 or T = 74 rows)
    # would be off by the size of the update itself
    for got, want, base in ((to64(y), y_o, to64(x)), (to64(dx), dx_o, to64(dy))):
        upd = float(np.sqrt(np.mean((want - base) ** 2)))
        bound = 2.0 ** -7 * np.abs(want) + 0.1 * upd
        worst = np.unravel_index(np.argmax(np.abs(got - want) - bound), want.shape)
        assert np.all(np.abs(got - want) <= bound), (worst, got[worst], want[worst], upd)
    grads = pair.gpu_grads("resident")
    for p in PROJ:
        gA, gB = grads[(1, p)]
        if lora_on:
            assert cosine(gA, g_o[p][0]) > 0.999, p
            assert cosine(gB, g_o[p][1]) > 0.999, p
        else:
            assert np.all(gA == 0) and np.all(gB == 0)
        assert np.all(grads[(0, p)][0] == 0)  # other layer untouched


@pytest.mark.parametrize("B,S", [(1, 512), (2, 256)])
def test_layer_whole_query_tiles(B, S):
    """Sequences of whole 128-row query tiles at head_dim 64: the attention forward's O tiles
    leave through its TMA store (a ragged last tile stores row by row), the K / V rings wrap
    (four key tiles over three stages at S = 512), and the causal diagonal falls inside tiles."""
    cfg = dict(synth.TINY)
    p = Pair(cfg, seed=6, modes=("resident",), max_tokens=B * S, w_std=0.08)
    try:
        gm = p.models["resident"]
        T, h = B * S, cfg["hidden"]
        x = bf16_tensor(synth.bf16_bits_from_f32(synth.normal(31, T, (T, h), 1.0)))
        dy = bf16_tensor(synth.bf16_bits_from_f32(synth.normal(32, T, (T, h), 1.0)))
        gm.lora_grads.zero_()
        y = gm.layer_fwd(1, x, B, S)
        dx = gm.layer_bwd(1, dy, B, S)
        torch.cuda.synchronize()
        lo = {q: p.olora[(1, q)] for q in PROJ}
        y_o, cache = om.layer_forward(cfg, p.olayers[1], lo, to64(x), B, S, enabled=True)
        dx_o, g_o = om.layer_backward(cfg, p.olayers[1], lo, cache, to64(dy), B, S, enabled=True)
        for got, want, base in ((to64(y), y_o, to64(x)), (to64(dx), dx_o, to64(dy))):
            upd = float(np.sqrt(np.mean((want - base) ** 2)))
            bound = 2.0 ** -7 * np.abs(want) + 0.1 * upd
            worst = np.unravel_index(np.argmax(np.abs(got - want) - bound), want.shape)
            assert np.all(np.abs(got - want) <= bound), (worst, got[worst], want[worst], upd)
        grads = p.gpu_grads("resident")
        for q in PROJ:
            assert cosine(grads[(1, q)][0], g_o[q][0]) > 0.999, q
            assert cosine(grads[(1, q)][1], g_o[q][1]) > 0.999, q
    finally:
        p.close()


def test_lora_off_equals_zero_b_bitwise():
    cfg = dict(synth.TINY)
    a = Pair(cfg, seed=4, modes=("resident",), want_oracle=False)
    b = Pair(cfg, seed=4, modes=("resident",), zero_b=True, want_oracle=False)
    try:
        T, h = 64, cfg["hidden"]
        x = bf16_tensor(synth.bf16_bits_from_f32(synth.normal(23, T, (T, h), 1.0)))
        a.models["resident"].set_lora_enabled(False)
        ya = a.models["resident"].layer_fwd(0, x, 1, 64)
        yb = b.models["resident"].layer_fwd(0, x, 1, 64)
        torch.cuda.synchronize()
        # B = 0 adds an exact zero to every fp32 accumulator: same bits as LoRA off
        assert torch.equal(ya.view(torch.int16), yb.view(torch.int16))
    finally:
        a.close()
        b.close()


def test_bwd_without_fwd_is_state_error():
    from layer_streamed_nf4_lut_b200._lib import SoupError
    cfg = dict(synth.TINY)
    p = Pair(cfg, seed=5, modes=("streamed",), want_oracle=False)
    try:
        dy = torch.zeros(64, cfg["hidden"], dtype=torch.bfloat16, device="cuda")
        with pytest.raises(SoupError) as ei:
            p.models["streamed"].layer_bwd(0, dy, 1, 64)
        assert ei.value.status == -2
    finally:
        p.close()
