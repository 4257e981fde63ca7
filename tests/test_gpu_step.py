"""GPU parity of whole training steps (SFT and DPO) against the oracle, the streamed ==
resident bit-exactness claim, the layer-load counts, determinism and error reporting."""
import math

import numpy as np
import pytest
import torch

import synth
from oracle import model as om
from tests.gpu_util import Pair, cosine, rel_err, to64

pytestmark = pytest.mark.gpu

PROJ = synth.PROJ_NAMES
TINY4 = dict(synth.TINY, n_layers=4, name="tiny-4L")


def _check_grads(pair, mode, og, min_cos=0.999):
    g = pair.gpu_grads(mode)
    worst = 1.0
    for k, (gA, gB) in g.items():
        worst = min(worst, cosine(gA, og[k][0]), cosine(gB, og[k][1]))
    assert worst > min_cos, worst


@pytest.fixture(scope="module")
def tiny_pair():
    p = Pair(dict(synth.TINY), seed=11, modes=("streamed", "resident"), max_tokens=4 * 64)
    yield p
    p.close()


def test_sft_step_matches_oracle(tiny_pair):
    cfg = tiny_pair.cfg
    ids = synth.token_batch(cfg, 31)
    loss = tiny_pair.models["streamed"].step(torch.from_numpy(ids).cuda(), apply_optimizer=False)
    ol, og, _ = om.sft_step(cfg, tiny_pair.olayers, tiny_pair.olora, tiny_pair.ohead, ids)
    assert abs(loss - ol) / abs(ol) < 1e-2
    _check_grads(tiny_pair, "streamed", og)


def test_sft_masked_zipf_batch(tiny_pair):
    cfg = dict(tiny_pair.cfg, batch=2)
    ids = synth.token_batch(cfg, 32, zipf=True)
    mask = synth.last_half_mask(2, cfg["seq"])
    loss = tiny_pair.models["resident"].step(ids, mask=mask, apply_optimizer=False)  # host ids
    ol, og, _ = om.sft_step(cfg, tiny_pair.olayers, tiny_pair.olora, tiny_pair.ohead, ids, mask)
    assert abs(loss - ol) / abs(ol) < 1e-2
    _check_grads(tiny_pair, "resident", og)


def test_streamed_equals_resident_bitwise(tiny_pair):
    cfg = dict(tiny_pair.cfg, batch=2)
    ids = torch.from_numpy(synth.token_batch(cfg, 33)).cuda()
    ls = tiny_pair.models["streamed"].step(ids, apply_optimizer=False)
    lr_ = tiny_pair.models["resident"].step(ids, apply_optimizer=False)
    assert ls == lr_  # difference 0.0
    gs, gr = tiny_pair.models["streamed"].lora_grads, tiny_pair.models["resident"].lora_grads
    assert torch.equal(gs.view(torch.int32), gr.view(torch.int32))


def test_dpo_step_matches_oracle(tiny_pair):
    cfg = dict(tiny_pair.cfg, batch=4, n_pairs=2, prefix_len=32, beta=0.1)
    ids = synth.preference_batch(cfg, 34)
    gm = tiny_pair.models["streamed"]
    loss = gm.step(torch.from_numpy(ids).cuda(), loss="dpo", n_pairs=2, prefix_len=32, beta=0.1, apply_optimizer=False)
    ol, og, aux = om.dpo_step(cfg, tiny_pair.olayers, tiny_pair.olora, tiny_pair.ohead, ids, 32, 0.1)
    pi, ref = gm.last_logps(4)
    assert rel_err(pi, aux["pi"]) < 1e-2 and rel_err(ref, aux["ref"]) < 1e-2
    # the loss is ln2 + small: check it against the closed form of the GPU's own log-probs too
    closed, _ = om.dpo_loss(pi.astype(np.float64), ref.astype(np.float64), 0.1)
    assert abs(loss - closed) < 1e-5
    assert abs(loss - ol) < 1e-2 * abs(ol)
    _check_grads(tiny_pair, "streamed", og)


def test_layer_load_counts():
    p = Pair(TINY4, seed=12, modes=("streamed",), want_oracle=False, max_tokens=4 * 64)
    try:
        gm = p.models["streamed"]
        L = TINY4["n_layers"]
        ids = torch.from_numpy(synth.token_batch(TINY4, 35)).cuda()
        gm.reset_stats()
        gm.step(ids, apply_optimizer=False)
        s1 = gm.stats()["layer_loads"]
        gm.reset_stats()
        gm.step(ids, apply_optimizer=False)
        s2 = gm.stats()["layer_loads"]
        cfg = dict(TINY4, batch=4)
        pids = torch.from_numpy(synth.preference_batch(dict(cfg, n_pairs=2, prefix_len=32), 36)).cuda()
        gm.reset_stats()
        gm.step(pids, loss="dpo", n_pairs=2, prefix_len=32, apply_optimizer=False)
        d = gm.stats()["layer_loads"]
        assert s1 == 2 * L - 2 - 2 or s1 == 2 * L - 2  # first step may find layers 0,1 from quantisation
        assert s2 == 2 * L - 4  # layers 0 and 1 stay resident from the previous backward
        assert d == 3 * L - 4
        # the pages' ratio (cold streamer): (3L-2)/(2L-2) = 94/62 = 1.516 at L = 32
        assert abs((3 * 32 - 2) / (2 * 32 - 2) - 1.52) < 0.005
    finally:
        p.close()


def test_run_to_run_deterministic(tiny_pair):
    ids = torch.from_numpy(synth.token_batch(tiny_pair.cfg, 37)).cuda()
    gm = tiny_pair.models["streamed"]
    l1 = gm.step(ids, apply_optimizer=False)
    g1 = gm.lora_grads.clone()
    l2 = gm.step(ids, apply_optimizer=False)
    assert l1 == l2 and torch.equal(g1.view(torch.int32), gm.lora_grads.view(torch.int32))


def test_adamw_step_matches_oracle():
    p = Pair(dict(synth.TINY), seed=13, modes=("resident",), want_oracle=False)
    try:
        gm = p.models["resident"]
        ids = torch.from_numpy(synth.token_batch(p.cfg, 38)).cuda()
        p0 = gm.lora_params.clone()
        gm.step(ids, lr=1e-3, apply_optimizer=True)
        g = to64(gm.lora_grads)
        want, _, _ = om.adamw(to64(p0), g, np.zeros_like(g), np.zeros_like(g), 1, 1e-3)
        assert np.max(np.abs(to64(gm.lora_params) - want)) < 1e-6
    finally:
        p.close()


def test_bad_token_id_reports_device_check():
    from layer_streamed_nf4_lut_b200._lib import SoupError
    p = Pair(dict(synth.TINY), seed=14, modes=("resident",), want_oracle=False)
    try:
        ids = synth.token_batch(p.cfg, 39)
        ids[0, 5] = p.cfg["vocab"] + 7
        with pytest.raises(SoupError) as ei:
            p.models["resident"].step(torch.from_numpy(ids).cuda(), apply_optimizer=False)
        assert ei.value.status == -6
        # the model stays usable after the error
        ids[0, 5] = 3
        loss = p.models["resident"].step(torch.from_numpy(ids).cuda(), apply_optimizer=False)
        assert math.isfinite(loss)
    finally:
        p.close()


def test_dpo_shared_load_schedule_same_bits_fewer_loads():
    p = Pair(TINY4, seed=15, modes=("streamed",), want_oracle=False, max_tokens=4 * 64)
    try:
        gm = p.models["streamed"]
        L = TINY4["n_layers"]
        cfg = dict(TINY4, batch=4, n_pairs=2, prefix_len=32)
        ids = torch.from_numpy(synth.preference_batch(cfg, 40)).cuda()
        kw = dict(loss="dpo", n_pairs=2, prefix_len=32, beta=0.1, apply_optimizer=False)
        gm.step(ids, **kw)  # warm: layers 0, 1 resident afterwards
        gm.reset_stats()
        l_re = gm.step(ids, **kw)
        loads_re = gm.stats()["layer_loads"]
        g_re = gm.lora_grads.clone()
        pi_re, ref_re = gm.last_logps(4)
        gm.reset_stats()
        l_sh = gm.step(ids, dpo_shared_load=True, **kw)
        loads_sh = gm.stats()["layer_loads"]
        pi_sh, ref_sh = gm.last_logps(4)
        assert l_sh == l_re
        assert torch.equal(g_re.view(torch.int32), gm.lora_grads.view(torch.int32))
        assert np.array_equal(pi_sh, pi_re) and np.array_equal(ref_sh, ref_re)
        assert loads_re == 3 * L - 4 and loads_sh == 2 * L - 4
    finally:
        p.close()


def test_side_stream_grads_same_bits(monkeypatch):
    """LoRA weight gradients computed on the side stream (default) equal those computed in
    line on the main stream, bit for bit."""
    cfg = dict(TINY4, batch=4)
    ids = torch.from_numpy(synth.token_batch(cfg, 48)).cuda()
    out = {}
    for flag in ("1", "0"):
        monkeypatch.setenv("SOUP_CONCURRENT_GRADS", flag)
        p = Pair(TINY4, seed=19, modes=("streamed",), want_oracle=False, max_tokens=4 * 64)
        try:
            gm = p.models["streamed"]
            losses = [gm.step(ids, apply_optimizer=False) for _ in range(3)]  # eager, capture, replay
            out[flag] = (losses, gm.lora_grads.clone())
        finally:
            p.close()
    assert out["1"][0] == out["0"][0]
    assert torch.equal(out["1"][1].view(torch.int32), out["0"][1].view(torch.int32))


def test_per_layer_adamw_in_backward_same_bits_as_whole_update():
    """With the optimizer on, soup_step updates each layer's LoRA slice during the backward pass
    (layer i+1's slice beside layer i's backward, layer 0's at the end); parameters, both AdamW
    moments and the losses equal, bit for bit, steps without the optimizer each followed by the
    whole-vector soup_optimizer_step, over eager, captured and replayed steps, with lr changing
    between steps and the two forms interleaved."""
    cfg = dict(TINY4, batch=2)
    ids = torch.from_numpy(synth.token_batch(cfg, 52)).cuda()
    out = {}
    # the mixed schedule alternates the two forms, so each layer's backward graph is captured
    # and replayed both with and without the update, and lr changes between steps
    schedules = {"in_backward": [True] * 5, "after": [False] * 5, "mixed": [True, False, True, True, False]}
    lrs = [1e-3, 2e-3, 1e-3, 5e-4, 1e-3]
    for mode, sched in schedules.items():
        p = Pair(TINY4, seed=29, modes=("streamed",), want_oracle=False, max_tokens=2 * 64)
        try:
            gm = p.models["streamed"]
            losses = []
            for in_bwd, lr in zip(sched, lrs):
                if in_bwd:
                    losses.append(gm.step(ids, lr=lr, apply_optimizer=True))
                else:
                    losses.append(gm.step(ids, lr=lr, apply_optimizer=False))
                    gm.optimizer_step(lr)
            torch.cuda.synchronize()
            out[mode] = (losses, gm.lora_params.clone(), gm.adam_m.clone(), gm.adam_v.clone())
        finally:
            p.close()
    for other in ("after", "mixed"):
        a, b = out["in_backward"], out[other]
        assert a[0] == b[0], other
        for x, y in zip(a[1:], b[1:]):
            assert torch.equal(x.view(torch.int32), y.view(torch.int32)), other
