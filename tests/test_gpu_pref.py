"""GPU parity of the KTO, ORPO and SimPO steps against the oracle (tiny shape), the loss of each
against its closed form evaluated on the GPU's own log-probs, and the KTO shared-load schedule."""
import numpy as np
import pytest
import torch

import synth
from oracle import pref
from tests.gpu_util import Pair, cosine, rel_err

pytestmark = pytest.mark.gpu

HP = dict(simpo=dict(beta=2.0, gamma=0.5), orpo=dict(lam=0.1), kto=dict(beta=0.1, lam_d=1.0, lam_u=1.33))
LABELS = np.array([1, 0, 0, 1], np.uint8)


@pytest.fixture(scope="module")
def pair():
    p = Pair(dict(synth.TINY), seed=16, modes=("streamed",), max_tokens=4 * 64)
    yield p
    p.close()


def _kw(kind):
    hp = HP[kind]
    kw = dict(loss=kind, n_pairs=2, prefix_len=32, apply_optimizer=False)
    if kind == "simpo":
        kw.update(beta=hp["beta"], gamma=hp["gamma"])
    elif kind == "orpo":
        kw.update(lambda_or=hp["lam"])
    else:
        kw.update(beta=hp["beta"], lambda_d=hp["lam_d"], lambda_u=hp["lam_u"], labels=LABELS)
    return kw


@pytest.mark.parametrize("kind", ["simpo", "orpo", "kto"])
def test_pref_step_matches_oracle(pair, kind):
    cfg = dict(pair.cfg, batch=4, n_pairs=2, prefix_len=32)
    ids = synth.preference_batch(cfg, 41)
    gm = pair.models["streamed"]
    loss = gm.step(torch.from_numpy(ids).cuda(), **_kw(kind))
    ol, og, aux = pref.pref_step(cfg, pair.olayers, pair.olora, pair.ohead, ids, 32, kind, HP[kind], LABELS)
    pi, ref = gm.last_logps(4)
    assert rel_err(pi, aux["pi"]) < 1e-2
    n = pref.response_counts(4, cfg["seq"], 32)
    pi64 = pi.astype(np.float64)
    if kind == "simpo":
        closed, _ = pref.simpo_loss(pi64, n, HP[kind]["beta"], HP[kind]["gamma"])
    elif kind == "orpo":
        closed, _ = pref.orpo_loss(pi64, n, HP[kind]["lam"])
    else:
        assert rel_err(ref, aux["ref"]) < 1e-2
        closed, _, _ = pref.kto_loss(pi64, ref.astype(np.float64), LABELS, HP[kind]["beta"], HP[kind]["lam_d"],
                                     HP[kind]["lam_u"])
    assert abs(loss - closed) < 1e-5 * max(1.0, abs(closed))
    assert abs(loss - ol) < 1e-2 * abs(ol)
    g = pair.gpu_grads("streamed")
    worst = min(min(cosine(gA, og[k][0]), cosine(gB, og[k][1])) for k, (gA, gB) in g.items())
    assert worst > 0.999, worst


def test_kto_shared_load_same_bits_and_host_labels(pair):
    cfg = dict(pair.cfg, batch=4, n_pairs=2, prefix_len=32)
    ids = synth.preference_batch(cfg, 42)
    gm = pair.models["streamed"]
    kw = _kw("kto")
    l_re = gm.step(torch.from_numpy(ids).cuda(), **kw)
    g_re = gm.lora_grads.clone()
    l_sh = gm.step(torch.from_numpy(ids).cuda(), dpo_shared_load=True, **kw)
    assert l_sh == l_re and torch.equal(g_re.view(torch.int32), gm.lora_grads.view(torch.int32))
    l_host = gm.step(ids, **kw)  # ids and labels from host memory
    assert l_host == l_re


def test_simpo_orpo_stream_like_sft():
    p = Pair(dict(synth.TINY, n_layers=4), seed=17, modes=("streamed",), want_oracle=False, max_tokens=4 * 64)
    try:
        gm = p.models["streamed"]
        cfg = dict(p.cfg, batch=4, n_pairs=2, prefix_len=32)
        ids = torch.from_numpy(synth.preference_batch(cfg, 43)).cuda()
        gm.step(ids, **_kw("simpo"))
        for kind in ("simpo", "orpo"):
            gm.reset_stats()
            gm.step(ids, **_kw(kind))
            assert gm.stats()["layer_loads"] == 2 * 4 - 4
        gm.reset_stats()
        gm.step(ids, **_kw("kto"))
        assert gm.stats()["layer_loads"] == 3 * 4 - 4
    finally:
        p.close()
