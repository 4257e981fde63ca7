"""Pins for the oracle's KTO / ORPO / SimPO losses: closed forms, reductions to the SFT loss,
library sigmoids, and finite differences through the whole model on tiny shapes."""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import model as om
from oracle import pref
from tests.test_oracle_model import TINYCFG, _fd_check, _rand_model


def _logsig(z):
    return F.logsigmoid(torch.tensor(z, dtype=torch.float64)).item()


def test_simpo_closed_forms():
    n = np.full(4, 10.0)
    pi = np.array([-20.0, -20.0, -31.0, -31.0])  # equal averages within each pair
    loss, dpi = pref.simpo_loss(pi, n, beta=2.0, gamma=0.0)
    assert loss == pytest.approx(math.log(2), rel=1e-15)
    assert np.allclose(dpi, [-2.0 * 0.5 / 10 / 2, 2.0 * 0.5 / 10 / 2] * 2, rtol=1e-15)
    # a margin gamma alone: -log sigmoid(-gamma)
    loss, _ = pref.simpo_loss(pi, n, beta=2.0, gamma=0.7)
    assert loss == pytest.approx(-_logsig(-0.7), rel=1e-14)
    # unequal lengths: the averages, not the sums, are compared
    pi = np.array([-12.0, -30.0])
    nn = np.array([4.0, 10.0])  # averages -3.0 and -3.0
    loss, _ = pref.simpo_loss(pi, nn, beta=1.5, gamma=0.0)
    assert loss == pytest.approx(math.log(2), rel=1e-15)
    # against a library log-sigmoid, and the swap identity L(swap) - L = z
    pi = np.array([-14.0, -19.0])
    loss, _ = pref.simpo_loss(pi, nn, beta=2.5, gamma=0.0)
    z = 2.5 * (-14.0 / 4 + 19.0 / 10)
    assert loss == pytest.approx(-_logsig(z), rel=1e-14)
    loss_sw, _ = pref.simpo_loss(pi[::-1].copy(), nn[::-1].copy(), beta=2.5, gamma=0.0)
    assert loss_sw - loss == pytest.approx(z, rel=1e-13)


def test_orpo_closed_forms():
    n = np.full(2, 8.0)
    a = math.log(0.5)  # odds(0.5) = 1, log odds = 0
    pi = np.array([8 * a, 8 * a])
    loss, _ = pref.orpo_loss(pi, n, lam=0.3)
    assert loss == pytest.approx(-a + 0.3 * math.log(2), rel=1e-14)
    # log(1 - e^a) on both branches against the direct form
    for x in (-0.01, -0.3, -math.log(2), -2.0, -20.0):
        assert pref._log1mexp(np.float64(x)) == pytest.approx(math.log(1 - math.exp(x)), rel=1e-12)
    # the odds ratio term by hand: a_c = ln 0.8, a_r = ln 0.2 -> odds 4 and 1/4 -> z = ln 16
    pi = np.array([8 * math.log(0.8), 8 * math.log(0.2)])
    loss, _ = pref.orpo_loss(pi, n, lam=1.0)
    assert loss == pytest.approx(-math.log(0.8) - _logsig(math.log(16.0)), rel=1e-13)


def test_orpo_without_odds_term_is_sft_on_chosen():
    """lam = 0: the chosen response's token-mean cross-entropy (the SFT loss masked to the
    chosen rows' response targets)."""
    rng = np.random.default_rng(3)
    B, S, V, pre = 2, 9, 11, 4
    logits = rng.standard_normal((B * S, V))
    ids = rng.integers(0, V, (B, S))
    pi, _ = om.sequence_logps(logits, ids, pre)
    loss, _ = pref.orpo_loss(pi, pref.response_counts(B, S, pre), lam=0.0)
    mask = np.zeros((B, S), np.uint8)
    mask[0, pre:] = 1
    want, _ = om.sft_loss(logits, ids, mask)
    assert loss == pytest.approx(want, rel=1e-13)


def test_kto_closed_forms():
    pi = np.array([-5.0, -6.0, -7.0, -8.0])
    labels = np.array([1, 0, 1, 0])
    loss, dpi, z0 = pref.kto_loss(pi, pi.copy(), labels, beta=0.1, lam_d=1.0, lam_u=1.0)
    assert z0 == 0.0 and loss == pytest.approx(0.5, rel=1e-15)
    assert np.allclose(dpi, [-0.1 / 4 / 4, 0.1 / 4 / 4] * 2, rtol=1e-15)
    # z0 is the clamped batch mean of the rewards
    ref = pi - np.array([1.0, 2.0, 3.0, -2.0])
    _, _, z0 = pref.kto_loss(pi, ref, labels, 0.1, 1.0, 1.0)
    assert z0 == pytest.approx(1.0, rel=1e-15)
    _, _, z0 = pref.kto_loss(pi, pi + 1.0, labels, 0.1, 1.0, 1.0)
    assert z0 == 0.0
    # one desirable row with reward r above z0 = 0 (other row pulls the mean below 0)
    pi2, ref2 = np.array([-3.0, -9.0]), np.array([-5.0, -4.0])  # r = 2, -5
    loss, _, z0 = pref.kto_loss(pi2, ref2, np.array([1, 0]), beta=0.5, lam_d=2.0, lam_u=1.5)
    sd = 1 / (1 + math.exp(-0.5 * 2.0))
    su = 1 / (1 + math.exp(-0.5 * (0.0 + 5.0)))
    assert z0 == 0.0 and loss == pytest.approx(((2.0 - 2.0 * sd) + (1.5 - 1.5 * su)) / 2, rel=1e-14)


def test_per_sequence_gradients_finite_difference():
    rng = np.random.default_rng(4)
    n = np.array([6.0, 6.0, 9.0, 9.0])
    pi = -np.abs(rng.normal(8, 2, 4))
    cases = [
        lambda x: pref.simpo_loss(x, n, 2.0, 0.5)[:2],
        lambda x: pref.orpo_loss(x, n, 0.2)[:2],
    ]
    for fn in cases:
        _, g = fn(pi)
        for b in range(4):
            e = np.zeros(4)
            e[b] = 1e-6
            fd = (fn(pi + e)[0] - fn(pi - e)[0]) / 2e-6
            assert fd == pytest.approx(g[b], rel=1e-6, abs=1e-10)
    # KTO, reference held, mean reward < 0: z0 stays clamped at 0 under the perturbations,
    # so the detached gradient is the full derivative there
    ref = pi + np.array([0.5, 1.0, 0.2, 0.9])
    fn = lambda x: pref.kto_loss(x, ref, [1, 0, 0, 1], 0.3, 1.0, 1.3)
    _, g, z0 = fn(pi)
    assert z0 == 0.0
    for b in range(4):
        e = np.zeros(4)
        e[b] = 1e-6
        fd = (fn(pi + e)[0] - fn(pi - e)[0]) / 2e-6
        assert fd == pytest.approx(g[b], rel=1e-6, abs=1e-10)


@pytest.mark.parametrize("kind", ["simpo", "orpo", "kto"])
def test_pref_step_lora_gradients_finite_difference(kind):
    cfg = dict(TINYCFG, n_layers=1)
    layers, lora, head = _rand_model(cfg, seed=6)
    lora = {k: [a.copy(), b.copy()] for k, (a, b) in lora.items()}
    rng = np.random.default_rng(13)
    S, pre = 7, 3
    ids = rng.integers(0, cfg["vocab"], (4, S))
    ids[1, :pre] = ids[0, :pre]
    ids[3, :pre] = ids[2, :pre]
    hp = dict(simpo=dict(beta=2.0, gamma=0.3), orpo=dict(lam=0.25), kto=dict(beta=0.5, lam_d=1.0, lam_u=1.2))[kind]
    labels = np.array([1, 0, 0, 1])
    loss, grads, aux = pref.pref_step(cfg, layers, lora, head, ids, pre, kind, hp, labels)
    if kind == "kto":
        # the finite difference sees z0 move unless it is clamped at 0 around this point
        r = aux["pi"] - aux["ref"]
        assert np.mean(r) < -1e-3 or np.mean(r) > 1e-3
        if np.mean(r) > 0:
            pytest.skip("z0 > 0 here: its dependence is detached by definition")
    fn = lambda: pref.pref_step(cfg, layers, lora, head, ids, pre, kind, hp, labels)[0]
    picks = [((0, p), w, (0, 1)) for p in om.PROJ for w in (0, 1)]
    _fd_check(fn, lora, {k: list(v) for k, v in grads.items()}, picks, tol=1e-5)
