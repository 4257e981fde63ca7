"""Preference steps with each pair's shared prefix run once (share_prefix): GPU against the
oracle's plain definition of the step, against the GPU's own plain layout, and the bitwise
claims (streamed == resident, one load per layer == re-stream) in the packed layout."""
import numpy as np
import pytest
import torch

import synth
from oracle import model as om
from oracle import pref
from tests.gpu_util import Pair, cosine, rel_err

pytestmark = pytest.mark.gpu

CFG = dict(synth.TINY, seq=128, name="tiny-s128")
PRE = 64


@pytest.fixture(scope="module")
def pair():
    p = Pair(dict(CFG), seed=22, modes=("streamed", "resident"), max_tokens=4 * 128)
    yield p
    p.close()


def _ids(seed):
    return synth.preference_batch(dict(CFG, batch=4, n_pairs=2, prefix_len=PRE), seed)


def _worst_cos(p, mode, og):
    g = p.gpu_grads(mode)
    return min(min(cosine(gA, og[k][0]), cosine(gB, og[k][1])) for k, (gA, gB) in g.items())


def test_dpo_shared_prefix_matches_oracle(pair):
    ids = _ids(51)
    gm = pair.models["streamed"]
    loss = gm.step(torch.from_numpy(ids).cuda(), loss="dpo", n_pairs=2, prefix_len=PRE, beta=0.1,
                   apply_optimizer=False, share_prefix=True)
    ol, og, aux = om.dpo_step(dict(CFG, batch=4), pair.olayers, pair.olora, pair.ohead, ids, PRE, 0.1)
    pi, ref = gm.last_logps(4)
    assert rel_err(pi, aux["pi"]) < 1e-2 and rel_err(ref, aux["ref"]) < 1e-2
    closed, _ = om.dpo_loss(pi.astype(np.float64), ref.astype(np.float64), 0.1)
    assert abs(loss - closed) < 1e-5
    assert abs(loss - ol) < 1e-2 * abs(ol)
    assert _worst_cos(pair, "streamed", og) > 0.999


def test_simpo_shared_prefix_matches_oracle(pair):
    ids = _ids(52)
    gm = pair.models["streamed"]
    loss = gm.step(torch.from_numpy(ids).cuda(), loss="simpo", n_pairs=2, prefix_len=PRE, beta=2.0, gamma=0.5,
                   apply_optimizer=False, share_prefix=True)
    ol, og, aux = pref.pref_step(dict(CFG, batch=4), pair.olayers, pair.olora, pair.ohead, ids, PRE, "simpo",
                                 dict(beta=2.0, gamma=0.5))
    pi, _ = gm.last_logps(4)
    assert rel_err(pi, aux["pi"]) < 1e-2
    assert abs(loss - ol) < 1e-2 * abs(ol)
    assert _worst_cos(pair, "streamed", og) > 0.999


def test_shared_prefix_close_to_plain_layout(pair):
    ids = torch.from_numpy(_ids(53)).cuda()
    gm = pair.models["streamed"]
    kw = dict(loss="dpo", n_pairs=2, prefix_len=PRE, beta=0.1, apply_optimizer=False)
    l_plain = gm.step(ids, **kw)
    g_plain = gm.lora_grads.clone()
    pi_p, ref_p = gm.last_logps(4)
    l_pack = gm.step(ids, share_prefix=True, **kw)
    pi_k, ref_k = gm.last_logps(4)
    assert rel_err(pi_k, pi_p) < 2e-3 and rel_err(ref_k, ref_p) < 2e-3
    assert abs(l_pack - l_plain) < 1e-3
    assert cosine(gm.lora_grads.double().cpu().numpy(), g_plain.double().cpu().numpy()) > 0.999


def test_shared_prefix_bitwise_claims(pair):
    ids = torch.from_numpy(_ids(54)).cuda()
    kw = dict(loss="dpo", n_pairs=2, prefix_len=PRE, beta=0.1, apply_optimizer=False, share_prefix=True)
    st, rs = pair.models["streamed"], pair.models["resident"]
    l_st = st.step(ids, **kw)
    g_st = st.lora_grads.clone()
    l_rs = rs.step(ids, **kw)
    assert l_st == l_rs and torch.equal(g_st.view(torch.int32), rs.lora_grads.view(torch.int32))
    l_sh = st.step(ids, dpo_shared_load=True, **kw)
    assert l_sh == l_st and torch.equal(g_st.view(torch.int32), st.lora_grads.view(torch.int32))
