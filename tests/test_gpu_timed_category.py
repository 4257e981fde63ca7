"""Timed category (soup_set_timed_category): event pairs around one kernel category's launches
in ordinary calls, including the replayed layer graphs.  Checks the launch count over eager,
capturing and replaying steps, that the instrumentation leaves every result bitwise unchanged,
and that an unknown category is refused."""
import pytest
import torch

import synth
from tests.gpu_util import Pair

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def pair():
    p = Pair(dict(synth.TINY), seed=13, modes=("streamed",), want_oracle=False)
    yield p
    p.close()


def test_timed_category_counts_and_bits(pair):
    gm = pair.models["streamed"]
    cfg = pair.cfg
    ids = torch.from_numpy(synth.token_batch(cfg, 41)).cuda()
    kw = dict(apply_optimizer=False)
    ref = [gm.step(ids, **kw) for _ in range(3)]  # eager, capture, replay without events
    g_ref = gm.lora_grads.clone()
    gm.set_timed_category("gemm_nf4_fwd")
    got = [gm.step(ids, **kw) for _ in range(3)]  # new graph key: eager, capture, replay
    t = gm.timed_category(reset=True)
    assert got == ref
    assert torch.equal(gm.lora_grads.view(torch.int32), g_ref.view(torch.int32))
    # q|k|v, o, gate|up and down forward GEMMs of every layer, every step
    assert t["name"] == "gemm_nf4_fwd"
    assert t["launches"] == 3 * 4 * cfg["n_layers"]
    assert t["total_ms"] > 0 and t["flops"] > 0
    gm.step(ids, **kw)
    t2 = gm.timed_category(reset=True)
    assert t2["launches"] == 4 * cfg["n_layers"]
    gm.set_timed_category(None)
    gm.step(ids, **kw)
    assert gm.timed_category()["launches"] == 0


def test_timed_all_categories(pair):
    gm = pair.models["streamed"]
    cfg = pair.cfg
    L = cfg["n_layers"]
    ids = torch.from_numpy(synth.token_batch(cfg, 42)).cuda()
    ref = gm.step(ids, apply_optimizer=False)
    gm.set_timed_category("all")
    for _ in range(2):  # eager, capture
        assert gm.step(ids, apply_optimizer=False) == ref
    gm.timed_profile(reset=True)
    st0 = gm.stats()["layer_loads"]
    assert gm.step(ids, apply_optimizer=False) == ref
    prof = gm.timed_profile(reset=True)
    gm.set_timed_category(None)
    assert prof["gemm_nf4_fwd"]["launches"] == 4 * L
    assert prof["gemm_nf4_dx"]["launches"] == 4 * L
    assert prof["gemm_lm_head_fwd"]["launches"] == 1 and prof["gemm_lm_head_dx"]["launches"] == 1
    assert prof.get("h2d_layer_copy", {"launches": 0})["launches"] == gm.stats()["layer_loads"] - st0
    assert all(v["total_ms"] > 0 for v in prof.values())


def test_timed_category_set_of_two(pair):
    gm = pair.models["streamed"]
    L = pair.cfg["n_layers"]
    ids = torch.from_numpy(synth.token_batch(pair.cfg, 43)).cuda()
    gm.set_timed_category("gemm_nf4_fwd,gemm_nf4_dx")
    for _ in range(3):
        gm.step(ids, apply_optimizer=False)
    prof = gm.timed_profile()
    t = gm.timed_category(reset=True)
    gm.set_timed_category(None)
    assert t["name"] == "gemm_nf4_fwd,gemm_nf4_dx"
    assert prof["gemm_nf4_fwd"]["launches"] == prof["gemm_nf4_dx"]["launches"] == 3 * 4 * L
    assert t["launches"] == 2 * 3 * 4 * L
    assert abs(t["total_ms"] - prof["gemm_nf4_fwd"]["total_ms"] - prof["gemm_nf4_dx"]["total_ms"]) < 1e-6
    # one empty calibration launch per layer call (forward and backward), not in the totals
    assert prof["event_overhead"]["launches"] >= 2 * L


def test_timed_category_unknown_name(pair):
    gm = pair.models["streamed"]
    with pytest.raises(Exception):
        gm.set_timed_category("no_such_kernel")
    with pytest.raises(Exception):
        gm.set_timed_category("gemm_nf4_fwd,event_overhead")
