"""The file-backed layer stack (stream_source = file): same bits as the page-locked RAM stack
and as a resident run, the same layer-load schedule, and every streamed byte read from the
file through the staging ring."""
import numpy as np
import pytest
import torch

import synth
from tests.gpu_util import Pair

pytestmark = pytest.mark.gpu

TINY4 = dict(synth.TINY, n_layers=4, name="tiny-4L")


@pytest.fixture(scope="module")
def models(tmp_path_factory):
    from layer_streamed_nf4_lut_b200.model import SoupModel
    p = Pair(TINY4, seed=18, modes=("streamed", "resident"), want_oracle=False, max_tokens=4 * 64)
    path = str(tmp_path_factory.mktemp("stack") / "tiny4.soup")
    fm = SoupModel(TINY4, mode="streamed", n_layer_buffers=2, max_tokens=4 * 64, source="file", stack_path=path)
    ram = p.models["streamed"]
    for i in range(TINY4["n_layers"]):
        fm.load_layer_nf4(i, ram.read_layer_nf4(i))
    fm.set_head(*p.head_t)
    fm.set_lora(p.params_t.clone())
    yield p, fm
    fm.close()
    p.close()


def test_file_blob_round_trip(models):
    p, fm = models
    assert fm.stats()["stream_source"] == 1
    for i in range(TINY4["n_layers"]):
        assert np.array_equal(fm.read_layer_nf4(i), p.models["streamed"].read_layer_nf4(i))


def test_file_stream_equals_ram_and_resident_bitwise(models):
    p, fm = models
    cfg = dict(TINY4, batch=4)
    ids = torch.from_numpy(synth.token_batch(cfg, 44)).cuda()
    l_file = fm.step(ids, apply_optimizer=False)
    l_ram = p.models["streamed"].step(ids, apply_optimizer=False)
    l_res = p.models["resident"].step(ids, apply_optimizer=False)
    assert l_file == l_ram == l_res
    for m in ("streamed", "resident"):
        assert torch.equal(fm.lora_grads.view(torch.int32), p.models[m].lora_grads.view(torch.int32))


def test_file_load_schedule_and_bytes(models):
    p, fm = models
    L = TINY4["n_layers"]
    cfg = dict(TINY4, batch=4)
    ids = torch.from_numpy(synth.token_batch(cfg, 45)).cuda()
    fm.step(ids, apply_optimizer=False)
    fm.reset_stats()
    fm.step(ids, apply_optimizer=False)
    st = fm.stats()
    assert st["layer_loads"] == 2 * L - 4
    assert st["file_bytes_read"] == st["layer_loads"] * fm.blob_bytes
    # DPO with one load per layer for both forwards, from the file
    pcfg = dict(cfg, n_pairs=2, prefix_len=32)
    pids = torch.from_numpy(synth.preference_batch(pcfg, 46)).cuda()
    kw = dict(loss="dpo", n_pairs=2, prefix_len=32, beta=0.1, apply_optimizer=False)
    l_f = fm.step(pids, dpo_shared_load=True, **kw)
    l_r = p.models["resident"].step(pids, **kw)
    assert l_f == l_r


def test_file_source_with_optimizer_matches_ram(models):
    p, fm = models
    cfg = dict(TINY4, batch=4)
    ids = torch.from_numpy(synth.token_batch(cfg, 47)).cuda()
    ram = p.models["streamed"]
    p0 = fm.lora_params.clone()
    ram.set_lora(p0.clone())
    for _ in range(3):
        lf = fm.step(ids, lr=1e-3, apply_optimizer=True)
        lr_ = ram.step(ids, lr=1e-3, apply_optimizer=True)
        assert lf == lr_
    assert torch.equal(fm.lora_params.view(torch.int32), ram.lora_params.view(torch.int32))
