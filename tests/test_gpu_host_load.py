"""soup_model_load_layer: float32 weights in host memory, quantised by the library on the
host into its page-locked stack.  The stored blob holds the oracle's bytes, and a model loaded
this way steps bit for bit like one quantised on the GPU from the same weights.  Also the
per-projection adapter setter against the flat parameter buffer."""
import numpy as np
import pytest
import torch

import synth
from oracle import nf4
from tests.gpu_util import Pair, bf16_tensor

pytestmark = pytest.mark.gpu

PROJ = synth.PROJ_NAMES


def test_host_load_bytes_equal_oracle_and_step_equals_device_quantised():
    from layer_streamed_nf4_lut_b200.model import SoupModel, blob_part
    cfg = dict(synth.TINY)
    ref = Pair(cfg, seed=71, modes=("streamed",), want_oracle=False)
    try:
        gm = SoupModel(cfg, mode="streamed", n_layer_buffers=2, max_tokens=64)
        try:
            for i, w in enumerate(ref.weights):
                gm.load_layer(i, {p: w[p] for p in PROJ}, ref.gamma_bits[i][0], ref.gamma_bits[i][1])
            for i, w in enumerate(ref.weights):
                blob = gm.read_layer_nf4(i)
                for j, p in enumerate(PROJ):
                    q = nf4.quantise(w[p])
                    for part, key in enumerate(("codes", "q8", "scales")):
                        off, sz = blob_part(cfg, j, part)
                        assert np.array_equal(blob[off:off + sz], np.ascontiguousarray(q[key]).view(np.uint8)), \
                            (i, p, key)
                    off, sz = blob_part(cfg, j, 3)
                    assert np.array_equal(blob[off:off + sz], np.float32(q["mean"]).reshape(1).view(np.uint8))
                for g in (0, 1):
                    off, sz = blob_part(cfg, 7 + g, 0)
                    assert np.array_equal(blob[off:off + sz], ref.gamma_bits[i][g].view(np.uint8))
            gm.set_head(*ref.head_t)
            gm.set_lora(ref.params_t.clone())
            ids = torch.from_numpy(synth.token_batch(cfg, 72)).cuda()
            l_host = gm.step(ids, apply_optimizer=False)
            l_dev = ref.models["streamed"].step(ids, apply_optimizer=False)
            assert l_host == l_dev
            assert torch.equal(gm.lora_grads.view(torch.int32), ref.models["streamed"].lora_grads.view(torch.int32))
        finally:
            gm.close()
    finally:
        ref.close()


def test_set_lora_proj_writes_the_projection_slice():
    cfg = dict(synth.TINY)
    p = Pair(cfg, seed=73, modes=("resident",), want_oracle=False)
    try:
        gm = p.models["resident"]
        ids = torch.from_numpy(synth.token_batch(cfg, 74)).cuda()
        l0 = gm.step(ids, apply_optimizer=False)
        before = gm.lora_params.clone()
        A = gm.lora_view(gm.lora_params, 1, "up", 0).clone() * 2.0
        B = gm.lora_view(gm.lora_params, 1, "up", 1).clone().cpu() * -1.0  # host memory works too
        gm.set_lora_proj(1, "up", A, B)
        assert torch.equal(gm.lora_view(gm.lora_params, 1, "up", 0), A)
        assert torch.equal(gm.lora_view(gm.lora_params, 1, "up", 1).cpu(), B)
        changed = (gm.lora_params != before).nonzero().flatten()
        from layer_streamed_nf4_lut_b200.model import lora_offset
        oa, ra, ca = lora_offset(cfg, 1, PROJ.index("up"), 0)
        ob, rb, cb = lora_offset(cfg, 1, PROJ.index("up"), 1)
        inside = ((changed >= oa) & (changed < oa + ra * ca)) | ((changed >= ob) & (changed < ob + rb * cb))
        assert bool(inside.all())
        l1 = gm.step(ids, apply_optimizer=False)
        assert l1 != l0  # the kernels see the new adapters (their bf16 copy was refreshed)
        gm.set_lora_proj(1, "up", A / 2.0, B.cuda() * -1.0)
        assert gm.step(ids, apply_optimizer=False) == l0
    finally:
        p.close()
