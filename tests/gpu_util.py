"""Builds a libsoup model and the matching float64 oracle model from the same seeded
inputs (synth), for the GPU parity tests.  The oracle quantises with its own code; the
library quantises on the GPU; the two never share code."""
from __future__ import annotations

import numpy as np
import torch

import synth
from oracle import model as om
from oracle import nf4

PROJ = synth.PROJ_NAMES


def bf16_tensor(bits: np.ndarray, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits, np.uint16).view(np.int16)).view(torch.bfloat16).to(device)


def to64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def rel_err(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30))


def cosine(a, b):
    a = np.asarray(a, np.float64).ravel()
    b = np.asarray(b, np.float64).ravel()
    return float(a @ b / max(np.linalg.norm(a) * np.linalg.norm(b), 1e-300))


class Pair:
    """A GPU model and the oracle's float64 weights for the same synthetic inputs."""

    def __init__(self, cfg, seed=0, modes=("streamed",), gamma_noise=0.1, zero_b=False, max_tokens=None,
                 n_layer_buffers=2, want_oracle=True, w_std=0.02):
        from layer_streamed_nf4_lut_b200.model import SoupModel
        self.cfg = cfg
        L = cfg["n_layers"]
        self.weights = [synth.layer_weights(cfg, seed, i, std=w_std, gamma_noise=gamma_noise) for i in range(L)]
        self.head_bits = synth.head_weights(cfg, seed, gamma_noise=gamma_noise)
        self.lora = synth.lora_weights(cfg, seed, zero_b=zero_b)
        self.gamma_bits = [(synth.bf16_bits_from_f32(w["attn_norm"]), synth.bf16_bits_from_f32(w["mlp_norm"]))
                           for w in self.weights]
        if want_oracle:
            qlayers = []
            for i, w in enumerate(self.weights):
                q = {p: nf4.quantise(w[p]) for p in PROJ}
                q["attn_norm"], q["mlp_norm"] = self.gamma_bits[i]
                qlayers.append(q)
            self.qlayers = qlayers
            self.olayers, self.ohead = om.model_from_quantised(cfg, qlayers, self.head_bits)
            self.olora = {k: (a.astype(np.float64), b.astype(np.float64)) for k, (a, b) in self.lora.items()}
        mt = max_tokens if max_tokens is not None else cfg["batch"] * cfg["seq"]
        self.models = {}
        emb, lm, g = self.head_bits
        self.head_t = (bf16_tensor(emb), bf16_tensor(g), bf16_tensor(lm))
        self.params_t = self.flat_lora()
        for mode in modes:
            gm = SoupModel(cfg, mode=mode, n_layer_buffers=n_layer_buffers, max_tokens=mt)
            for i, w in enumerate(self.weights):
                wt = {p: torch.from_numpy(w[p]).cuda() for p in PROJ}
                gm.quantize_layer(i, wt, bf16_tensor(self.gamma_bits[i][0]), bf16_tensor(self.gamma_bits[i][1]))
                del wt
            gm.set_head(*self.head_t)
            gm.set_lora(self.params_t.clone())
            self.models[mode] = gm

    def flat_lora(self) -> torch.Tensor:
        from layer_streamed_nf4_lut_b200.model import lora_numel, lora_offset
        flat = np.zeros(lora_numel(self.cfg), np.float32)
        for (layer, p), (A, B) in self.lora.items():
            j = PROJ.index(p)
            oa, _, _ = lora_offset(self.cfg, layer, j, 0)
            ob, _, _ = lora_offset(self.cfg, layer, j, 1)
            flat[oa:oa + A.size] = A.ravel()
            flat[ob:ob + B.size] = B.ravel()
        return torch.from_numpy(flat).cuda()

    def gpu_grads(self, mode):
        gm = self.models[mode]
        out = {}
        for layer in range(self.cfg["n_layers"]):
            for p in PROJ:
                out[(layer, p)] = (to64(gm.lora_view(gm.lora_grads, layer, p, 0)),
                                   to64(gm.lora_view(gm.lora_grads, layer, p, 1)))
        return out

    def close(self):
        for gm in self.models.values():
            gm.close()
        self.models = {}
