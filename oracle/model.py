"""Llama-style decoder layer with LoRA, the SFT and DPO losses, their backward passes and
AdamW, in float64 (oracle; test infrastructure only).

What the pages fix (see the package docstring for the page list):
* the trained model is a decoder stack, "Llama-3.1-8B-Instruct", any AutoModelForCausalLM
  text model; the base is frozen and LoRA adapters are trained (rug.gal radar "Soup ...
  layer streaming", "En detalle"; imasters "Como cabe um 8B em 4 GB");
* LoRA r and alpha are configuration values (`lora: r: 64, alpha: 16` in the soup.yaml
  example of the guillermodelpino page);
* the task is `sft`, and DPO obtains its reference log-probs from the same base with the
  LoRA adapters switched off (rug.gal "En detalle"; imasters "Do SFT para os métodos de
  preferência");
* streaming does not change the result: it only reorders when data crosses to the GPU
  (rug.gal "En detalle"; imasters "Do SFT ...", "diferença 0,0").  The oracle therefore
  defines the result of a plain resident step and has no streaming in it.

Textbook readings used where the pages are silent:
* layer: pre-norm Llama block, x1 = x + O(attn(RoPE(Q n1), RoPE(K n1), V n1)),
  x2 = x1 + D(silu(G n2) * U n2), n = RMSNorm(x) * gamma, no biases, no dropout.
* RMSNorm: x / sqrt(mean(x^2) + eps) * gamma.
* RoPE: rotate-half pairing (i, i + d/2), angle = pos * theta^(-2i/d), positions restart
  at 0 for every sequence, no frequency rescaling.
* attention: causal softmax(q k^T / sqrt(d)) v, query head h reads kv head h // (hq/hkv).
* LoRA (Hu et al. 2021): y = x W^T + (alpha/r) (x A^T) B^T on all seven projections.
* SFT loss: mean over counted targets of -log softmax(logits[j-1])[id_j]; targets are the
  positions j >= 1 of each sequence (optionally filtered by a mask on j).
* DPO (Rafailov et al. 2023): pi, ref = sums of target log-probs over the response
  (targets j >= prefix_len); L = -(1/P) sum_p log sigmoid(beta[(pi_c - ref_c) - (pi_r - ref_r)]).
* AdamW (Loshchilov & Hutter 2019) with bias correction, decoupled weight decay.
"""
from __future__ import annotations

import math
import numpy as np

PROJ = ("q", "k", "v", "o", "gate", "up", "down")


# --------------------------------------------------------------------------- basic ops
def rmsnorm(x, gamma, eps):
    """y = x * r * gamma with r = 1/sqrt(mean(x^2) + eps); returns (y, r[T,1])."""
    r = 1.0 / np.sqrt(np.mean(x * x, axis=1, keepdims=True) + eps)
    return x * r * gamma, r


def rmsnorm_backward(dy, x, r, gamma):
    """d/dx of RMSNorm (gamma frozen)."""
    gd = dy * gamma
    h = x.shape[1]
    dot = np.sum(gd * x, axis=1, keepdims=True)
    return r * gd - x * (r ** 3) * dot / h


def rope_tables(S, d, theta):
    """cos, sin of angle[pos, i] = pos * theta^(-2i/d), i < d/2."""
    i = np.arange(d // 2, dtype=np.float64)
    inv = theta ** (-(2.0 * i) / d)
    ang = np.arange(S, dtype=np.float64)[:, None] * inv[None, :]
    return np.cos(ang), np.sin(ang)


def rope(z, cos, sin):
    """Rotate-half RoPE on z[B, S, H, d]; cos/sin are [S, d/2]."""
    half = z.shape[-1] // 2
    c = cos[None, :, None, :]
    s = sin[None, :, None, :]
    z1, z2 = z[..., :half], z[..., half:]
    return np.concatenate([z1 * c - z2 * s, z2 * c + z1 * s], axis=-1)


def rope_backward(dz, cos, sin):
    """Transpose of the RoPE rotation (rotation by -angle)."""
    half = dz.shape[-1] // 2
    c = cos[None, :, None, :]
    s = sin[None, :, None, :]
    d1, d2 = dz[..., :half], dz[..., half:]
    return np.concatenate([d1 * c + d2 * s, d2 * c - d1 * s], axis=-1)


def attention_forward(q, k, v):
    """Causal GQA attention. q[B,S,hq,d], k/v[B,S,hkv,d] -> o[B,S,hq,d], lse[B,hq,S]."""
    B, S, hq, d = q.shape
    hkv = k.shape[2]
    grp = hq // hkv
    scale = 1.0 / math.sqrt(d)
    o = np.zeros_like(q)
    lse = np.zeros((B, hq, S))
    future = np.triu(np.ones((S, S), dtype=bool), 1)
    for b in range(B):
        for h in range(hq):
            g = h // grp
            s = (q[b, :, h, :] @ k[b, :, g, :].T) * scale
            s[future] = -np.inf
            mx = s.max(axis=1, keepdims=True)
            p = np.exp(s - mx)
            l = p.sum(axis=1, keepdims=True)
            lse[b, h] = (mx + np.log(l))[:, 0]
            o[b, :, h, :] = (p / l) @ v[b, :, g, :]
    return o, lse


def attention_backward(do, q, k, v, lse):
    """Gradients of causal GQA attention w.r.t. q, k, v (softmax recomputed from lse)."""
    B, S, hq, d = q.shape
    hkv = k.shape[2]
    grp = hq // hkv
    scale = 1.0 / math.sqrt(d)
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    future = np.triu(np.ones((S, S), dtype=bool), 1)
    for b in range(B):
        for h in range(hq):
            g = h // grp
            s = (q[b, :, h, :] @ k[b, :, g, :].T) * scale
            s[future] = -np.inf
            P = np.exp(s - lse[b, h][:, None])
            dv[b, :, g, :] += P.T @ do[b, :, h, :]
            dP = do[b, :, h, :] @ v[b, :, g, :].T
            dS = P * (dP - np.sum(dP * P, axis=1, keepdims=True))
            dq[b, :, h, :] = (dS @ k[b, :, g, :]) * scale
            dk[b, :, g, :] += (dS.T @ q[b, :, h, :]) * scale
    return dq, dk, dv


def silu(x):
    return x / (1.0 + np.exp(-x))


def swiglu_backward(dm, g, u):
    sig = 1.0 / (1.0 + np.exp(-g))
    dg = dm * u * sig * (1.0 + g * (1.0 - sig))
    du = dm * g * sig
    return dg, du


def lora_linear(x, W, ab, s, enabled):
    """x W^T (+ s (x A^T) B^T when the adapter is present and enabled)."""
    y = x @ W.T
    if enabled and ab is not None:
        A, B = ab
        y = y + s * ((x @ A.T) @ B.T)
    return y


def lora_linear_backward(dy, x, W, ab, s, enabled):
    """Returns (dx, dA, dB); W is frozen so it gets no gradient."""
    dx = dy @ W
    if not (enabled and ab is not None):
        return dx, None, None
    A, B = ab
    v = dy @ B
    dx = dx + s * (v @ A)
    dA = s * (v.T @ x)
    dB = s * (dy.T @ (x @ A.T))
    return dx, dA, dB


# --------------------------------------------------------------------------- layer
def layer_forward(cfg, W, lora_l, x, B, S, enabled=True):
    """One decoder layer. x[T=B*S, h] float64 -> (x2, cache)."""
    hq, hkv, d = cfg["n_heads"], cfg["n_kv_heads"], cfg["head_dim"]
    eps = cfg["rms_eps"]
    s = cfg["lora_alpha"] / cfg["lora_r"]
    lo = lora_l or {}
    T = B * S
    n1, r1 = rmsnorm(x, W["attn_norm"], eps)
    q = lora_linear(n1, W["q"], lo.get("q"), s, enabled).reshape(B, S, hq, d)
    k = lora_linear(n1, W["k"], lo.get("k"), s, enabled).reshape(B, S, hkv, d)
    v = lora_linear(n1, W["v"], lo.get("v"), s, enabled).reshape(B, S, hkv, d)
    cos, sin = rope_tables(S, d, cfg["rope_theta"])
    qr, kr = rope(q, cos, sin), rope(k, cos, sin)
    o, lse = attention_forward(qr, kr, v)
    a = o.reshape(T, hq * d)
    x1 = x + lora_linear(a, W["o"], lo.get("o"), s, enabled)
    n2, r2 = rmsnorm(x1, W["mlp_norm"], eps)
    g = lora_linear(n2, W["gate"], lo.get("gate"), s, enabled)
    u = lora_linear(n2, W["up"], lo.get("up"), s, enabled)
    m = silu(g) * u
    x2 = x1 + lora_linear(m, W["down"], lo.get("down"), s, enabled)
    cache = dict(x=x, n1=n1, r1=r1, qr=qr, kr=kr, v=v, lse=lse, a=a, x1=x1, n2=n2, r2=r2,
                 g=g, u=u, m=m, cos=cos, sin=sin)
    return x2, cache


def layer_backward(cfg, W, lora_l, cache, dx2, B, S, enabled=True):
    """Backward of layer_forward. Returns (dx, {proj: (dA, dB)})."""
    hq, hkv, d = cfg["n_heads"], cfg["n_kv_heads"], cfg["head_dim"]
    s = cfg["lora_alpha"] / cfg["lora_r"]
    lo = lora_l or {}
    T = B * S
    grads = {}
    dm, dA, dB = lora_linear_backward(dx2, cache["m"], W["down"], lo.get("down"), s, enabled)
    grads["down"] = (dA, dB)
    dg, du = swiglu_backward(dm, cache["g"], cache["u"])
    dn2g, dA, dB = lora_linear_backward(dg, cache["n2"], W["gate"], lo.get("gate"), s, enabled)
    grads["gate"] = (dA, dB)
    dn2u, dA, dB = lora_linear_backward(du, cache["n2"], W["up"], lo.get("up"), s, enabled)
    grads["up"] = (dA, dB)
    dx1 = dx2 + rmsnorm_backward(dn2g + dn2u, cache["x1"], cache["r2"], W["mlp_norm"])
    da, dA, dB = lora_linear_backward(dx1, cache["a"], W["o"], lo.get("o"), s, enabled)
    grads["o"] = (dA, dB)
    dqr, dkr, dv = attention_backward(da.reshape(B, S, hq, d), cache["qr"], cache["kr"], cache["v"], cache["lse"])
    dq = rope_backward(dqr, cache["cos"], cache["sin"]).reshape(T, hq * d)
    dk = rope_backward(dkr, cache["cos"], cache["sin"]).reshape(T, hkv * d)
    dv = dv.reshape(T, hkv * d)
    dn1 = np.zeros_like(cache["n1"])
    for p, dyp in (("q", dq), ("k", dk), ("v", dv)):
        dxp, dA, dB = lora_linear_backward(dyp, cache["n1"], W[p], lo.get(p), s, enabled)
        dn1 += dxp
        grads[p] = (dA, dB)
    dx = dx1 + rmsnorm_backward(dn1, cache["x"], cache["r1"], W["attn_norm"])
    return dx, grads


# --------------------------------------------------------------------------- head + losses
def head_forward(cfg, head, xL):
    hf, rf = rmsnorm(xL, head["final_norm"], cfg["rms_eps"])
    return hf @ head["lm_head"].T, (xL, rf)


def head_backward(head, hcache, dlogits):
    xL, rf = hcache
    return rmsnorm_backward(dlogits @ head["lm_head"], xL, rf, head["final_norm"])


def log_softmax(logits):
    mx = logits.max(axis=1, keepdims=True)
    lse = mx + np.log(np.sum(np.exp(logits - mx), axis=1, keepdims=True))
    return logits - lse


def sft_loss(logits, ids, mask=None):
    """Token-mean next-token cross-entropy. logits[B*S, V], ids[B, S], mask[B, S] on targets.

    Returns (loss, dlogits)."""
    B, S = ids.shape
    V = logits.shape[1]
    lp = log_softmax(logits).reshape(B, S, V)
    valid = np.zeros((B, S), dtype=bool)
    valid[:, 1:] = True
    if mask is not None:
        valid &= mask.astype(bool)
    n = int(valid.sum())
    dl = np.zeros((B, S, V))
    loss = 0.0
    if n == 0:
        return 0.0, dl.reshape(B * S, V)
    for b in range(B):
        for j in range(1, S):
            if not valid[b, j]:
                continue
            t = ids[b, j]
            loss -= lp[b, j - 1, t]
            dl[b, j - 1] = np.exp(lp[b, j - 1]) / n
            dl[b, j - 1, t] -= 1.0 / n
    return loss / n, dl.reshape(B * S, V)


def sequence_logps(logits, ids, start):
    """Per-row sum of log p(id_j | prefix) over targets j in [max(start,1), S)."""
    B, S = ids.shape
    V = logits.shape[1]
    lp = log_softmax(logits).reshape(B, S, V)
    out = np.zeros(B)
    for b in range(B):
        for j in range(max(start, 1), S):
            out[b] += lp[b, j - 1, ids[b, j]]
    return out, lp


def dpo_loss(pi, ref, beta):
    """Rows 2p (chosen) and 2p+1 (rejected). Returns (loss, dL/dpi)."""
    P = len(pi) // 2
    dpi = np.zeros_like(pi)
    loss = 0.0
    for p in range(P):
        z = beta * ((pi[2 * p] - ref[2 * p]) - (pi[2 * p + 1] - ref[2 * p + 1]))
        loss += np.logaddexp(0.0, -z)        # -log sigmoid(z)
        sneg = 1.0 / (1.0 + np.exp(z))        # sigmoid(-z)
        dpi[2 * p] = -beta * sneg / P
        dpi[2 * p + 1] = beta * sneg / P
    return loss / P, dpi


def dpo_dlogits(lp, ids, start, dpi):
    """dL/dlogits given dL/dpi: dpi[b] * (onehot - softmax) on response targets."""
    B, S, V = lp.shape
    dl = np.zeros((B, S, V))
    for b in range(B):
        for j in range(max(start, 1), S):
            dl[b, j - 1] = -dpi[b] * np.exp(lp[b, j - 1])
            dl[b, j - 1, ids[b, j]] += dpi[b]
    return dl.reshape(B * S, V)


# --------------------------------------------------------------------------- whole model
def forward(cfg, layers, lora, head, ids, enabled=True):
    B, S = ids.shape
    x = head["embed"][ids.reshape(-1)]
    caches = []
    for i, W in enumerate(layers):
        x, c = layer_forward(cfg, W, _lora_of(lora, i), x, B, S, enabled)
        caches.append(c)
    logits, hc = head_forward(cfg, head, x)
    return logits, caches, hc


def backward(cfg, layers, lora, head, caches, hc, dlogits, B, S, enabled=True):
    dx = head_backward(head, hc, dlogits)
    grads = {}
    for i in reversed(range(len(layers))):
        dx, g = layer_backward(cfg, layers[i], _lora_of(lora, i), caches[i], dx, B, S, enabled)
        for p, ab in g.items():
            grads[(i, p)] = ab
    return grads


def sft_step(cfg, layers, lora, head, ids, mask=None, enabled=True):
    """Loss and LoRA gradients of one SFT step."""
    B, S = ids.shape
    logits, caches, hc = forward(cfg, layers, lora, head, ids, enabled)
    loss, dl = sft_loss(logits, ids, mask)
    grads = backward(cfg, layers, lora, head, caches, hc, dl, B, S, enabled)
    return loss, grads, logits


def dpo_step(cfg, layers, lora, head, ids, prefix_len, beta):
    """Loss and LoRA gradients of one DPO step; reference = same base with LoRA off."""
    B, S = ids.shape
    ref_logits, _, _ = forward(cfg, layers, lora, head, ids, enabled=False)
    ref, _ = sequence_logps(ref_logits, ids, prefix_len)
    logits, caches, hc = forward(cfg, layers, lora, head, ids, enabled=True)
    pi, lp = sequence_logps(logits, ids, prefix_len)
    loss, dpi = dpo_loss(pi, ref, beta)
    dl = dpo_dlogits(lp, ids, prefix_len, dpi)
    grads = backward(cfg, layers, lora, head, caches, hc, dl, B, S, True)
    return loss, grads, dict(pi=pi, ref=ref)


def adamw(p, g, m, v, t, lr, b1=0.9, b2=0.999, eps=1e-8, wd=0.0):
    """One AdamW update (step number t >= 1). Returns new (p, m, v)."""
    m = b1 * m + (1.0 - b1) * g
    v = b2 * v + (1.0 - b2) * g * g
    mh = m / (1.0 - b1 ** t)
    vh = v / (1.0 - b2 ** t)
    p = p - lr * (mh / (np.sqrt(vh) + eps) + wd * p)
    return p, m, v


def bf16_round_f64(x):
    """float64 -> nearest bfloat16 value (ties to even) in ONE rounding, as float64.

    Normal-range finite inputs; the significand keeps 8 bits (frexp mantissa in [0.5, 1))."""
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)
    return np.ldexp(np.rint(m * 256.0), e - 8)


def merge_lora(W, A, B, s):
    """Merged weight of one projection: the base fused with its LoRA adapter.

    The pages list a merge command that fuses the trained adapter into the base model
    (guillermodelpino page, the commands of the full cycle: `soup merge --adapter`;
    imasters page, "O que muda para quem constrói no Brasil": merging the LoRA into the
    base).  They give no formula; the plainest reading is the LoRA identity (Hu et al.
    2021): x W'^T = x W^T + s (x A^T) B^T for every x, i.e. W' = W + s B A, stored in the
    working precision of the weights (bf16).  A and B enter with the precision the training
    forward gives them (bf16 values); the sum is exact here and rounded once.

    W: [out, in] dequantised base (bf16 values); A: [r, in]; B: [out, r]; s = alpha / r.
    Returns float64 values that are bf16 numbers."""
    from .nf4 import bf16_round
    Ab = bf16_round(np.asarray(A, dtype=np.float32)).astype(np.float64)
    Bb = bf16_round(np.asarray(B, dtype=np.float32)).astype(np.float64)
    return bf16_round_f64(np.asarray(W, dtype=np.float64) + s * (Bb @ Ab))


def _lora_of(lora, i):
    if lora is None:
        return None
    return {p: lora[(i, p)] for p in PROJ if (i, p) in lora}


# --------------------------------------------------------------------------- inputs
def model_from_quantised(cfg, qlayers, head_bits):
    """Build float64 weights from oracle-quantised layers and bf16 head bit patterns.

    qlayers[i] = {proj: nf4 dict, 'attn_norm': bf16 bits, 'mlp_norm': bf16 bits}."""
    from . import nf4
    layers = []
    for ql in qlayers:
        W = {p: nf4.dequant(ql[p]).astype(np.float64) for p in PROJ}
        W["attn_norm"] = nf4.bf16_bits_to_f64(ql["attn_norm"])
        W["mlp_norm"] = nf4.bf16_bits_to_f64(ql["mlp_norm"])
        layers.append(W)
    emb, lm, g = head_bits
    head = dict(embed=nf4.bf16_bits_to_f64(emb), lm_head=nf4.bf16_bits_to_f64(lm), final_norm=nf4.bf16_bits_to_f64(g))
    return layers, head


def step_flops(cfg, T, S):
    """Algorithmic FLOPs of one SFT step over T tokens in sequences of length S: frozen
    GEMMs forward + dX, LoRA forward + backward, causal attention, lm_head fwd + dX."""
    h, I, V, L = cfg["hidden"], cfg["intermediate"], cfg["vocab"], cfg["n_layers"]
    hq, hkv, d, r = cfg["n_heads"], cfg["n_kv_heads"], cfg["head_dim"], cfg["lora_r"]
    p_layer = h * hq * d + 2 * h * hkv * d + hq * d * h + 3 * h * I
    io = (h + hq * d) + 2 * (h + hkv * d) + (hq * d + h) + 2 * (h + I) + (I + h)
    per_tok = 4 * p_layer + 6 * r * io + 6 * S * d * hq
    return L * per_tok * T + 4 * h * V * T
