"""Pins for the float64 layer / loss / optimizer oracle: closed forms, special cases that
reduce to library routines, finite differences and autograd on tiny shapes."""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import model as om

torch.set_default_dtype(torch.float64)

TINYCFG = dict(n_layers=2, hidden=32, n_heads=4, n_kv_heads=2, head_dim=8, intermediate=48, vocab=64,
               rms_eps=1e-5, rope_theta=5e5, lora_r=4, lora_alpha=8.0)


def _rand_model(cfg, seed=0, zero_b=False, std=0.2):
    rng = np.random.default_rng(seed)
    h, I, V, r = cfg["hidden"], cfg["intermediate"], cfg["vocab"], cfg["lora_r"]
    hq, hkv, d = cfg["n_heads"], cfg["n_kv_heads"], cfg["head_dim"]
    shapes = dict(q=(hq * d, h), k=(hkv * d, h), v=(hkv * d, h), o=(h, hq * d), gate=(I, h), up=(I, h), down=(h, I))
    layers, lora = [], {}
    for i in range(cfg["n_layers"]):
        W = {p: rng.standard_normal(s) * std for p, s in shapes.items()}
        W["attn_norm"] = 1.0 + 0.1 * rng.standard_normal(h)
        W["mlp_norm"] = 1.0 + 0.1 * rng.standard_normal(h)
        layers.append(W)
        for p, (o, n_in) in shapes.items():
            A = rng.uniform(-1, 1, (r, n_in)) / math.sqrt(n_in)
            B = rng.standard_normal((o, r)) * 0.1
            if zero_b:
                B = np.zeros_like(B)
            lora[(i, p)] = (A, B)
    head = dict(embed=rng.standard_normal((V, h)) * 0.5, lm_head=rng.standard_normal((V, h)) * 0.2,
                final_norm=1.0 + 0.1 * rng.standard_normal(h))
    return layers, lora, head


def test_rmsnorm_closed_form():
    rng = np.random.default_rng(0)
    x = rng.standard_normal((5, 64)) * 3
    y, r = om.rmsnorm(x, np.ones(64), 1e-5)
    ms = np.mean(x * x, axis=1)
    assert np.allclose(np.mean(y * y, axis=1), ms / (ms + 1e-5), rtol=1e-13)
    g = rng.standard_normal(64)
    yt = F.rms_norm(torch.from_numpy(x), (64,), torch.from_numpy(g), eps=1e-5).numpy()
    assert np.allclose(om.rmsnorm(x, g, 1e-5)[0], yt, rtol=1e-12, atol=1e-14)


def test_rope_complex_form_identity_and_norm():
    rng = np.random.default_rng(1)
    B, S, H, d = 2, 7, 3, 16
    z = rng.standard_normal((B, S, H, d))
    cos, sin = om.rope_tables(S, d, 5e5)
    out = om.rope(z, cos, sin)
    # complex formulation: (z1 + i z2) * exp(i * pos * theta^(-2k/d))
    zc = z[..., :d // 2] + 1j * z[..., d // 2:]
    k = np.arange(d // 2)
    ang = np.arange(S)[:, None] * (5e5 ** (-2.0 * k / d))[None, :]
    rc = zc * np.exp(1j * ang)[None, :, None, :]
    assert np.allclose(out, np.concatenate([rc.real, rc.imag], axis=-1), atol=1e-13)
    assert np.allclose(out[:, 0], z[:, 0], atol=0)  # position 0 is the identity
    assert np.allclose(np.linalg.norm(out, axis=-1), np.linalg.norm(z, axis=-1), rtol=1e-13)
    # backward is the transpose of the rotation
    dz = rng.standard_normal(z.shape)
    assert np.isclose(np.sum(om.rope_backward(dz, cos, sin) * z), np.sum(dz * out), rtol=1e-12)


def test_attention_s1_returns_v():
    rng = np.random.default_rng(2)
    q = rng.standard_normal((2, 1, 4, 8))
    k = rng.standard_normal((2, 1, 2, 8))
    v = rng.standard_normal((2, 1, 2, 8))
    o, lse = om.attention_forward(q, k, v)
    assert np.allclose(o[:, 0, 0], v[:, 0, 0]) and np.allclose(o[:, 0, 3], v[:, 0, 1])


@pytest.mark.parametrize("hq,hkv", [(4, 4), (4, 2), (6, 1)])
def test_attention_vs_torch_sdpa_gqa(hq, hkv):
    rng = np.random.default_rng(3)
    B, S, d = 2, 9, 8
    q = rng.standard_normal((B, S, hq, d))
    k = rng.standard_normal((B, S, hkv, d))
    v = rng.standard_normal((B, S, hkv, d))
    o, lse = om.attention_forward(q, k, v)
    tq, tk, tv = (torch.from_numpy(a).permute(0, 2, 1, 3) for a in (q, k, v))
    tk = tk.repeat_interleave(hq // hkv, dim=1)
    tv = tv.repeat_interleave(hq // hkv, dim=1)
    ref = F.scaled_dot_product_attention(tq, tk, tv, is_causal=True).permute(0, 2, 1, 3).numpy()
    assert np.allclose(o, ref, atol=1e-12)
    # lse: log sum exp of the causal scores
    s = torch.einsum("bhqd,bhkd->bhqk", tq, tk) / math.sqrt(d)
    s = s.masked_fill(torch.triu(torch.ones(S, S, dtype=torch.bool), 1), float("-inf"))
    assert np.allclose(lse, torch.logsumexp(s, -1).numpy(), atol=1e-12)


def test_attention_backward_vs_autograd():
    rng = np.random.default_rng(4)
    B, S, hq, hkv, d = 2, 6, 4, 2, 8
    q, k, v = rng.standard_normal((B, S, hq, d)), rng.standard_normal((B, S, hkv, d)), rng.standard_normal((B, S, hkv, d))
    do = rng.standard_normal((B, S, hq, d))
    o, lse = om.attention_forward(q, k, v)
    dq, dk, dv = om.attention_backward(do, q, k, v, lse)
    tq, tk, tv = (torch.from_numpy(a).requires_grad_() for a in (q, k, v))
    ref = F.scaled_dot_product_attention(tq.permute(0, 2, 1, 3), tk.permute(0, 2, 1, 3).repeat_interleave(2, 1),
                                         tv.permute(0, 2, 1, 3).repeat_interleave(2, 1), is_causal=True)
    ref.permute(0, 2, 1, 3).backward(torch.from_numpy(do))
    assert np.allclose(dq, tq.grad.numpy(), atol=1e-12)
    assert np.allclose(dk, tk.grad.numpy(), atol=1e-12)
    assert np.allclose(dv, tv.grad.numpy(), atol=1e-12)


def test_swiglu_vs_torch():
    rng = np.random.default_rng(5)
    g, u, dm = rng.standard_normal((3, 50)) * 4
    tg, tu = torch.from_numpy(g).requires_grad_(), torch.from_numpy(u).requires_grad_()
    (F.silu(tg) * tu).backward(torch.from_numpy(dm))
    dg, du = om.swiglu_backward(dm, g, u)
    assert np.allclose(om.silu(g), F.silu(torch.from_numpy(g)).numpy(), rtol=1e-14)
    assert np.allclose(dg, tg.grad.numpy(), atol=1e-13) and np.allclose(du, tu.grad.numpy(), atol=1e-13)


def test_ce_zero_head_is_log_vocab_and_rows_sum_zero():
    rng = np.random.default_rng(6)
    V = 1024
    ids = rng.integers(0, V, (2, 9))
    loss, dl = om.sft_loss(np.zeros((18, V)), ids)
    assert loss == pytest.approx(math.log(V), rel=1e-15)  # ln 1024 = 6.9315
    logits = rng.standard_normal((18, V)) * 3
    loss, dl = om.sft_loss(logits, ids)
    assert np.allclose(dl.sum(axis=1), 0.0, atol=1e-15)
    # against torch's cross_entropy on the shifted targets
    lt = torch.from_numpy(logits).reshape(2, 9, V)[:, :-1].reshape(-1, V)
    assert loss == pytest.approx(F.cross_entropy(lt, torch.from_numpy(ids[:, 1:].reshape(-1))).item(), rel=1e-13)


def test_ce_mask_last_half():
    rng = np.random.default_rng(7)
    V, S = 50, 8
    ids = rng.integers(0, V, (2, S))
    logits = rng.standard_normal((2 * S, V))
    mask = np.zeros((2, S), np.uint8)
    mask[:, S // 2:] = 1
    loss, dl = om.sft_loss(logits, ids, mask)
    lt = torch.from_numpy(logits).reshape(2, S, V)[:, S // 2 - 1:S - 1].reshape(-1, V)
    assert loss == pytest.approx(F.cross_entropy(lt, torch.from_numpy(ids[:, S // 2:].reshape(-1))).item(), rel=1e-13)
    assert np.all(dl.reshape(2, S, V)[:, :S // 2 - 1] == 0) and np.all(dl.reshape(2, S, V)[:, -1] == 0)


def test_dpo_closed_forms():
    beta, P = 0.1, 2
    pi = np.array([-10.0, -12.0, -7.0, -7.5])
    loss, dpi = om.dpo_loss(pi, pi.copy(), beta)
    assert loss == pytest.approx(math.log(2), rel=1e-15)
    assert np.allclose(dpi, [-beta / (2 * P), beta / (2 * P)] * P, rtol=1e-15)
    ref = np.array([-11.0, -11.0, -8.0, -7.0])
    loss, dpi = om.dpo_loss(pi, ref, beta)
    z = beta * np.array([(pi[0] - ref[0]) - (pi[1] - ref[1]), (pi[2] - ref[2]) - (pi[3] - ref[3])])
    assert loss == pytest.approx(-F.logsigmoid(torch.from_numpy(z)).mean().item(), rel=1e-14)
    # swapping chosen and rejected flips z
    sw = np.array([1, 0, 3, 2])
    loss2, _ = om.dpo_loss(pi[sw], ref[sw], beta)
    assert loss2 == pytest.approx(-F.logsigmoid(torch.from_numpy(-z)).mean().item(), rel=1e-14)


def test_lora_zero_b_and_disabled_equal_base():
    cfg = TINYCFG
    layers, lora0, head = _rand_model(cfg, seed=1, zero_b=True)
    ids = np.random.default_rng(8).integers(0, cfg["vocab"], (2, 6))
    l_base, _, _ = om.forward(cfg, layers, None, head, ids)
    l_b0, _, _ = om.forward(cfg, layers, lora0, head, ids)
    assert np.array_equal(l_base, l_b0)
    layers, lora, head = _rand_model(cfg, seed=1)
    l_off, _, _ = om.forward(cfg, layers, lora, head, ids, enabled=False)
    l_on, _, _ = om.forward(cfg, layers, lora, head, ids, enabled=True)
    assert np.array_equal(l_off, l_base)
    assert not np.allclose(l_on, l_base)


def _fd_check(fn, params, grads, picks, h=1e-6, tol=1e-6):
    for key, which, idx in picks:
        arr = params[key][which]
        g = grads[key][which][idx]
        old = arr[idx]
        arr[idx] = old + h
        lp = fn()
        arr[idx] = old - h
        lm = fn()
        arr[idx] = old
        fd = (lp - lm) / (2 * h)
        assert abs(fd - g) <= tol * max(1.0, abs(g), abs(fd)) + 1e-9, (key, which, idx, fd, g)


def test_sft_gradients_finite_difference():
    cfg = TINYCFG
    layers, lora, head = _rand_model(cfg, seed=2)
    lora = {k: [a.copy(), b.copy()] for k, (a, b) in lora.items()}
    rng = np.random.default_rng(9)
    ids = rng.integers(0, cfg["vocab"], (2, 6))
    mask = (rng.uniform(size=(2, 6)) > 0.3).astype(np.uint8)
    loss, grads, _ = om.sft_step(cfg, layers, lora, head, ids, mask)
    fn = lambda: om.sft_step(cfg, layers, lora, head, ids, mask)[0]
    picks = []
    for i in range(cfg["n_layers"]):
        for p in om.PROJ:
            A, B = lora[(i, p)]
            picks.append(((i, p), 0, (int(rng.integers(A.shape[0])), int(rng.integers(A.shape[1])))))
            picks.append(((i, p), 1, (int(rng.integers(B.shape[0])), int(rng.integers(B.shape[1])))))
    _fd_check(fn, lora, {k: list(v) for k, v in grads.items()}, picks)


def test_layer_input_gradient_finite_difference():
    cfg = TINYCFG
    layers, lora, head = _rand_model(cfg, seed=3)
    rng = np.random.default_rng(10)
    B, S = 2, 5
    x = rng.standard_normal((B * S, cfg["hidden"]))
    w = rng.standard_normal((B * S, cfg["hidden"]))
    lo = {p: lora[(0, p)] for p in om.PROJ}
    y, cache = om.layer_forward(cfg, layers[0], lo, x, B, S)
    dx, _ = om.layer_backward(cfg, layers[0], lo, cache, w, B, S)
    for _ in range(12):
        t, c = int(rng.integers(B * S)), int(rng.integers(cfg["hidden"]))
        xp, xm = x.copy(), x.copy()
        xp[t, c] += 1e-6
        xm[t, c] -= 1e-6
        fd = (np.sum(om.layer_forward(cfg, layers[0], lo, xp, B, S)[0] * w) -
              np.sum(om.layer_forward(cfg, layers[0], lo, xm, B, S)[0] * w)) / 2e-6
        assert abs(fd - dx[t, c]) <= 1e-6 * max(1.0, abs(fd))


def test_dpo_gradients_finite_difference():
    cfg = dict(TINYCFG, n_layers=1)
    layers, lora, head = _rand_model(cfg, seed=4)
    lora = {k: [a.copy(), b.copy()] for k, (a, b) in lora.items()}
    rng = np.random.default_rng(11)
    S, pre = 7, 3
    ids = rng.integers(0, cfg["vocab"], (4, S))
    ids[1, :pre] = ids[0, :pre]
    ids[3, :pre] = ids[2, :pre]
    loss, grads, aux = om.dpo_step(cfg, layers, lora, head, ids, pre, 0.1)
    fn = lambda: om.dpo_step(cfg, layers, lora, head, ids, pre, 0.1)[0]
    picks = [((0, p), w, (0, 1)) for p in om.PROJ for w in (0, 1)]
    _fd_check(fn, lora, {k: list(v) for k, v in grads.items()}, picks, tol=1e-5)
    # at the initial point (B != 0) policy != ref; with B = 0 they coincide and L = ln 2
    layers0, lora0, head0 = _rand_model(cfg, seed=4, zero_b=True)
    l0, _, aux0 = om.dpo_step(cfg, layers0, lora0, head0, ids, pre, 0.1)
    assert np.array_equal(aux0["pi"], aux0["ref"]) and l0 == pytest.approx(math.log(2), rel=1e-14)


def test_layer_against_torch_autograd():
    """Forward with torch library ops, backward by autograd, against the hand-derived one."""
    cfg = TINYCFG
    layers, lora, head = _rand_model(cfg, seed=5)
    rng = np.random.default_rng(12)
    B, S = 2, 6
    hq, hkv, d, h = cfg["n_heads"], cfg["n_kv_heads"], cfg["head_dim"], cfg["hidden"]
    s = cfg["lora_alpha"] / cfg["lora_r"]
    x = rng.standard_normal((B * S, h))
    wout = rng.standard_normal((B * S, h))
    lo = {p: lora[(0, p)] for p in om.PROJ}
    W = layers[0]
    y, cache = om.layer_forward(cfg, W, lo, x, B, S)
    dx, grads = om.layer_backward(cfg, W, lo, cache, wout, B, S)

    T = lambda a: torch.from_numpy(np.ascontiguousarray(a))
    tx = T(x).requires_grad_()
    tl = {p: (T(a).requires_grad_(), T(b).requires_grad_()) for p, (a, b) in lo.items()}
    lin = lambda z, p: F.linear(z, T(W[p])) + s * F.linear(F.linear(z, tl[p][0]), tl[p][1])
    n1 = F.rms_norm(tx, (h,), T(W["attn_norm"]), eps=1e-5)
    q = lin(n1, "q").reshape(B, S, hq, d)
    k = lin(n1, "k").reshape(B, S, hkv, d)
    v = lin(n1, "v").reshape(B, S, hkv, d)
    pos = torch.arange(S, dtype=torch.float64)[:, None]
    inv = 5e5 ** (-(2.0 * torch.arange(d // 2, dtype=torch.float64)) / d)
    ang = pos * inv
    def rot(z):
        zc = torch.complex(z[..., :d // 2], z[..., d // 2:]) * torch.polar(torch.ones_like(ang), ang)[None, :, None, :]
        return torch.cat([zc.real, zc.imag], -1)
    qr, kr = rot(q), rot(k)
    o = F.scaled_dot_product_attention(qr.transpose(1, 2), kr.transpose(1, 2).repeat_interleave(hq // hkv, 1),
                                       v.transpose(1, 2).repeat_interleave(hq // hkv, 1), is_causal=True)
    a = o.transpose(1, 2).reshape(B * S, hq * d)
    x1 = tx + lin(a, "o")
    n2 = F.rms_norm(x1, (h,), T(W["mlp_norm"]), eps=1e-5)
    x2 = x1 + lin(F.silu(lin(n2, "gate")) * lin(n2, "up"), "down")
    assert np.allclose(x2.detach().numpy(), y, atol=1e-12)
    x2.backward(T(wout))
    assert np.allclose(tx.grad.numpy(), dx, atol=1e-11)
    for p in om.PROJ:
        assert np.allclose(tl[p][0].grad.numpy(), grads[p][0], atol=1e-11), p
        assert np.allclose(tl[p][1].grad.numpy(), grads[p][1], atol=1e-11), p


def test_adamw_first_step_sign_and_vs_torch():
    rng = np.random.default_rng(13)
    p0 = rng.standard_normal(100)
    gs = [rng.standard_normal(100) for _ in range(4)]
    p, m, v = om.adamw(p0, gs[0], np.zeros(100), np.zeros(100), 1, 2e-5)
    assert np.allclose(p0 - p, 2e-5 * gs[0] / (np.abs(gs[0]) + 1e-8), rtol=1e-12)
    tp = torch.from_numpy(p0.copy()).requires_grad_()
    opt = torch.optim.AdamW([tp], lr=1e-3, betas=(0.9, 0.999), eps=1e-8, weight_decay=0.01)
    p, m, v = p0.copy(), np.zeros(100), np.zeros(100)
    for t, g in enumerate(gs, 1):
        tp.grad = torch.from_numpy(g.copy())
        opt.step()
        p, m, v = om.adamw(p, g, m, v, t, 1e-3, wd=0.01)
    assert np.allclose(p, tp.detach().numpy(), rtol=1e-12, atol=1e-15)


def test_step_flops_8b():
    import synth
    f = om.step_flops(synth.L8B, 512, 512)
    assert abs(f / 1e12 - 16.1) < 0.2
