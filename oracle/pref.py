"""KTO, ORPO and SimPO losses on the streamed step, in float64 (oracle; test infrastructure only).

The pages name these methods beside DPO and say that KTO takes its reference the way DPO does,
from the same streamed base with the LoRA adapters switched off (rug.gal radar "Soup ... layer
streaming", "En detalle"; imasters "Do SFT para os métodos de preferência").  They print no
formula; each loss below follows the paper that defines it.  All three act on per-sequence
sums of target log-probs over the response (targets j >= max(prefix_len, 1)), like DPO, so
their gradient reaches the logits as one coefficient per sequence: dL/dlogits = dL/dpi_b *
(onehot - softmax) on the response targets of row b.

* SimPO (Meng, Xia, Chen 2024): reference-free, length-normalised.  Pairs are rows (2p, 2p+1)
  = (chosen, rejected); a = pi / n (n = response targets of the row);
  L = mean_p -log sigmoid(beta (a_c - a_r) - gamma).
* ORPO (Hong, Lee, Thorne 2024): reference-free.  a as above; odds(a) = e^a / (1 - e^a);
  L = mean_p [ -a_c + lam * -log sigmoid(log odds(a_c) - log odds(a_r)) ]
  (the SFT term is the chosen response's mean negative log-likelihood).
* KTO (Ethayarajh et al. 2024): unpaired rows, label 1 = desirable, 0 = undesirable;
  r_b = pi_b - ref_b (reference = LoRA off); z0 = max(0, mean_b r_b), held constant (no
  gradient flows through it); v_b = lam_d sigmoid(beta (r_b - z0)) if desirable,
  lam_u sigmoid(beta (z0 - r_b)) if not; L = mean_b (lam_{y_b} - v_b).
  The paper estimates z0 from mismatched (prompt, completion) pairs; here it is the batch
  mean of the rows' own rewards (a reading, recorded with the design).
"""
from __future__ import annotations

import numpy as np

from . import model as om


def _sigmoid(z):
    return 1.0 / (1.0 + np.exp(-z))


def _log1mexp(a):
    """log(1 - e^a) for a < 0, stable on both sides of -ln 2."""
    return np.where(a > -np.log(2.0), np.log(-np.expm1(a)), np.log1p(-np.exp(a)))


def simpo_loss(pi, n, beta, gamma):
    """pi[2P] response log-prob sums, n[2P] response target counts.  Returns (loss, dL/dpi)."""
    pi = np.asarray(pi, np.float64)
    n = np.asarray(n, np.float64)
    P = len(pi) // 2
    dpi = np.zeros_like(pi)
    loss = 0.0
    for p in range(P):
        c, r = 2 * p, 2 * p + 1
        z = beta * (pi[c] / n[c] - pi[r] / n[r]) - gamma
        loss += np.logaddexp(0.0, -z)
        sneg = _sigmoid(-z)
        dpi[c] = -sneg * beta / n[c] / P
        dpi[r] = sneg * beta / n[r] / P
    return loss / P, dpi


def orpo_loss(pi, n, lam):
    """Returns (loss, dL/dpi)."""
    pi = np.asarray(pi, np.float64)
    n = np.asarray(n, np.float64)
    P = len(pi) // 2
    dpi = np.zeros_like(pi)
    loss = 0.0
    for p in range(P):
        c, r = 2 * p, 2 * p + 1
        ac, ar = pi[c] / n[c], pi[r] / n[r]
        z = (ac - _log1mexp(ac)) - (ar - _log1mexp(ar))
        loss += -ac + lam * np.logaddexp(0.0, -z)
        sneg = _sigmoid(-z)
        # d log odds(a) / da = 1 / (1 - e^a)
        dpi[c] = (-1.0 - lam * sneg / (-np.expm1(ac))) / n[c] / P
        dpi[r] = (lam * sneg / (-np.expm1(ar))) / n[r] / P
    return loss / P, dpi


def kto_loss(pi, ref, labels, beta, lam_d, lam_u):
    """Returns (loss, dL/dpi, z0)."""
    pi = np.asarray(pi, np.float64)
    ref = np.asarray(ref, np.float64)
    labels = np.asarray(labels).astype(bool)
    B = len(pi)
    r = pi - ref
    z0 = max(0.0, float(np.mean(r)))
    dpi = np.zeros(B)
    loss = 0.0
    for b in range(B):
        if labels[b]:
            s = _sigmoid(beta * (r[b] - z0))
            loss += lam_d - lam_d * s
            dpi[b] = -lam_d * beta * s * (1.0 - s) / B
        else:
            s = _sigmoid(beta * (z0 - r[b]))
            loss += lam_u - lam_u * s
            dpi[b] = lam_u * beta * s * (1.0 - s) / B
    return loss / B, dpi, z0


def response_counts(B, S, prefix_len):
    return np.full(B, S - max(prefix_len, 1), dtype=np.float64)


def pref_step(cfg, layers, lora, head, ids, prefix_len, kind, hp, labels=None):
    """Loss and LoRA gradients of one KTO / ORPO / SimPO step.

    hp: SimPO {beta, gamma}; ORPO {lam}; KTO {beta, lam_d, lam_u} (+ labels[B])."""
    B, S = ids.shape
    ref = None
    if kind == "kto":
        ref_logits, _, _ = om.forward(cfg, layers, lora, head, ids, enabled=False)
        ref, _ = om.sequence_logps(ref_logits, ids, prefix_len)
    logits, caches, hc = om.forward(cfg, layers, lora, head, ids, enabled=True)
    pi, lp = om.sequence_logps(logits, ids, prefix_len)
    n = response_counts(B, S, prefix_len)
    if kind == "simpo":
        loss, dpi = simpo_loss(pi, n, hp["beta"], hp["gamma"])
    elif kind == "orpo":
        loss, dpi = orpo_loss(pi, n, hp["lam"])
    elif kind == "kto":
        loss, dpi, _ = kto_loss(pi, ref, labels, hp["beta"], hp["lam_d"], hp["lam_u"])
    else:
        raise ValueError(kind)
    dl = om.dpo_dlogits(lp, ids, prefix_len, dpi)
    grads = om.backward(cfg, layers, lora, head, caches, hc, dl, B, S, True)
    return loss, grads, dict(pi=pi, ref=ref)
