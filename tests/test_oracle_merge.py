"""Pins of the oracle's LoRA merge (W' = bf16(W + s B A)) and its one-step bf16 rounding."""
from fractions import Fraction

import numpy as np

from oracle import model as om
from oracle import nf4


def _bf16_neighbours(x: float):
    """The two bf16 numbers around x, found by truncating its float32 bits (and the next
    one up); x is a normal float64."""
    f = np.float32(x)
    u = np.array([f], dtype=np.float32).view(np.uint32)[0]
    lo_bits = np.uint32(u & np.uint32(0xFFFF0000))
    cands = []
    for d in (-1, 0, 1, 2):
        b = np.uint32(int(lo_bits) + d * 0x10000)
        cands.append(float(np.array([b], dtype=np.uint32).view(np.float32)[0]))
    return cands


def _round_brute(x: Fraction) -> float:
    """Nearest bf16 to the exact rational x, ties to the even significand (brute force over
    the neighbouring bf16 numbers)."""
    best = None
    for c in _bf16_neighbours(float(x)):
        d = abs(Fraction(c) - x)
        bits = int(np.array([c], dtype=np.float32).view(np.uint32)[0]) >> 16
        key = (d, bits & 1)
        if best is None or key < best[0]:
            best = (key, c)
    return best[1]


def test_bf16_round_f64_hand_values():
    # 1 + 2^-8 lies halfway between 1 and 1 + 2^-7: ties go to the even significand (1.0)
    assert om.bf16_round_f64(1.0 + 2.0 ** -8) == 1.0
    # 1 + 3 * 2^-8 lies halfway between 1 + 2^-7 and 1 + 2^-6: even is 1 + 2^-6
    assert om.bf16_round_f64(1.0 + 3 * 2.0 ** -8) == 1.0 + 2.0 ** -6
    # just above the tie rounds up; a float32 pre-rounding would have lost the 2^-40
    assert om.bf16_round_f64(1.0 + 2.0 ** -8 + 2.0 ** -40) == 1.0 + 2.0 ** -7
    assert om.bf16_round_f64(-3.0) == -3.0
    assert om.bf16_round_f64(0.0) == 0.0


def test_bf16_round_f64_is_nearest_brute_force():
    rng = np.random.default_rng(3)
    x = rng.normal(0.0, 1.0, 400) * np.exp2(rng.integers(-20, 20, 400))
    got = om.bf16_round_f64(x)
    for xi, gi in zip(x, got):
        assert gi == _round_brute(Fraction(float(xi))), xi


def test_merge_zero_b_is_base():
    rng = np.random.default_rng(4)
    W = nf4.bf16_round(rng.normal(0, 0.02, (48, 64)).astype(np.float32)).astype(np.float64)
    A = rng.normal(0, 0.1, (8, 64))
    B = np.zeros((48, 8))
    assert np.array_equal(om.merge_lora(W, A, B, 2.0), W)


def test_merge_rank1_hand_case():
    # W = 0, r = 1: W'[i, j] = s * b_i * a_j, all products exact in bf16
    A = np.array([[0.5, -1.0, 0.25]])
    B = np.array([[2.0], [-0.75]])
    got = om.merge_lora(np.zeros((2, 3)), A, B, 0.25)
    want = np.array([[0.25, -0.5, 0.125], [-0.09375, 0.1875, -0.046875]])
    assert np.array_equal(got, want)


def test_merge_brute_force_exact_sum():
    rng = np.random.default_rng(5)
    out, inn, r, s = 5, 7, 3, 16.0 / 3
    W = nf4.bf16_round(rng.normal(0, 0.02, (out, inn)).astype(np.float32)).astype(np.float64)
    A = rng.normal(0, 0.2, (r, inn)).astype(np.float32)
    B = rng.normal(0, 0.05, (out, r)).astype(np.float32)
    got = om.merge_lora(W, A, B, s)
    Ab = nf4.bf16_round(A).astype(np.float64)
    Bb = nf4.bf16_round(B).astype(np.float64)
    sf = Fraction(s)
    for i in range(out):
        for j in range(inn):
            acc = Fraction(W[i, j]) + sf * sum(Fraction(Bb[i, k]) * Fraction(Ab[k, j]) for k in range(r))
            assert got[i, j] == _round_brute(acc), (i, j)


def test_merged_forward_equals_lora_forward():
    # x W'^T = x W^T + s (x A^T) B^T up to the one bf16 rounding of W'
    rng = np.random.default_rng(6)
    out, inn, r, s = 32, 96, 8, 2.0
    W = nf4.bf16_round(rng.normal(0, 0.02, (out, inn)).astype(np.float32)).astype(np.float64)
    A = rng.normal(0, 0.1, (r, inn))
    B = rng.normal(0, 0.05, (out, r))
    Wm = om.merge_lora(W, A, B, s)
    x = rng.normal(0, 1, (10, inn))
    Ab = nf4.bf16_round(A.astype(np.float32)).astype(np.float64)
    Bb = nf4.bf16_round(B.astype(np.float32)).astype(np.float64)
    exact = x @ W.T + s * (x @ Ab.T) @ Bb.T
    # |W' - (W + s B A)| <= half a bf16 ulp <= 2^-9 |W'| per element
    bound = np.abs(x) @ (np.abs(Wm).T * 2.0 ** -9) + 1e-12
    assert np.all(np.abs(x @ Wm.T - exact) <= bound)
