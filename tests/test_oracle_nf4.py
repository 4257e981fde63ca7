"""Pins for the NF4 / double-quant oracle: a published table, exact round trips, brute force
on tiny inputs, hand-worked bytes, and bf16 rounding against torch's converter."""
import os

import numpy as np
import pytest
import torch

from oracle import nf4

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_codebook_matches_qlora_table():
    # QLoRA paper appendix values (tests/golden/nf4_codebook_qlora.txt)
    g = np.loadtxt(os.path.join(GOLDEN, "nf4_codebook_qlora.txt"))
    c = nf4.codebook()
    assert c.dtype == np.float32 and c.shape == (16,)
    assert np.max(np.abs(c.astype(np.float64) - g)) < 1e-6


def test_codebook_structure():
    c = nf4.codebook()
    assert np.all(np.diff(c) > 0), "strictly ascending, 16 distinct"
    assert c[0] == -1.0 and c[15] == 1.0 and c[7] == 0.0
    assert np.sum(c > 0) == 8 and np.sum(c < 0) == 7


def test_roundtrip_every_code_exact():
    # a block holding every level times an absmax re-quantises to the same codes
    c = nf4.codebook()
    for m in (1.0, 0.037, 3.5e-3, 17.25):
        q = np.array([i % 16 for i in range(64)], dtype=np.uint8)
        w = (c[q].astype(np.float64) * m).astype(np.float32)
        nf = nf4.quantise(w)
        got = nf4.unpack_codes(nf["codes"], 64)
        assert np.array_equal(got, q), m
        assert nf["absmax"][0] == np.float32(np.max(np.abs(w)))


def test_codes_brute_force_nearest():
    rng = np.random.default_rng(1)
    w = rng.standard_normal(64 * 37).astype(np.float32) * 0.02
    nf = nf4.quantise(w)
    q = nf4.unpack_codes(nf["codes"], w.size)
    c = nf4.codebook().astype(np.float64)
    for b in range(37):
        blk = w[b * 64:(b + 1) * 64].astype(np.float64)
        m = np.max(np.abs(blk))
        for i in range(64):
            r = blk[i] / m
            best = min(range(16), key=lambda j: (abs(r - c[j]), j))
            assert q[b * 64 + i] == best


def test_packing_low_nibble_first_and_partial_block():
    c = nf4.codebook()
    # 3 elements: codes 3, 12, 15 -> bytes [0xC3, 0x0F]; a single partial block
    w = np.array([c[3] * 0.5, c[12] * 0.5, c[15] * 0.5], dtype=np.float32)
    nf = nf4.quantise(w)
    assert list(nf["codes"]) == [0xC3, 0x0F]
    assert nf["q8"].size == 1 and nf["scales"].size == 1


def test_zero_block():
    w = np.zeros(128, dtype=np.float32)
    w[64:] = np.linspace(-1, 1, 64, dtype=np.float32)
    nf = nf4.quantise(w)
    q = nf4.unpack_codes(nf["codes"], 128)
    assert np.all(q[:64] == 7) and nf["absmax"][0] == 0.0
    deq = nf4.dequant(nf)
    assert np.all(deq[:64] == 0.0)


def test_double_quant_closed_form_and_idempotent():
    # absmax [0.1, 0.3] (two blocks): mu = 0.2, s2 = 0.1/127, q8 = [-127, 127]
    w = np.zeros(128, np.float32)
    w[0] = 0.1
    w[64] = -0.3
    nf = nf4.quantise(w)
    mu = np.float32((np.float64(np.float32(0.1)) + np.float64(np.float32(0.3))) / 2)
    assert nf["mean"] == mu
    amax = max(abs(np.float64(np.float32(0.1)) - np.float64(mu)), abs(np.float64(np.float32(0.3)) - np.float64(mu)))
    assert nf["scales"][0] == np.float32(amax / 127)
    assert list(nf["q8"]) == [-127, 127]
    # idempotence: quantising the reconstructed absmax with the same mu, s2 returns q8
    rng = np.random.default_rng(2)
    w = (rng.standard_normal(64 * 700) * 0.02).astype(np.float32)
    nf = nf4.quantise(w)
    mhat = nf4.absmax_dequant(nf)
    s2 = np.repeat(nf["scales"], 256)[:mhat.size].astype(np.float64)
    q8b = np.clip(np.rint((mhat.astype(np.float64) - np.float64(nf["mean"])) / s2), -127, 127)
    assert np.array_equal(q8b.astype(np.int8), nf["q8"])
    assert np.max(np.abs(mhat.astype(np.float64) - nf["absmax"])) <= nf4.dq_error_bound(nf)
    assert nf["scales"].size == 3  # 700 blocks -> groups of 256, 256, 188


def test_mean_is_sequential_float64_sum():
    rng = np.random.default_rng(3)
    w = (rng.standard_normal(64 * 513) * 0.05).astype(np.float32)
    nf = nf4.quantise(w)
    acc = 0.0
    for v in nf["absmax"]:
        acc += float(v)
    assert nf["mean"] == np.float32(acc / 513)


def test_bf16_round_matches_torch():
    rng = np.random.default_rng(4)
    x = np.concatenate([(rng.standard_normal(100000) * 10 ** rng.uniform(-6, 6, 100000)).astype(np.float32),
                        np.array([1.00390625, 1.01171875, -1.00390625, 65504.0, 3.0e38], np.float32)])
    ours = nf4.bf16_round(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float32).numpy()
    assert np.array_equal(ours.view(np.uint32), ref.view(np.uint32))
    # ties to even, worked by hand: 1 + 2^-8 -> 1.0 ; 1 + 3*2^-8 -> 1 + 2^-6
    assert nf4.bf16_round(np.array([1.00390625], np.float32))[0] == 1.0
    assert nf4.bf16_round(np.array([1.01171875], np.float32))[0] == 1.015625


def test_dequant_definition_single_values():
    c = nf4.codebook()
    w = np.array([0.0] * 63 + [0.3], np.float32)
    w[5] = c[13] * 0.3
    nf = nf4.quantise(w)
    deq = nf4.dequant(nf)
    mhat = nf4.absmax_dequant(nf)[0]
    assert deq[5] == nf4.bf16_round(np.array([c[13] * mhat], np.float32))[0]
    assert deq[63] == nf4.bf16_round(np.array([np.float32(1.0) * mhat], np.float32))[0]


def test_stream_bytes_8b_layer():
    # 8B-shaped layer: 218.1M NF4 parameters -> 112.53 MB streamed per layer
    h, I, d, hq, hkv = 4096, 14336, 128, 32, 8
    ns = [hq * d * h, hkv * d * h, hkv * d * h, h * hq * d, I * h, I * h, h * I]
    assert sum(ns) == 218103808
    b = nf4.layer_stream_bytes(ns, h)
    assert abs(b / 1e6 - 112.53) < 0.01
