"""Seeded synthetic inputs shared by the oracle-side tests and the CUDA-side tests/bench.

This module only draws random numbers and names workload shapes.  It holds none of
the trained method's arithmetic (no quantisation, no layer math, no loss).

Counter-based generator (host, numpy): every value is a pure function of
(seed, stream, index), so the result never depends on chunking or threading.
  u64 = splitmix64_finalize(seed * 0x9E3779B97F4A7C15 ^ stream * 0xD1B54A32D192ED03 + index)
The SplitMix64 finaliser is the published one (Steele, Lea, Flood, "Fast splittable
pseudorandom number generators", OOPSLA 2014): xor-shift 30 / mul 0xBF58476D1CE4E5B9 /
xor-shift 27 / mul 0x94D049BB133111EB / xor-shift 31.
Uniforms take the top 53 bits; normals use the Box-Muller transform on two
independent uniform streams (index 2i and 2i+1).

For workloads too large to draw on the host in reasonable time (the 8B / 70B shapes),
`normal_device` draws with torch's counter-based Philox generator on the GPU.  Those
draws are seeded and reproducible but are not the same numbers as the host stream;
they are only used where no oracle comparison of individual values is made.
"""
from __future__ import annotations

import math
import numpy as np

_M64 = np.uint64(0xFFFFFFFFFFFFFFFF)
_G1 = np.uint64(0x9E3779B97F4A7C15)
_G2 = np.uint64(0xD1B54A32D192ED03)
_C1 = np.uint64(0xBF58476D1CE4E5B9)
_C2 = np.uint64(0x94D049BB133111EB)


def _finalize(z: np.ndarray) -> np.ndarray:
    z = z.copy()
    z ^= z >> np.uint64(30)
    z *= _C1
    z ^= z >> np.uint64(27)
    z *= _C2
    z ^= z >> np.uint64(31)
    return z


def raw_u64(seed: int, stream: int, index: np.ndarray) -> np.ndarray:
    """64 random bits for each counter value in `index` (uint64 array)."""
    with np.errstate(over="ignore"):
        key = (np.uint64(seed & 0xFFFFFFFFFFFFFFFF) * _G1) ^ (np.uint64(stream & 0xFFFFFFFFFFFFFFFF) * _G2)
        return _finalize(index.astype(np.uint64) + key)


def uniform01(seed: int, stream: int, n: int, offset: int = 0) -> np.ndarray:
    """n doubles in the open interval (0, 1)."""
    idx = np.arange(offset, offset + n, dtype=np.uint64)
    bits = raw_u64(seed, stream, idx) >> np.uint64(11)
    return (bits.astype(np.float64) + 0.5) * (1.0 / 9007199254740992.0)


def normal(seed: int, stream: int, shape, std: float = 1.0, chunk: int = 1 << 22) -> np.ndarray:
    """float32 array of N(0, std^2) draws (Box-Muller, computed in float64)."""
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.float32)
    for lo in range(0, n, chunk):
        m = min(chunk, n - lo)
        idx = np.arange(lo, lo + m, dtype=np.uint64)
        u1 = ((raw_u64(seed, stream, idx * np.uint64(2)) >> np.uint64(11)).astype(np.float64) + 0.5) / 9007199254740992.0
        u2 = ((raw_u64(seed, stream, idx * np.uint64(2) + np.uint64(1)) >> np.uint64(11)).astype(np.float64) + 0.5) / 9007199254740992.0
        out[lo:lo + m] = (std * np.sqrt(-2.0 * np.log(u1)) * np.cos(2.0 * math.pi * u2)).astype(np.float32)
    return out.reshape(shape)


def uniform_sym(seed: int, stream: int, shape, bound: float) -> np.ndarray:
    """float32 draws from U(-bound, bound)."""
    n = int(np.prod(shape))
    u = uniform01(seed, stream, n)
    return ((2.0 * u - 1.0) * bound).astype(np.float32).reshape(shape)


def token_ids_uniform(seed: int, stream: int, n: int, vocab: int) -> np.ndarray:
    """int32 ids uniform over [0, vocab)."""
    idx = np.arange(n, dtype=np.uint64)
    bits = raw_u64(seed, stream, idx)
    return (bits % np.uint64(vocab)).astype(np.int32)


def token_ids_zipf(seed: int, stream: int, n: int, vocab: int, s: float = 1.1) -> np.ndarray:
    """int32 ids with Zipf(s) rank frequencies over ranks 1..vocab; rank k -> id k-1.

    Sampled by inverse CDF over a float64 table of cumulative k^-s weights."""
    w = np.arange(1, vocab + 1, dtype=np.float64) ** (-s)
    cdf = np.cumsum(w)
    cdf /= cdf[-1]
    u = uniform01(seed, stream, n)
    return np.minimum(np.searchsorted(cdf, u, side="left"), vocab - 1).astype(np.int32)


def bf16_bits_from_f32(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 bit patterns (round to nearest even).

    Used only to turn synthetic float32 draws into bf16 input tensors."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    bias = ((u >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((u + bias) >> np.uint32(16)).astype(np.uint16)


def normal_device(shape, seed: int, std: float, device="cuda"):
    """Large N(0, std^2) float32 tensor drawn on the GPU with torch's Philox generator."""
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    t = torch.empty(shape, dtype=torch.float32, device=device)
    t.normal_(0.0, std, generator=g)
    return t


# ----------------------------------------------------------------------------------
# Workload shapes (sizes only).  Llama-style decoder dimensions; LoRA on q,k,v,o,gate,up,down.
# ----------------------------------------------------------------------------------
TINY = dict(name="tiny-2L-h256", n_layers=2, hidden=256, n_heads=4, n_kv_heads=2, head_dim=64,
            intermediate=688, vocab=1024, rms_eps=1e-5, rope_theta=5e5, lora_r=8, lora_alpha=16.0,
            batch=1, seq=64)
L8B = dict(name="llama8b-shape", n_layers=32, hidden=4096, n_heads=32, n_kv_heads=8, head_dim=128,
           intermediate=14336, vocab=128256, rms_eps=1e-5, rope_theta=5e5, lora_r=64, lora_alpha=16.0,
           batch=1, seq=512)
L8B_B4 = dict(L8B, name="llama8b-shape-b4-zipf-masked", batch=4, seq=512)
L8B_DPO = dict(L8B, name="llama8b-shape-dpo-2pairs", batch=4, seq=512, n_pairs=2, prefix_len=256, beta=0.1)
L70B = dict(name="llama70b-shape", n_layers=80, hidden=8192, n_heads=64, n_kv_heads=8, head_dim=128,
            intermediate=28672, vocab=128256, rms_eps=1e-5, rope_theta=5e5, lora_r=64, lora_alpha=16.0,
            batch=1, seq=2048)

PROJ_NAMES = ("q", "k", "v", "o", "gate", "up", "down")

# stream ids for the draws (kept apart so every tensor has its own counter space)
STREAM_W = 1000        # + 16*layer + proj
STREAM_GAMMA = 5000    # + 2*layer + {0,1}
STREAM_EMBED = 7001
STREAM_LMHEAD = 7002
STREAM_FINAL_GAMMA = 7003
STREAM_LORA_A = 8000   # + 16*layer + proj
STREAM_LORA_B = 9000   # + 16*layer + proj
STREAM_IDS = 11000
STREAM_MASK = 12000


def proj_shape(cfg: dict, p: str):
    """(out, in) of a projection."""
    h, d = cfg["hidden"], cfg["head_dim"]
    if p == "q":
        return cfg["n_heads"] * d, h
    if p in ("k", "v"):
        return cfg["n_kv_heads"] * d, h
    if p == "o":
        return h, cfg["n_heads"] * d
    if p in ("gate", "up"):
        return cfg["intermediate"], h
    if p == "down":
        return h, cfg["intermediate"]
    raise KeyError(p)


def layer_weights(cfg: dict, seed: int, layer: int, std: float = 0.02, gamma_noise: float = 0.0):
    """float32 base weights of one decoder layer (host draws) and its two RMSNorm gains.

    gamma_noise = 0 gives gains of exactly 1 (the workload's value); tests pass 0.1 so a
    missing gain would be caught."""
    w = {}
    for j, p in enumerate(PROJ_NAMES):
        w[p] = normal(seed, STREAM_W + 16 * layer + j, proj_shape(cfg, p), std)
    h = cfg["hidden"]
    for j, g in enumerate(("attn_norm", "mlp_norm")):
        if gamma_noise:
            w[g] = (1.0 + normal(seed, STREAM_GAMMA + 2 * layer + j, (h,), gamma_noise)).astype(np.float32)
        else:
            w[g] = np.ones(h, dtype=np.float32)
    return w


def head_weights(cfg: dict, seed: int, std: float = 0.02, gamma_noise: float = 0.0):
    """bf16 bit patterns (uint16) of the embedding [V,h], lm_head [V,h] and final gain [h]."""
    V, h = cfg["vocab"], cfg["hidden"]
    emb = bf16_bits_from_f32(normal(seed, STREAM_EMBED, (V, h), std))
    lm = bf16_bits_from_f32(normal(seed, STREAM_LMHEAD, (V, h), std))
    if gamma_noise:
        g = bf16_bits_from_f32((1.0 + normal(seed, STREAM_FINAL_GAMMA, (h,), gamma_noise)).astype(np.float32))
    else:
        g = bf16_bits_from_f32(np.ones(h, dtype=np.float32))
    return emb, lm, g


def lora_weights(cfg: dict, seed: int, b_std: float = 0.01, zero_b: bool = False):
    """{(layer, proj): (A[r,in], B[out,r])} float32.

    A ~ U(-1/sqrt(in), 1/sqrt(in)) (Kaiming-uniform with a = sqrt 5); B ~ N(0, b_std^2)."""
    r = cfg["lora_r"]
    out = {}
    for layer in range(cfg["n_layers"]):
        for j, p in enumerate(PROJ_NAMES):
            o, i = proj_shape(cfg, p)
            A = uniform_sym(seed, STREAM_LORA_A + 16 * layer + j, (r, i), 1.0 / math.sqrt(i))
            B = np.zeros((o, r), np.float32) if zero_b else normal(seed, STREAM_LORA_B + 16 * layer + j, (o, r), b_std)
            out[(layer, p)] = (A, B)
    return out


def token_batch(cfg: dict, seed: int, zipf: bool = False):
    """int32 ids [B, S]."""
    B, S = cfg["batch"], cfg["seq"]
    if zipf:
        return token_ids_zipf(seed, STREAM_IDS, B * S, cfg["vocab"]).reshape(B, S)
    return token_ids_uniform(seed, STREAM_IDS, B * S, cfg["vocab"]).reshape(B, S)


def preference_batch(cfg: dict, seed: int):
    """int32 ids [2P, S]: rows 2p (chosen) and 2p+1 (rejected) share ids[:, :prefix_len]."""
    P, S, pre, V = cfg["n_pairs"], cfg["seq"], cfg["prefix_len"], cfg["vocab"]
    ids = token_ids_uniform(seed, STREAM_IDS, 2 * P * S, V).reshape(2 * P, S)
    for p in range(P):
        ids[2 * p + 1, :pre] = ids[2 * p, :pre]
    return ids


def last_half_mask(B: int, S: int) -> np.ndarray:
    """uint8 [B, S] target mask: 1 for target positions j in [S/2, S)."""
    m = np.zeros((B, S), np.uint8)
    m[:, S // 2:] = 1
    return m
