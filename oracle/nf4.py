"""NF4 4-bit quantisation with double-quantised absmax (oracle; test infrastructure only).

The pages fix only the name and the bit width: the base is kept "en precisión NF4 (4 bits
por parámetro)" (rug.gal radar "Soup ... layer streaming", "En detalle"; the soup.yaml
example `quantization: 4bit  # NF4` in "Como cabe um 8B em 4 GB" of the imasters page).
Block size 64 and a double-quantised absmax with groups of 256 blocks are workload
parameters.  Everything else below is the plainest reading, listed in the design notes:

* codebook: QLoRA's 4-bit NormalFloat (Dettmers et al. 2023, section "4-bit NormalFloat
  Quantization"): quantiles of N(0,1), 8 for the positive half and 7 for the negative half
  plus an exact zero, probabilities evenly spaced from 1 - delta down to 1/2 with
  delta = (1/(2*15) + 1/(2*16)) / 2, then divided by the largest so the range is [-1, 1].
* per block of 64 consecutive elements of the row-major flattened tensor: absmax
  m = max |w|; code q = argmin_j |w/m - c_j| evaluated in float64, ties to the lower
  index; m = 0 gives every element the code of 0.0.  The last block may be partial.
* packing: element 2i in the low nibble of byte i, element 2i+1 in the high nibble.
* double quantisation of the absmax: mu = float32(sequential float64 sum of m / n_blocks);
  per group of 256 blocks (last group may be partial) s2 = float32(max |m - mu| / 127), or
  1 when that maximum is 0; q8 = clamp(round_half_even((m - mu) / s2), -127, 127) in
  float64; reconstructed mhat = float32(float32(q8 * s2) + mu) (two float32 roundings, no
  fused multiply-add).  Codes are chosen with the original m.
* dequantised weight: bf16_round_nearest_even(float32(c_q * mhat)).
"""
from __future__ import annotations

import math
import numpy as np

BLOCK = 64
DQ_GROUP = 256


def codebook() -> np.ndarray:
    """The 16 NF4 levels, ascending, as float32 (derived in float64)."""
    from scipy.special import ndtri  # inverse standard-normal CDF
    delta = 0.5 * (1.0 / 30.0 + 1.0 / 32.0)
    pos = ndtri(np.linspace(1.0 - delta, 0.5, 9)[:8])
    neg = -ndtri(np.linspace(1.0 - delta, 0.5, 8)[:7])
    vals = np.sort(np.concatenate([neg, [0.0], pos]))
    vals = vals / vals.max()
    return vals.astype(np.float32)


def bf16_round(x: np.ndarray) -> np.ndarray:
    """float32 -> nearest bfloat16 (ties to even), returned as float32 values.

    Finite inputs only (NaN payloads are not handled)."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    bias = ((u >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    r = (u + bias) & np.uint32(0xFFFF0000)
    return r.view(np.float32)


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """bfloat16 bit patterns (uint16) -> float64 values."""
    return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def _codes_for_blocks(blocks: np.ndarray, m: np.ndarray, c64: np.ndarray) -> np.ndarray:
    """argmin_j |w/m - c_j| per element, float64, first index on ties."""
    zero_code = int(np.nonzero(c64 == 0.0)[0][0])
    safe = np.where(m > 0, m, 1.0)
    r = blocks / safe[:, None]
    dist = np.abs(r[..., None] - c64[None, None, :])
    q = np.argmin(dist, axis=-1).astype(np.uint8)
    q[m == 0] = zero_code
    return q


def quantise(w: np.ndarray, chunk_blocks: int = 1 << 15) -> dict:
    """Quantise a float32 tensor (any shape, row-major) to NF4 with double-quantised absmax.

    Returns dict(codes uint8[ceil(n/2)], absmax float32[nb] (raw m), q8 int8[nb],
    scales float32[ng], mean float32 scalar, n, shape)."""
    w = np.ascontiguousarray(w, dtype=np.float32)
    shape = w.shape
    flat = w.reshape(-1)
    n = flat.size
    nb = (n + BLOCK - 1) // BLOCK
    c64 = codebook().astype(np.float64)
    padded = np.zeros(nb * BLOCK, dtype=np.float32)
    padded[:n] = flat
    blocks_all = padded.reshape(nb, BLOCK)
    m = np.abs(blocks_all).max(axis=1).astype(np.float32)  # exact: max of |float32|
    q = np.empty((nb, BLOCK), dtype=np.uint8)
    for lo in range(0, nb, chunk_blocks):
        hi = min(nb, lo + chunk_blocks)
        q[lo:hi] = _codes_for_blocks(blocks_all[lo:hi].astype(np.float64), m[lo:hi].astype(np.float64), c64)
    qf = q.reshape(-1)[:n]
    if n % 2:
        qf = np.concatenate([qf, np.zeros(1, np.uint8)])
    codes = (qf[0::2] | (qf[1::2] << np.uint8(4))).astype(np.uint8)

    # double quantisation of the absmax
    mu64 = np.add.accumulate(m.astype(np.float64))[-1] / nb  # sequential left-to-right sum
    mu = np.float32(mu64)
    ng = (nb + DQ_GROUP - 1) // DQ_GROUP
    scales = np.empty(ng, dtype=np.float32)
    q8 = np.empty(nb, dtype=np.int8)
    for g in range(ng):
        seg = m[g * DQ_GROUP:(g + 1) * DQ_GROUP].astype(np.float64) - np.float64(mu)
        amax = np.abs(seg).max()
        s2 = np.float32(amax / 127.0) if amax > 0 else np.float32(1.0)
        scales[g] = s2
        q8[g * DQ_GROUP:(g + 1) * DQ_GROUP] = np.clip(np.rint(seg / np.float64(s2)), -127, 127).astype(np.int8)
    return dict(codes=codes, absmax=m, q8=q8, scales=scales, mean=mu, n=n, shape=shape)


def absmax_dequant(nf: dict) -> np.ndarray:
    """Reconstructed per-block absmax mhat (float32)."""
    nb = nf["q8"].size
    s2 = np.repeat(nf["scales"], DQ_GROUP)[:nb]
    prod = (nf["q8"].astype(np.float32) * s2).astype(np.float32)
    return (prod + np.float32(nf["mean"])).astype(np.float32)


def unpack_codes(codes: np.ndarray, n: int) -> np.ndarray:
    q = np.empty(codes.size * 2, dtype=np.uint8)
    q[0::2] = codes & np.uint8(0x0F)
    q[1::2] = codes >> np.uint8(4)
    return q[:n]


def dequant(nf: dict) -> np.ndarray:
    """Dequantised weights as float32 values that are exactly bfloat16."""
    n = nf["n"]
    q = unpack_codes(nf["codes"], n)
    c = codebook()
    mhat = absmax_dequant(nf)
    scale = np.repeat(mhat, BLOCK)[:n]
    prod = (c[q] * scale).astype(np.float32)  # one float32 multiply
    return bf16_round(prod).reshape(nf["shape"])


def dequant_bits(nf: dict) -> np.ndarray:
    """Dequantised weights as bfloat16 bit patterns (uint16)."""
    v = dequant(nf)
    return (np.ascontiguousarray(v).view(np.uint32) >> np.uint32(16)).astype(np.uint16)


def blob_segment_bytes(n: int) -> dict:
    """Byte counts of one tensor's quantised parts (no padding)."""
    nb = (n + BLOCK - 1) // BLOCK
    ng = (nb + DQ_GROUP - 1) // DQ_GROUP
    return dict(codes=(n + 1) // 2, q8=nb, scales=4 * ng, mean=4)


def layer_stream_bytes(n_per_proj, hidden: int) -> int:
    """Algorithmic bytes of one streamed layer: codes + q8 absmax + fp32 group scales +
    fp32 means + two bf16 RMSNorm gains (no alignment padding)."""
    tot = 0
    for n in n_per_proj:
        b = blob_segment_bytes(n)
        tot += b["codes"] + b["q8"] + b["scales"] + b["mean"]
    return tot + 2 * 2 * hidden


def dq_error_bound(nf: dict) -> float:
    """max |mhat - m| allowed: half a step of s2 plus float32 rounding of the two ops."""
    return float(np.max(nf["scales"])) * 0.5 + 4 * float(np.finfo(np.float32).eps) * float(max(1e-30, np.max(nf["absmax"])))


__all__ = ["codebook", "quantise", "dequant", "dequant_bits", "absmax_dequant", "bf16_round",
           "bf16_bits_to_f64", "unpack_codes", "blob_segment_bytes", "layer_stream_bytes",
           "BLOCK", "DQ_GROUP", "math"]
