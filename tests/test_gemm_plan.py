"""GEMM scheduling, host side (no GPU): the planner's tile / split-K / stream-K choices for the
8B projection shapes, and the stream-K partition checked against a brute-force enumeration
of the flattened k-blocks (every k-block owned once, partial tiles only at the ends of a
CTA's range, workspace slots unique, each tile's shares in k order)."""
import pytest

from layer_streamed_nf4_lut_b200 import model as M

H, I, QKV = 4096, 14336, 6144


@pytest.mark.parametrize("rows", [512, 2048])
def test_plan_for_the_8b_projections(rows):
    fwd = {name: M.gemm_plan(rows, n, k) for name, n, k in
           [("qkv", QKV, H), ("o", H, H), ("gate_up", 2 * I, H), ("down", H, I)]}
    dx = {name: M.gemm_plan(rows, n, k, transposed=True) for name, n, k in
          [("qkv", H, QKV), ("o", H, H), ("gate_up", H, 2 * I), ("down", I, H)]}
    streamk = {f"{d} {n}" for d, plans in (("fwd", fwd), ("dx", dx)) for n, p in plans.items() if p["stream_k_ctas"]}
    if rows == 512:
        # the long GEMMs whose whole-tile grids leave SMs idle; q|k|v and o stay on whole tiles
        assert streamk == {"fwd gate_up", "dx gate_up", "fwd down"}
        p = fwd["gate_up"]
        assert (p["mt"], p["bn"], p["stream_k_ctas"], p["stream_k_tiles"], p["stream_k_kblocks"]) == (2, 128, 148, 448, 64)
    else:
        assert streamk == set()
    for p in list(fwd.values()) + list(dx.values()):
        assert p["splits"] == 1  # NF4 GEMMs never split K across CTAs of one tile


def test_plan_for_the_lora_gemms():
    u = M.gemm_plan(512, 64, I, nf4=False)  # x A^T of the down projection
    assert u["splits"] > 4 and u["fused_reduce"] == 0  # many partials: the wide reduction kernel
    assert M.gemm_plan(512, 64, 1024, nf4=False)["splits"] <= 4  # few: summed by the tile's last CTA
    assert M.gemm_plan(4096, 64, 512, nf4=False)["splits"] == 1  # dA / dB at 512 tokens: 8 k-blocks, whole
    assert M.gemm_plan(512, 64, 4096, nf4=False, sms=148)["stream_k_ctas"] == 0


def test_plan_rejects_bad_sizes():
    for args in [(0, 64, 64), (64, 60, 64), (64, 64, 60)]:
        with pytest.raises(Exception):
            M.gemm_plan(*args)


def _brute_pieces(tiles, nkt, ctas, c):
    lo, hi = tiles * nkt * c // ctas, tiles * nkt * (c + 1) // ctas
    out = []
    x = lo
    while x < hi:
        t = x // nkt
        end = min(hi, (t + 1) * nkt)
        out.append((t, x - t * nkt, end - t * nkt))
        x = end
    return out


@pytest.mark.parametrize("tiles,nkt,ctas", [(448, 64, 148), (64, 448, 148), (64, 225, 148), (96, 65, 148),
                                            (7, 3, 5), (1, 10, 3), (300, 1, 148), (52, 128, 148), (5, 97, 13)])
def test_stream_k_partition(tiles, nkt, ctas):
    writers = {}
    slots = set()
    for c in range(ctas):
        pieces = M.stream_k_pieces(tiles, nkt, ctas, c)
        assert [(t, a, b) for t, a, b, _ in pieces] == _brute_pieces(tiles, nkt, ctas, c)
        for i, (t, a, b, slot) in enumerate(pieces):
            whole = a == 0 and b == nkt
            assert (slot == -1) == whole
            if not whole:
                assert i in (0, len(pieces) - 1)  # a range cuts tiles only at its two ends
                assert slot == 2 * c + (0 if i == 0 else 1) and slot not in slots
                slots.add(slot)
                writers.setdefault(t, []).append((a, c, slot))
    covered = 0
    for t in range(tiles):
        shares = M.stream_k_shares(tiles, nkt, ctas, t)
        if t not in writers:
            assert len(shares) == 1 and shares[0][1] == -1
            covered += nkt
            continue
        w = sorted(writers[t])  # in k order
        assert shares == [(c, slot) for _, c, slot in w]
        covered += nkt
    assert covered == tiles * nkt


def test_stream_k_partitions_the_planner_picks_have_at_most_4_shares():
    for rows in (300, 512):
        for n, k, tr in [(2 * I, H, False), (H, 2 * I, True), (H, I, False), (3208, 8192, False), (3208, 12800, True)]:
            p = M.gemm_plan(rows, n, k, transposed=tr)
            if not p["stream_k_ctas"]:
                continue
            T, nkt, G = p["stream_k_tiles"], p["stream_k_kblocks"], p["stream_k_ctas"]
            assert max(len(M.stream_k_shares(T, nkt, G, t)) for t in range(T)) <= 4
