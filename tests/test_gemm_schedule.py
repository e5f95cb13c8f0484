"""Host checks of the W4A16 GEMM's tile schedule (no GPU).

The schedule, as stated in the header of awq_w4a16_gemm and in the launcher:
128-channel x BN-token tiles (BN = 256 unless 256-token tiles cannot give every
SM a tile and 128-token tiles would give more); data-parallel over
min(tiles, SMs) persistent CTAs, unless whole tiles fill under 80 % of the
waves x SMs tile slots (M > 32, at least 8 k-blocks per SM), in which case all
but the last full wave and the partial one stay whole and the k-blocks of the
rest are split evenly, one contiguous range per CTA; split tiles are finished by
a fixup kernel from two fp32 slots per CTA.

This module models that schedule in Python and checks
- that the library plans the same thing (launch count and workspace size for
  148 SMs, the count the library assumes without a device);
- that every (tile, k-block) is computed exactly once, that a CTA's partial
  segments are its first (slot 0) and last (slot 1) stream-K segments, and that
  the fixup finds each contributor's part where it was written, for many shapes
  and SM counts;
- that the grouped tile order visits every tile once (ragged last block
  included), and that the CTA-pair schedule computes every output tile once,
  the channel tile past the last only on the second CTA of the last pair.
"""
import pytest

import weight_only_bit_awq_b200 as awq


def cdiv(a, b):
    return -(-a // b)


def plan(M, K, N, sm):
    nt = cdiv(N, 128)
    bn = 256 if (M > 128 and (cdiv(M, 256) * nt >= sm or cdiv(M, 128) * nt <= cdiv(M, 256) * nt)) else 128
    KB = K // 128
    T = cdiv(M, bn) * nt
    waves = cdiv(T, sm)
    tsk = T if T < sm else sm + T % sm
    if M > 32 and T % sm != 0 and 100 * T < 80 * waves * sm and tsk * KB >= 8 * sm:
        return dict(bn=bn, T=T, KB=KB, P=sm, Tdp=T - tsk, sk=True)
    return dict(bn=bn, T=T, KB=KB, P=min(T, sm), Tdp=T, sk=False)


def segments(p, c):
    """(tile, kb0, kb1) of CTA c, in the order every role of the kernel walks them."""
    P, T, KB, Tdp = p["P"], p["T"], p["KB"], p["Tdp"]
    ndp = (Tdp - 1 - c) // P + 1 if c < Tdp else 0
    usk = (T - Tdp) * KB
    ub, ue = c * usk // P, (c + 1) * usk // P
    out = [(c + j * P, 0, KB) for j in range(ndp)]
    if ub < ue:
        for s in range(ub // KB, (ue - 1) // KB + 1):
            out.append((Tdp + s, ub - s * KB if s == ub // KB else 0, min(KB, ue - s * KB)))
    return out, ndp, usk


def check_schedule(M, K, N, sm):
    p = plan(M, K, N, sm)
    owner, slots = {}, {}
    for c in range(p["P"]):
        segs, ndp, _ = segments(p, c)
        for j, (t, kb0, kb1) in enumerate(segs):
            assert 0 <= t < p["T"] and 0 <= kb0 < kb1 <= p["KB"]
            for kb in range(kb0, kb1):
                assert (t, kb) not in owner
                owner[(t, kb)] = c
            if (kb0, kb1) != (0, p["KB"]):           # a part of a split tile
                assert p["sk"] and t >= p["Tdp"] and j in (ndp, len(segs) - 1)
                w = 0 if j == ndp else 1
                assert (c, w) not in slots
                slots[(c, w)] = t
    assert len(owner) == p["T"] * p["KB"]
    if not p["sk"]:
        assert not slots
        return p
    # the fixup's view of tile s: contributors and the slot each wrote
    P, KB, Tdp = p["P"], p["KB"], p["Tdp"]
    usk = (p["T"] - Tdp) * KB
    for s in range(p["T"] - Tdp):
        cta_of = lambda u: ((u + 1) * P - 1) // usk
        cf, cl = cta_of(s * KB), cta_of((s + 1) * KB - 1)
        contrib = sorted({owner[(Tdp + s, kb)] for kb in range(KB)})
        assert contrib == list(range(cf, cl + 1))
        if cf == cl:
            continue
        for cc in contrib:
            w = 0 if cc * usk // P >= s * KB else 1
            assert slots[(cc, w)] == Tdp + s
    return p


SHAPES = [(M, K, N) for M in (33, 100, 129, 255, 257, 300, 513, 1000, 2048, 4096)
          for K in (128, 1024, 2048, 4096, 14336) for N in (16, 272, 1024, 4096, 28672)]


@pytest.mark.parametrize("sm", [148, 132, 8, 3])
def test_every_k_block_once_and_parts_where_the_fixup_reads_them(sm):
    n_sk = sum(check_schedule(M, K, N, sm)["sk"] for (M, K, N) in SHAPES)
    assert n_sk > 0


def test_the_library_plans_the_same_schedule():
    # without a device the library plans for 148 SMs
    seen = set()
    for (M, K, N) in SHAPES + [(512, 4096, 28672), (512, 14336, 4096), (512, 14848, 59392), (40, 24576, 1024),
                               (40, 1024, 38400), (300, 1024, 9600), (513, 2048, 6400), (40, 2048, 19200)]:
        p = plan(M, K, N, 148)
        seen.add(p["sk"])
        assert awq.awq_linear_launches(M, K, N, 128) == (2 if p["sk"] else 1), (M, K, N)
        slots = 148 * 2 * p["bn"] * 128 * 4 if p["sk"] else 0
        assert awq.awq_workspace_bytes(M, K, N) == 256 + slots, (M, K, N)
    assert seen == {True, False}


# ---- tile order and the CTA-pair schedule ----
# Tiles t = 0 .. MT x NT - 1 map to (token tile, channel tile) in blocks of GM
# token tiles (the last block may hold fewer); within a block the token tile
# runs fastest, so the CTAs working at the same time share a few weight tiles.
# The CTA-pair kernel walks pair tiles (token tile, channel-tile pair np) in
# that order with NP = ceil(NT / 2) in place of NT: cluster cl of P2 takes pair
# tiles cl, cl + P2, ...; the pair's CTA of rank r computes channel tile
# 2 np + r, which is past the last when NT is odd (that CTA only takes part in
# the pair's MMAs).


def tile_coords(t, MT, NT, GM):
    blk, w = t // (GM * NT), t % (GM * NT)
    gb = min(GM, MT - blk * GM)
    return blk * GM + w % gb, w // gb


def gm_of(M, K, BN):
    """Token tiles per block: the block's x within ~48 MB of L2, at least one."""
    return max(1, min((48 << 20) // (BN * K * 2), cdiv(M, BN)))


def test_the_tile_order_visits_every_tile_once():
    for MT in range(1, 13):
        for NT in range(1, 13):
            for GM in range(1, MT + 1):
                seen = [tile_coords(t, MT, NT, GM) for t in range(MT * NT)]
                assert sorted(seen) == [(m, n) for m in range(MT) for n in range(NT)], (MT, NT, GM)


@pytest.mark.parametrize("M,K,N", [(2048, 4096, 28672), (8192, 14848, 59392), (500, 256, 15232), (257, 128, 272),
                                   (4096, 14336, 4096), (1024, 2048, 16 * 128 * 3)])
@pytest.mark.parametrize("P2", [1, 3, 74, 148])
def test_cta_pairs_compute_every_output_tile_once(M, K, N, P2):
    MT, NT = cdiv(M, 256), cdiv(N, 128)
    NP = cdiv(NT, 2)
    T2 = MT * NP
    GM = gm_of(M, K, 256)
    done = {}
    for cl in range(P2):
        ntiles = (T2 - 1 - cl) // P2 + 1 if cl < T2 else 0
        for j in range(ntiles):
            mt, np_ = tile_coords(cl + j * P2, MT, NP, GM)
            for rank in (0, 1):
                nt = 2 * np_ + rank
                if nt >= NT:
                    assert NT % 2 == 1 and np_ == NP - 1 and rank == 1
                    continue
                assert (mt, nt) not in done
                done[(mt, nt)] = (cl, rank)
    assert sorted(done) == [(m, n) for m in range(MT) for n in range(NT)]
