"""Host checks of the decode GEMV's stream-K schedule (no GPU).

The schedule, as the GEMV states it: output channels in groups of 8 row blocks
(128 channels, the last group possibly shorter); each group's K in units of KU
k-blocks, UPG = ceil(KB / KU) units per group; the U = groups x UPG units in
group-major order, CTA c of P taking the units [c U / P, (c + 1) U / P). A CTA
writes fp16 y for every group whose units it holds all of. For a group it holds
only part of, it writes fp32 partial sums into its slot 0 if that group is its
first, into slot 1 otherwise. The fixup kernel finds the contributors of a
group as the CTAs from cta_of(first unit) to cta_of(last unit); it reads the
first one's slot 0 if that CTA's range starts at the group's first unit and its
slot 1 otherwise, then slot 0 of every later one, and adds them in CTA order.

This module models that schedule in Python and checks, for many shapes and CTA
counts:
- every (group, unit) is computed by exactly one CTA, and cta_of inverts the
  range split;
- each group is either written whole by one CTA, or summed by the fixup from
  exactly the CTAs that hold its units, each part read from the slot it was
  written to, and no CTA writes two groups into one slot;
- the library plans what the model says at M = 1: the GEMV alone when no CTA
  boundary falls inside a group, else the GEMV and its fixup (launch counts for
  148 SMs, the count the library assumes without a device).
"""
import pytest

import weight_only_bit_awq_b200 as awq

SMS = 148            # SM count the library plans for without a device
CTAS_PER_SM = 2      # resident GEMV CTAs per SM at M <= 16


def cdiv(a, b):
    return -(-a // b)


def first_unit(c, U, P):
    return c * U // P


def cta_of(u, U, P):
    return ((u + 1) * P - 1) // U


def schedule(groups, UPG, P):
    """What each CTA writes: direct[g] = CTA that wrote group g as fp16;
    slots[(c, s)] = group whose partial sums CTA c wrote into its slot s."""
    U = groups * UPG
    direct, slots, owner = {}, {}, {}
    for c in range(P):
        u0, u1 = first_unit(c, U, P), first_unit(c + 1, U, P)
        for u in range(u0, u1):
            assert u not in owner, f"unit {u} computed twice"
            owner[u] = c
        if u1 == u0:
            continue
        g_first = u0 // UPG
        for g in range(g_first, (u1 - 1) // UPG + 1):
            if u0 <= g * UPG and (g + 1) * UPG <= u1:
                assert g not in direct
                direct[g] = c
            else:
                s = 0 if g == g_first else 1
                assert (c, s) not in slots, f"CTA {c} writes two groups into slot {s}"
                slots[(c, s)] = g
    assert sorted(owner) == list(range(U)), "some unit is computed by no CTA"
    return direct, slots, owner


def check_fixup(groups, UPG, P):
    U = groups * UPG
    direct, slots, owner = schedule(groups, UPG, P)
    for u in range(U):
        assert cta_of(u, U, P) == owner[u]
    for g in range(groups):
        holders = sorted({owner[u] for u in range(g * UPG, (g + 1) * UPG)})
        c_first, c_last = cta_of(g * UPG, U, P), cta_of((g + 1) * UPG - 1, U, P)
        assert list(range(c_first, c_last + 1)) == holders
        if c_first == c_last:
            assert direct.get(g) == c_first
            assert all(v != g for v in slots.values())
            continue
        assert g not in direct
        which_first = 0 if first_unit(c_first, U, P) == g * UPG else 1
        reads = [(c_first, which_first)] + [(c, 0) for c in range(c_first + 1, c_last + 1)]
        for c, s in reads:
            assert slots.get((c, s)) == g, f"group {g}: CTA {c} slot {s} holds {slots.get((c, s))}"
        assert sum(1 for v in slots.values() if v == g) == len(reads)


@pytest.mark.parametrize("groups,UPG", [(1, 1), (1, 8), (3, 5), (32, 8), (96, 8), (172, 8), (32, 22), (224, 8),
                                        (448, 16), (64, 56), (7, 3), (13, 17)])
def test_every_unit_once_and_parts_where_the_fixup_reads_them(groups, UPG):
    U = groups * UPG
    cands = {1, 2, 3, 7, 148, 296, U // 2, U - 1, U}
    for P in sorted(p for p in cands if 1 <= p <= U):
        check_fixup(groups, UPG, P)


def test_exhaustive_small_schedules():
    for groups in range(1, 9):
        for UPG in range(1, 9):
            for P in range(1, groups * UPG + 1):
                check_fixup(groups, UPG, P)


def plan_m1(K, N):
    """The plan at M = 1, groups of 128 (integer path): units of 4 k-blocks
    unless that gives fewer units than SMs (then 2, then 1), on
    min(U, 2 x SMs) CTAs. Returns (groups, UPG, P)."""
    KB, NB = K // 128, N // 16
    groups = cdiv(NB, 8)
    for ku in (4, 2, 1):
        U = groups * cdiv(KB, ku)
        if ku != 1 and (ku > KB or U < SMS):
            continue
        return groups, cdiv(KB, ku), min(U, CTAS_PER_SM * SMS)


@pytest.mark.parametrize("K", [128, 512, 1024, 4096, 8192, 11008, 14336, 28672])
@pytest.mark.parametrize("N", [16, 272, 4096, 6144, 12288, 18944, 22016, 28672, 37888, 57344])
def test_the_library_plans_the_fixup_the_model_needs(K, N):
    groups, UPG, P = plan_m1(K, N)
    has_split = any(first_unit(c, groups * UPG, P) % UPG != 0 for c in range(1, P))
    assert awq.awq_linear_launches(1, K, N, 128) == (2 if has_split else 1)
