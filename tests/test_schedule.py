"""The stream-K schedule of the GEMM kernels, evaluated on the host by the
library's own code (skinny_debug_schedule), against the properties the
kernel's split-K fixup relies on:

  * the CTAs' ranges partition the tiles, in CTA order;
  * the reported first/last row tiles and their lowest/highest sharers are
    those of the ranges;
  * every CTA publishes partial sums for at most one row tile (one slot);
  * the finisher of a shared row tile is its highest contributor, which
    reaches that row tile LAST in its backwards walk (its first row tile),
    while every other contributor reaches it first or holds nothing else;
  * so a finisher only ever waits for lower-numbered CTAs;
  * the ranges differ by at most one quantum, longest first (the CTAs that
    are dispatched first take the longer ranges);
  * without split-K every row tile has exactly one contributor.
"""
import ctypes

import numpy as np
import pytest

import fp8_weight_only_w4a16_b200 as sk

SHAPES = [(128, 16), (130, 150016), (256, 512), (300, 1040), (1000, 2048), (5120, 5120), (34816, 5120),
          (5120, 17408), (151936, 5120), (257, 144), (64, 64000)]


def schedule(N, K, sms, split):
    cap = 4096
    out = (ctypes.c_int * (6 * cap))()
    ctas = ctypes.c_int(0)
    st = sk.library().skinny_debug_schedule(N, K, sms, split, out, cap, ctypes.byref(ctas))
    assert st == sk.OK, sk.status_string(st)
    return np.array(out[:6 * ctas.value]).reshape(ctas.value, 6)


@pytest.mark.parametrize("N,K", SHAPES)
@pytest.mark.parametrize("sms", [1, 7, 148, 160])
@pytest.mark.parametrize("split", [1, 0])
def test_schedule_properties(N, K, sms, split):
    C = -(-K // 512)
    G = -(-N // 128)
    U = G * C
    s = schedule(N, K, sms, split)
    P = s.shape[0]
    assert P == min(sms, U if split else G)
    u_last, n_units, first_g, last_g, first_owner, last_owner = s.T
    u_begin = u_last - n_units + 1
    # a partition of [0, U) in CTA order, every range non-empty
    assert u_begin[0] == 0 and u_last[-1] == U - 1 and np.all(n_units >= 1)
    assert np.all(u_begin[1:] == u_last[:-1] + 1)
    assert np.all(first_g == u_begin // C) and np.all(last_g == u_last // C)
    owner = np.repeat(np.arange(P), n_units)               # owner[u]
    for b in range(P):
        assert first_owner[b] == owner[first_g[b] * C]
        assert last_owner[b] == owner[last_g[b] * C + C - 1]
    # contributors of each row tile, and the publications they imply
    publishes = np.zeros(P, int)
    for g in range(G):
        cs = np.unique(owner[g * C:(g + 1) * C])
        c_first, c_last = cs[0], cs[-1]
        if not split:
            assert c_first == c_last
        if c_first == c_last:
            continue
        # the finisher reaches g last: g is the first row tile of its range
        assert first_g[c_last] == g
        for c in cs[:-1]:
            publishes[c] += 1
            # a publisher reaches g first (its last row tile) or g is all it holds
            assert last_g[c] == g
        assert np.all(cs[:-1] < c_last)                     # waits only on lower CTAs
    assert np.all(publishes <= 1)
    # CTAs dispatched first (lower numbers) take the longer ranges: lengths
    # differ by at most one quantum and never increase with the CTA number
    quantum = 1 if split else C
    assert n_units.max() - n_units.min() <= quantum
    assert np.all(np.diff(n_units) <= 0)


def test_schedule_rejects_bad_arguments():
    out = (ctypes.c_int * 6)()
    ctas = ctypes.c_int(0)
    lib = sk.library()
    assert lib.skinny_debug_schedule(128, 40, 148, 1, out, 1, ctypes.byref(ctas)) == sk.ERR_INVALID_ARG
    assert lib.skinny_debug_schedule(5120, 5120, 148, 1, out, 1, ctypes.byref(ctas)) == sk.ERR_WORKSPACE
    assert ctas.value == 148
