"""Host model check of the stream-K split used by the decode GEMM and the dgrad
(no GPU). The kernels cut W = tiles x stages-per-tile tile-stages into P equal
contiguous ranges, CTA b owning [range_lo(b), range_lo(b + 1)); a tile cut by
a range boundary is computed in pieces, each leaving its partial sums in a
slot of its CTA and counting itself on the counter of the tile's first CTA.
The arithmetic below restates the kernels' range_lo / cta_of / piece_slot
(csrc/lut_mma.cuh, csrc/decode_gemm.cu) and checks, over a grid of shapes
including fewer tile-stages than CTAs, that
  - every tile-stage belongs to exactly one CTA, and cta_of names it;
  - the pieces of a cut tile are exactly the CTAs cta_of(first) .. cta_of(last);
  - no two pieces share a partial-sum slot, and a reader finds each piece's slot;
  - a counter (indexed by the tile's first CTA) serves one cut tile only.
"""
import pytest


def range_lo(W, P, b):
    return (W * b) // P


def cta_of(W, P, s):
    return ((s + 1) * P - 1) // W


def piece_slot(W, P, KC, t, c):
    return c * 2 + (0 if range_lo(W, P, c) // KC == t else 1)


def check(T, KC, P):
    W = T * KC
    P = min(P, W)
    owner = [None] * W
    pieces, slots, counters = {}, {}, {}
    for b in range(P):
        lo, hi = range_lo(W, P, b), range_lo(W, P, b + 1)
        assert lo < hi                      # every CTA kept has work
        s = lo
        while s < hi:
            t = s // KC
            k0 = s - t * KC
            k1 = min(KC, k0 + (hi - s))
            for x in range(s, s + (k1 - k0)):
                assert owner[x] is None
                owner[x] = b
                assert cta_of(W, P, x) == b
            first, last = cta_of(W, P, t * KC), cta_of(W, P, t * KC + KC - 1)
            assert first <= b <= last
            assert (first == last) == (k0 == 0 and k1 == KC)   # whole tile <=> one CTA
            if first != last:
                sl = piece_slot(W, P, KC, t, b)
                assert 0 <= sl < 2 * P and sl not in slots
                slots[sl] = (t, b)
                assert counters.setdefault(first, t) == t
                pieces.setdefault(t, []).append(b)
            s += k1 - k0
    assert all(o is not None for o in owner)
    for t, cs in pieces.items():
        first, last = cta_of(W, P, t * KC), cta_of(W, P, t * KC + KC - 1)
        assert cs == list(range(first, last + 1))
        for c in cs:
            assert slots[piece_slot(W, P, KC, t, c)] == (t, c)


@pytest.mark.parametrize("T", [1, 2, 3, 7, 128, 147, 148, 149, 300, 1111])
def test_stream_k_pieces_and_slots(T):
    for KC in (1, 2, 3, 4, 8, 12, 32, 45):
        for P in (1, 2, 3, 64, 148):
            check(T, KC, P)
