"""Piece planning of the host-buffer pipelines (attn_fwd_host,
attn_fwd_varlen_host), on the CPU: every head (every sequence) lands in
exactly one piece, and the job's first and last pieces are the small ones."""
from __future__ import annotations

import random

import pytest

from quantized_attention_07_b200.api import dense_host_pieces, varlen_host_order


@pytest.mark.parametrize("B,Hkv,per", [(1, 32, 2), (1, 24, 6), (2, 16, 16), (1, 8, 2),
                                       (1, 1, 1), (2, 1, 1), (1, 2, 2), (3, 4, 4), (1, 6, 4)])
def test_dense_pieces_cover_every_head_once_with_one_head_ends(B, Hkv, per):
    p = dense_host_pieces(B, Hkv, per)
    covered = sorted((b, h) for b, h0, nh in p for h in range(h0, h0 + nh))
    assert covered == [(b, h) for b in range(B) for h in range(Hkv)]
    assert all(1 <= nh <= per for _, _, nh in p)
    assert p[0][2] == 1 and p[-1][2] == 1
    # pieces stay within one batch entry and are contiguous runs of heads
    assert all(h0 + nh <= Hkv for _, h0, nh in p)


def test_varlen_order_is_a_permutation_with_the_smallest_ends():
    rng = random.Random(5)
    for _ in range(300):
        n = rng.randint(1, 9)
        cu = [0]
        for _ in range(n):
            cu.append(cu[-1] + rng.randint(0, 60))
        pieces = [(i, i + 1) for i in range(n)]
        got = varlen_host_order(pieces, cu)
        assert sorted(got) == pieces
        if n > 2:
            size = lambda x: cu[x[1]] - cu[x[0]]
            s = sorted(size(x) for x in pieces)
            assert size(got[0]) == s[0] and size(got[-1]) == s[1]
            # the middle keeps its order
            mid = [x for x in pieces if x not in (got[0], got[-1])]
            assert got[1:-1] == mid
