"""Pins for the oracle's all-to-all (rco_all_to_all_v and all_to_all).

  * a hand-derived p = 2 example of the pages' primitive (golden file);
  * invariants: with equal splits the exchange is an involution (applying it
    twice gives the inputs back); with split counts, the return exchange with
    the transposed counts restores every rank's buffer (dispatch then
    combine); every element arrives at the rank it was sent to, blocks arrive
    in source-rank order, each block in its original order, nothing is lost;
  * the payload formula of the pages: with balanced routing a rank's logical
    payload per phase is t*k*h*b and t*k*h*b*(p-1)/p of it crosses ranks.
"""
import numpy as np
import pytest

import oracle
from conftest import golden


def _codes(p, counts):
    """Rank r's send buffer: block q holds code(r, q, j) = r<<40 | q<<20 | j."""
    out = []
    for r in range(p):
        blocks = [(np.uint64(r) << np.uint64(40)) | (np.uint64(q) << np.uint64(20)) |
                  np.arange(counts[r][q], dtype=np.uint64) for q in range(p)]
        out.append(np.concatenate(blocks) if blocks else np.zeros(0, np.uint64))
    return out


def test_golden_p2():
    g = golden("all_to_all_p2.json")
    sends = [np.array(x, np.int32) for x in g["send"]]
    got = oracle.all_to_all(sends)
    for q in range(g["p"]):
        assert got[q].tolist() == g["recv"][q]


@pytest.mark.parametrize("p,m,dt", [(2, 3, np.float32), (4, 1, np.int32), (8, 17, np.uint16), (16, 5, np.float64)])
def test_equal_splits_is_an_involution(p, m, dt):
    r = np.random.default_rng(p * 100 + m)
    xs = [r.integers(0, 1 << 15, p * m).astype(dt) for _ in range(p)]
    back = oracle.all_to_all(oracle.all_to_all(xs))
    for a, b in zip(xs, back):
        assert np.array_equal(a.view(np.uint8), b.view(np.uint8))


@pytest.mark.parametrize("p,seed", [(2, 1), (3, 2), (8, 3), (16, 4)])
def test_split_counts_route_every_element(p, seed):
    r = np.random.default_rng(seed)
    counts = r.integers(0, 40, (p, p))
    counts[r.integers(0, p), :] = 0          # a rank that sends nothing
    counts[:, r.integers(0, p)] = 0          # a rank that receives nothing
    sends = _codes(p, counts)
    recv = oracle.all_to_all_v(sends, counts)
    for q in range(p):
        code = recv[q]
        assert code.size == counts[:, q].sum()
        src = (code >> np.uint64(40)).astype(np.int64)
        dst = ((code >> np.uint64(20)) & np.uint64((1 << 20) - 1)).astype(np.int64)
        j = (code & np.uint64((1 << 20) - 1)).astype(np.int64)
        assert np.all(dst == q)                       # arrived where it was sent
        assert np.all(np.diff(src) >= 0)              # blocks in source-rank order
        for s in range(p):                            # each block whole and in order
            assert np.array_equal(j[src == s], np.arange(counts[s][q]))
    # dispatch then combine (transposed counts) restores every rank's buffer
    back = oracle.all_to_all_v(recv, counts.T)
    for a, b in zip(sends, back):
        assert np.array_equal(a, b)


def test_payload_formula_balanced_routing():
    # t tokens per rank, top-k, hidden h, b bytes per element, EP group p
    t, k, h, b, p = 64, 2, 48, 2, 8
    per_pair = t * k * h // p                          # elements r -> q, balanced
    counts = np.full((p, p), per_pair, np.uint64)
    sends = [np.zeros(t * k * h, np.uint16) for _ in range(p)]
    tr = [0, 0]
    oracle.all_to_all_v(sends, counts, traffic=tr)
    assert tr[0] + tr[1] == p * t * k * h * b          # logical payload t*k*h*b per rank
    assert tr[1] == p * t * k * h * b * (p - 1) // p   # t*k*h*b*(p-1)/p crosses ranks, per rank
