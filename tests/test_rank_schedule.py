"""The rank-view ring schedule, simulated on the CPU: every rank pulls its
predecessor's message as the header of the library states it (reduce-scatter
step k: chunk (rank-k-2) mod p, the partial kept in the receiver's own output
buffer, the last step scaled into the output; all-gather step k: chunk
(rank-k-1) mod p copied from the predecessor), one step of every rank before
the next step of any.  This is a second derivation of the literal ring from
the "Ring AllReduce" section of "LLM Parallelism 基础" and must equal the
oracle's ring bit for bit; it pins the per-rank indexing that the rank view
documents, independently of the GPU."""
import numpy as np
import pytest

import oracle
import rc_inputs


def _pull_ring(xs, op, scale):
    p, n = len(xs), len(xs[0])
    C = -(-n // p)
    x = [np.array(v, copy=True) for v in xs]
    y = [np.zeros_like(v) for v in xs]
    isf = x[0].dtype == np.float32

    def comb(a, b):
        if op == "sum":
            return a + b  # float32 IEEE add, or int32 wrapping add
        if op == "max":
            return np.where(b > a, b, a)
        return np.where(b < a, b, a)

    def sl(c):
        return slice(min(n, c * C), min(n, (c + 1) * C))

    for k in range(p - 1):  # reduce-scatter
        for d in range(p):
            r = (d - 1) % p
            c = (d - k - 2) % p
            msg = x[r][sl(c)] if k == 0 else y[r][sl(c)]
            acc = comb(msg, x[d][sl(c)])
            if k == p - 2:
                assert c == d  # the receiver ends owning its own chunk
                if op == "sum" and isf and scale != 1.0:
                    acc = (acc * np.float32(scale)).astype(np.float32)
            y[d][sl(c)] = acc
    for k in range(p - 1):  # all-gather
        for d in range(p):
            r = (d - 1) % p
            c = (d - k - 1) % p
            y[d][sl(c)] = y[r][sl(c)]
    return y


@pytest.mark.parametrize("p", [2, 3, 4, 5, 8])
@pytest.mark.parametrize("n", [1, 7, 64, 1001])
@pytest.mark.parametrize("op", ["sum", "max", "min"])
def test_pull_ring_equals_oracle_ring_f32(p, n, op):
    xs = rc_inputs.uniform(p, n, seed=p * 100 + n)
    scale = 1.0 / p if op == "sum" else 1.0
    want = oracle.ring_all_reduce(xs, "f32", op, scale)
    got = _pull_ring(xs, op, scale)
    for r in range(p):
        assert np.array_equal(got[r].view(np.uint32), want[r].view(np.uint32)), (p, n, op, r)


@pytest.mark.parametrize("p", [2, 4, 7])
def test_pull_ring_equals_oracle_ring_i32(p):
    xs = rc_inputs.int_uniform(p, 333, seed=p)
    with np.errstate(over="ignore"):
        got = _pull_ring(xs, "sum", 1.0)
    want = oracle.ring_all_reduce(xs, "i32", "sum", 1.0)
    for r in range(p):
        assert np.array_equal(got[r], want[r])


def test_a_wrong_chunk_rule_is_caught():
    """Pulling chunk (rank-k-1) in the reduce-scatter (the all-gather's rule)
    breaks the fold: the check above would see it."""
    p, n = 4, 64
    xs = rc_inputs.uniform(p, n, seed=1)
    want = oracle.ring_all_reduce(xs, "f32", "sum", 1.0)
    C = n // p
    x = [v.copy() for v in xs]
    y = [np.zeros_like(v) for v in xs]
    for k in range(p - 1):
        for d in range(p):
            r, c = (d - 1) % p, (d - k - 1) % p
            s = slice(c * C, (c + 1) * C)
            y[d][s] = (x[r][s] if k == 0 else y[r][s]) + x[d][s]
    assert not all(np.array_equal(y[r], want[r]) for r in range(p))
