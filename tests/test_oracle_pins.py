"""Pins for the CPU oracle: values the pages print, hand-derived cases of the
pages' ring and hierarchical procedures, closed forms, identities, brute force
and IEEE rounding.  CPU only.

A plausible slip anywhere in the oracle -- a dropped rank, a wrong sign, the
fold starting at the wrong rank, operands swapped in a compare-select, the
scale applied per term, a wrong reduce_scatter slice, a wrong rounding rule,
strided instead of contiguous groups -- breaks at least one test here;
test_oracle_mutations.py plants each of those slips in a copy of the oracle
and checks that this file's pins catch it.
"""
import math
import struct
from fractions import Fraction

import numpy as np
import pytest
import torch

from conftest import golden
import rc_inputs

DTS = ["f32", "bf16", "i32"]
OPS = ["sum", "max", "min"]


def _bits(a):
    a = np.asarray(a)
    if a.dtype == np.float32:
        return a.view(np.uint32)
    return a


def assert_bits_equal(a, b):
    np.testing.assert_array_equal(_bits(a), _bits(b))


# ---------------------------------------------------------------- page values
def test_worked_example(oracle_mod):
    g = golden("worked_example.json")
    xs = [np.array(v, np.float32) for v in g["inputs"]]
    # the shared generator reproduces the page's inputs
    for a, b in zip(xs, rc_inputs.worked_example()):
        assert_bits_equal(a, b)
    for y in oracle_mod.all_reduce(xs):
        assert y.tolist() == g["all_reduce_sum"]
    rs = oracle_mod.reduce_scatter(xs)
    assert [y.tolist() for y in rs] == g["reduce_scatter_sum"]
    for y in oracle_mod.all_gather(rs):
        assert y.tolist() == g["all_gather_of_reduce_scatter"]
    for root in range(4):
        assert oracle_mod.reduce(xs, root=root).tolist() == g["all_reduce_sum"]
    for y in oracle_mod.ring_all_reduce(xs):
        assert y.tolist() == g["all_reduce_sum"]


def test_ring_order_golden(oracle_mod):
    """The ring order decides the rounding; hand-derived from the ring steps."""
    g = golden("ring_order_fp32.json")
    xs = [np.array(v, np.float32) for v in g["inputs"]]
    exact = [float(sum(Fraction(float(x[i])) for x in xs)) for i in range(4)]
    assert exact == g["exact_sum"]
    for y in oracle_mod.all_reduce(xs):
        assert y.tolist() == g["all_reduce_sum"]
    for y in oracle_mod.ring_all_reduce(xs):
        assert y.tolist() == g["all_reduce_sum"]
    assert [v for y in oracle_mod.reduce_scatter(xs) for v in y.tolist()] == g["all_reduce_sum"]
    assert oracle_mod.reduce(xs, root=2).tolist() == g["all_reduce_sum"]


def test_signed_zero_compare_select(oracle_mod):
    g = golden("max_signed_zero.json")
    xs = [np.array(v, np.uint32).view(np.float32) for v in g["inputs_bits"]]
    for op, key in (("max", "max_bits"), ("min", "min_bits")):
        for y in oracle_mod.all_reduce(xs, op=op):
            assert y.view(np.uint32).tolist() == g[key]
        for y in oracle_mod.ring_all_reduce(xs, op=op):
            assert y.view(np.uint32).tolist() == g[key]


def test_hier_groups_golden(oracle_mod):
    g = golden("hier_groups_fp32.json")
    xa = [np.array(v, np.float32) for v in g["case_a_inputs"]]
    xb = [np.array(v, np.float32) for v in g["case_b_inputs"]]
    for y in oracle_mod.hier_all_reduce(xa, g["group_size"]):
        assert y[0] == g["case_a_hier_elem0"]
    assert oracle_mod.all_reduce(xa)[0][0] == g["case_a_flat_elem0"]
    for y in oracle_mod.hier_all_reduce(xb, g["group_size"]):
        assert y[0] == g["case_b_hier_elem0"]


def test_bf16_rounding_golden(oracle_mod):
    g = golden("bf16_rounding.json")
    f = np.array([c[0] for c in g["cases"]], np.uint32).view(np.float32)
    want = np.array([c[1] for c in g["cases"]], np.uint16)
    np.testing.assert_array_equal(oracle_mod.f32_to_bf16(f), want)


def test_bf16_rounding_matches_torch(oracle_mod):
    """torch's fp32 -> bf16 cast is round-to-nearest-even: a library routine
    the oracle's own narrowing must agree with, ties and edges included."""
    rng = np.random.default_rng(7)
    u = rng.integers(0, 2**32, 200_000, dtype=np.uint64).astype(np.uint32)
    ties = (rng.integers(0, 2**16, 50_000, dtype=np.uint64).astype(np.uint32) << 16) | 0x8000
    near = ties[:20000] + np.uint32(1)
    x = np.concatenate([u, ties, near]).view(np.float32)
    x = x[~np.isnan(x)]
    want = torch.from_numpy(x.copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(oracle_mod.f32_to_bf16(x), want)


def test_busbw_formula_matches_page_table():
    """The pages' bus-bandwidth accounting reproduces their printed table
    (p = 4, 100*1024^2 four-byte elements, GiB/s)."""
    import bench
    s = 4 * 100 * 1024 ** 2
    ar = [bench.busbw_all_reduce(s, 4, t * 1e-3) / 2 ** 30 for t in (1.60, 1.50, 1.38, 1.38)]
    assert [round(v) for v in ar] == [366, 391, 425, 425]   # page: 366 / 390 / 426 / 425
    assert all(abs(a - b) <= 1.5 for a, b in zip(ar, [366, 390, 426, 425]))
    rs = [bench.busbw_reduce_scatter(4 * s, 4, t * 1e-3) / 2 ** 30 for t in (2.61, 2.47, 2.39, 2.39)]
    assert all(abs(a - b) <= 1.5 for a, b in zip(rs, [450, 475, 490, 490]))


# ---------------------------------------------------------------- closed forms
@pytest.mark.parametrize("p", [1, 2, 3, 4, 5, 8, 16])
@pytest.mark.parametrize("n", [1, 3, 7, 64, 1000])
def test_closed_form_sum(oracle_mod, p, n):
    """x_r[i] = i + r  =>  sum = p*i + p(p-1)/2, max = i + p - 1, min = i."""
    i = np.arange(n)
    xs = [(i + r).astype(np.float32) for r in range(p)]
    want = (p * i + p * (p - 1) // 2).astype(np.float32)
    for y in oracle_mod.all_reduce(xs):
        assert_bits_equal(y, want)
    for y in oracle_mod.ring_all_reduce(xs):
        assert_bits_equal(y, want)
    for y in oracle_mod.hier_all_reduce(xs, 1):
        assert_bits_equal(y, want)
    assert_bits_equal(oracle_mod.all_reduce(xs, op="max")[0], (i + p - 1).astype(np.float32))
    assert_bits_equal(oracle_mod.all_reduce(xs, op="min")[-1], i.astype(np.float32))
    xi = [(i + r).astype(np.int32) for r in range(p)]
    assert_bits_equal(oracle_mod.all_reduce(xi, "i32")[0], want.astype(np.int32))
    if p * (n + p) < 256:   # every value and partial exact in bf16's 8 bits
        xb = [oracle_mod.f32_to_bf16(x) for x in xs]
        assert_bits_equal(oracle_mod.bf16_to_f32(oracle_mod.all_reduce(xb, "bf16")[-1]), want)
    if n % p == 0:
        rs = oracle_mod.reduce_scatter(xs)
        assert_bits_equal(np.concatenate(rs), want)


@pytest.mark.parametrize("p", [2, 4, 8, 16])
def test_closed_form_scale(oracle_mod, p):
    """AVG as sum times 1/p: exact for these integers since p is a power of two."""
    n = 4096
    i = np.arange(n)
    xs = [(i + r).astype(np.float32) for r in range(p)]
    want = ((p * i + p * (p - 1) // 2) / p).astype(np.float32)
    assert_bits_equal(oracle_mod.all_reduce(xs, scale=1.0 / p)[0], want)
    rs = oracle_mod.reduce_scatter(xs, "f32", "bf16", scale=1.0 / p)
    ref = torch.from_numpy(want).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert_bits_equal(np.concatenate(rs), ref)


def test_int32_wraps(oracle_mod):
    xs = [np.array([2**31 - 1, -2**31, 5], np.int32), np.array([1, -1, -7], np.int32)]
    y = oracle_mod.all_reduce(xs, "i32")[0]
    assert y.tolist() == [-2**31, 2**31 - 1, -2]


# ---------------------------------------------------------------- identities
def _data(p, n, dt, seed):
    if dt == "i32":
        return rc_inputs.int_uniform(p, n, seed)
    return rc_inputs.uniform(p, n, seed, dt)


@pytest.mark.parametrize("dt", DTS)
@pytest.mark.parametrize("op", OPS)
@pytest.mark.parametrize("p,n", [(2, 64), (3, 99), (4, 1000), (8, 4096), (16, 512)])
def test_identities(oracle_mod, dt, op, p, n):
    """all_reduce == all_gather(reduce_scatter) and == broadcast(reduce), bit for bit."""
    xs = _data(p, n, dt, seed=p * 1000 + n)
    ar = oracle_mod.all_reduce(xs, dt, op)
    for y in ar[1:]:
        assert_bits_equal(y, ar[0])
    ag = oracle_mod.all_gather(oracle_mod.reduce_scatter(xs, dt, dt, op), dt)
    for y in ag:
        assert_bits_equal(y, ar[0])
    for root in (0, p - 1):
        red = oracle_mod.reduce(xs, root, dt, op)
        for y in oracle_mod.broadcast(red, p, root, dt):
            assert_bits_equal(y, ar[0])


@pytest.mark.parametrize("p", [2, 4, 8])
def test_fused_cast_is_one_rounding(oracle_mod, p):
    """reduce_scatter fp32 -> bf16 with scale equals one RNE of the scaled fp32 all_reduce."""
    n = 8192
    xs = rc_inputs.normal(p, n, seed=11, sigma=1e-3)
    ar = oracle_mod.all_reduce(xs, "f32", "sum", scale=1.0 / p)[0]
    rs = np.concatenate(oracle_mod.reduce_scatter(xs, "f32", "bf16", "sum", 1.0 / p))
    assert_bits_equal(rs, oracle_mod.f32_to_bf16(ar))


# ---------------------------------------------------------------- ring literal
@pytest.mark.parametrize("p", [1, 2, 3, 4, 5, 7, 8, 9, 16])
@pytest.mark.parametrize("n", [1, 2, 5, 17, 64, 100, 1000])
def test_ring_equals_direct_fold(oracle_mod, p, n):
    """Two independent codings of one order: the step-by-step ring of the pages
    and the direct per-element fold.  Bit-exact for every dtype and op."""
    for dt in DTS:
        xs = _data(p, n, dt, seed=17 + p + n)
        for op in OPS:
            st = oracle_mod.RingStats(p)
            ring = oracle_mod.ring_all_reduce(xs, dt, op, stats=st)
            flat = oracle_mod.all_reduce(xs, dt, op)
            for a, b in zip(ring, flat):
                assert_bits_equal(a, b)
            assert int(st.steps[0]) == 2 * (p - 1)
            C = -(-n // p)
            if n % p == 0:
                assert st.elems_sent.tolist() == [2 * (p - 1) * C] * p


def test_ring_traffic_cost_model(oracle_mod):
    """Ring cost model: each of the N ranks sends S/N bytes per step over
    2(N-1) steps, so 2(N-1)/N * S per rank (reduce-scatter + all-gather)."""
    p, n = 8, 2097152
    xs = rc_inputs.normal(p, n, seed=1, sigma=1e-2)
    st = oracle_mod.RingStats(p)
    oracle_mod.ring_all_reduce(xs, stats=st)
    S = n * 4
    assert int(st.steps[0]) == 14
    for sent in st.elems_sent:
        assert int(sent) * 4 == 2 * (p - 1) * S // p


# ---------------------------------------------------------------- hierarchical
def test_hier_traffic_page_example(oracle_mod):
    """2 nodes x 4 GPUs, B = 8 MB each: 32 MB enters each node's step 1, a node
    sends B (8 MB) upward instead of B x N (32 MB): four times less."""
    p, G, n = 8, 4, 4194304  # bf16: 8 MiB per rank
    xs = rc_inputs.normal(p, n, seed=2, sigma=1.0, dt="bf16")
    t = np.zeros(4, np.uint64)
    oracle_mod.hier_all_reduce(xs, G, "bf16", traffic=t)
    ng, s = p // G, 2
    assert int(t[0]) * s // ng == 32 * 2**20
    assert int(t[1]) * s == 8 * 2**20
    assert int(t[2]) * s == 32 * 2**20
    assert int(t[2]) // int(t[1]) == G


@pytest.mark.parametrize("p,G", [(8, 4), (8, 2), (4, 2), (16, 4), (6, 3)])
def test_hier_vs_flat(oracle_mod, p, G):
    n = 3000
    for dt in DTS:
        xs = _data(p, n, dt, seed=p * 10 + G)
        for op in OPS:
            h = oracle_mod.hier_all_reduce(xs, G, dt, op)
            f = oracle_mod.all_reduce(xs, dt, op)
            if dt == "i32" or op != "sum":
                for a, b in zip(h, f):     # order-free results
                    assert_bits_equal(a, b)
            elif dt == "f32":
                xa = np.abs(np.stack(xs).astype(np.float64)).sum(0)
                bound = p * 2.0 ** -24 * xa
                assert np.all(np.abs(h[0].astype(np.float64) - f[0]) <= bound)
            else:
                hf = oracle_mod.bf16_to_f32(h[0]).astype(np.float64)
                ff = oracle_mod.bf16_to_f32(f[0]).astype(np.float64)
                xa = np.abs(np.stack([oracle_mod.bf16_to_f32(x) for x in xs]).astype(np.float64)).sum(0)
                ulp = np.abs(ff) * 2.0 ** -7 + 2.0 ** -133
                assert np.all(np.abs(hf - ff) <= p * 2.0 ** -24 * xa + ulp)


@pytest.mark.parametrize("G", [2, 3])
def test_hier_order_closed_form(oracle_mod, G):
    """Hand-derived values where only the two-level ring order gives the
    right bits (p = 6).  Element 0 lies in chunk 0 at both levels, so a
    group of size G folds its local ranks 1, 2, ..., 0 and the leaders fold
    groups 1, 2, ..., 0.  With a = 2^24: (a + 1) rounds to a (tie to even),
    so (a + 1) + (-a) = 0, while any other association of {a, 1, -a} gives 1.
    G = 2 (three groups) puts a, 1, -a in groups 1, 2, 0; G = 3 (one group
    of three ranks with the result) puts them on local ranks 1, 2, 0."""
    p, n, a = 6, 6, np.float32(2.0 ** 24)
    xs = [np.zeros(n, np.float32) for _ in range(p)]
    if G == 2:   # group g = ranks 2g, 2g+1; S_g = x_{2g+1} + x_{2g}
        xs[3][0], xs[5][0], xs[1][0] = a, 1.0, -a
    else:        # group 0 = ranks 0, 1, 2 folded 1, 2, 0; group 1 is zero
        xs[1][0], xs[2][0], xs[0][0] = a, 1.0, -a
    for y in oracle_mod.hier_all_reduce(xs, G):
        assert y[0] == 0.0 and not np.signbit(y[0])
    # the flat ring order (ranks 1, 2, 3, 4, 5, 0) over the same data: for
    # G = 2 it meets -a first and ends at 1; for G = 3 it matches the groups'
    flat = oracle_mod.all_reduce(xs)[0][0]
    assert flat == (1.0 if G == 2 else 0.0)


def test_hier_degenerate_groups_equal_flat(oracle_mod):
    """G = p (one group) and G = 1 (p groups of one) are the flat ring order."""
    p, n = 8, 4096
    xs = rc_inputs.uniform(p, n, seed=5)
    f = oracle_mod.all_reduce(xs)
    for G in (1, p):
        for a, b in zip(oracle_mod.hier_all_reduce(xs, G), f):
            assert_bits_equal(a, b)


# ---------------------------------------------------------------- brute force
@pytest.mark.parametrize("seed", range(12))
def test_brute_force_tiny(oracle_mod, seed):
    rng = np.random.default_rng(seed)
    p = int(rng.integers(1, 5))
    n = int(rng.integers(1, 17))
    xs = [rng.standard_normal(n).astype(np.float32) * np.float32(10.0 ** rng.integers(-3, 4))
          for _ in range(p)]
    y = oracle_mod.all_reduce(xs)[0]
    for i in range(n):
        exact = sum(Fraction(float(x[i])) for x in xs)
        bound = p * 2.0 ** -24 * sum(abs(float(x[i])) for x in xs)
        assert abs(float(Fraction(float(y[i])) - exact)) <= bound
    assert oracle_mod.all_reduce(xs, op="max")[0].tolist() == [max(float(x[i]) for x in xs) for i in range(n)]
    assert oracle_mod.all_reduce(xs, op="min")[0].tolist() == [min(float(x[i]) for x in xs) for i in range(n)]
    xi = [rng.integers(-2**31, 2**31, n, dtype=np.int64).astype(np.int32) for _ in range(p)]
    yi = oracle_mod.all_reduce(xi, "i32")[0]
    for i in range(n):
        s = sum(int(x[i]) for x in xi) % 2**32
        assert int(yi[i]) % 2**32 == s


@pytest.mark.parametrize("seed", range(6))
def test_brute_force_bf16(oracle_mod, seed):
    """bf16 result = one RNE of the fp32 sum: within half a bf16 ulp of the
    fp32 result, and the fp32 result within the fold bound of the exact sum."""
    rng = np.random.default_rng(100 + seed)
    p, n = int(rng.integers(2, 5)), int(rng.integers(1, 17))
    xs = rc_inputs.uniform(p, n, seed=seed, dt="bf16")
    y = oracle_mod.bf16_to_f32(oracle_mod.all_reduce(xs, "bf16")[0])
    xf = [oracle_mod.bf16_to_f32(x) for x in xs]
    for i in range(n):
        exact = sum(Fraction(float(x[i])) for x in xf)
        bound = p * 2.0 ** -24 * sum(abs(float(x[i])) for x in xf)
        half_ulp = 2.0 ** (math.frexp(float(y[i]))[1] - 9) if y[i] != 0 else 2.0 ** -134
        assert abs(float(Fraction(float(y[i])) - exact)) <= bound + half_ulp


# ---------------------------------------------------------------- arguments
def test_invalid_arguments(oracle_mod):
    xs = rc_inputs.uniform(4, 10, seed=0)
    with pytest.raises(oracle_mod.OracleError):
        oracle_mod.reduce_scatter(xs)                          # 4 does not divide 10
    with pytest.raises(oracle_mod.OracleError):
        oracle_mod.all_reduce(xs, op="max", scale=0.5)         # scale only for fp sum
    with pytest.raises(oracle_mod.OracleError):
        oracle_mod.all_reduce(rc_inputs.int_uniform(2, 8, 0), "i32", scale=0.5)
    with pytest.raises(oracle_mod.OracleError):
        oracle_mod.reduce(xs, root=4)
    with pytest.raises(oracle_mod.OracleError):
        oracle_mod.hier_all_reduce(xs, 3)


# ---------------------------------------------------------------- sampled form
# reduce_at(xs, idx) returns y[idx[j]] for selected indices only; the GPU tests
# use it as the checker for full-size outputs.  Its own loop, index check and
# output store are pinned here: by the hand-derived ring-order case, by the
# closed forms, and by agreement with the pinned all_reduce / reduce_scatter
# (y = sum_r x_r of "分布式训练/推理", section "通信原语：rank、world size 和
# collective operations", in the ring order of "LLM Parallelism 基础", section
# "Ring AllReduce").
def _boundaries(n, p):
    """Every chunk boundary +-1, the first and the last index, clipped to [0, n)."""
    C = -(-n // p)
    idx = {0, n - 1}
    for c in range(1, p + 1):
        for d in (-1, 0, 1):
            if 0 <= c * C + d < n:
                idx.add(c * C + d)
    return np.array(sorted(idx), np.uint64)


def test_reduce_at_ring_order_golden(oracle_mod):
    """The hand-derived ring-order case, sampled in a shuffled order with a
    repeated index: every element is 0 in ring order (2 in rank order)."""
    g = golden("ring_order_fp32.json")
    xs = [np.array(v, np.float32) for v in g["inputs"]]
    idx = np.array([3, 0, 2, 1, 0], np.uint64)
    got = oracle_mod.reduce_at(xs, idx)
    assert got.tolist() == [g["all_reduce_sum"][int(i)] for i in idx]
    assert got.dtype == np.float32


@pytest.mark.parametrize("p", [1, 2, 3, 5, 8, 16])
@pytest.mark.parametrize("n", [1, 7, 1000, 4099])
def test_reduce_at_closed_form(oracle_mod, p, n):
    """x_r[i] = i + r: y[i] = p*i + p(p-1)/2, max i + p - 1, min i, at every
    chunk boundary +-1 and at random indices, in the order asked for."""
    i = np.arange(n)
    rng = np.random.default_rng(p * 7919 + n)
    idx = np.concatenate([_boundaries(n, p), rng.integers(0, n, 64, dtype=np.uint64)])
    rng.shuffle(idx)
    ii = idx.astype(np.int64)
    xs = [(i + r).astype(np.float32) for r in range(p)]
    want = (p * ii + p * (p - 1) // 2).astype(np.float32)
    assert_bits_equal(oracle_mod.reduce_at(xs, idx), want)
    assert_bits_equal(oracle_mod.reduce_at(xs, idx, op="max"), (ii + p - 1).astype(np.float32))
    assert_bits_equal(oracle_mod.reduce_at(xs, idx, op="min"), ii.astype(np.float32))
    xi = [(i + r).astype(np.int32) for r in range(p)]
    assert_bits_equal(oracle_mod.reduce_at(xi, idx, "i32"), want.astype(np.int32))
    if p & (p - 1) == 0:
        # AVG as x 1/p (exact for a power of two), narrowed once to bf16:
        # torch's fp32 -> bf16 cast is round-to-nearest-even
        avg = ((p * ii + p * (p - 1) // 2) / p).astype(np.float32)
        ref = torch.from_numpy(avg).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
        got = oracle_mod.reduce_at(xs, idx, "f32", "bf16", scale=1.0 / p)
        assert got.dtype == np.uint16
        assert_bits_equal(got, ref)


@pytest.mark.parametrize("dt", DTS)
@pytest.mark.parametrize("p,n", [(2, 63), (3, 100), (4, 1000), (7, 4097), (8, 4096), (16, 1023)])
def test_reduce_at_matches_all_reduce(oracle_mod, dt, p, n):
    """Order-sensitive random data: the sampled values equal the all-reduce's
    at every chunk boundary +-1 and at shuffled random indices, every op."""
    xs = _data(p, n, dt, seed=31 * p + n)
    rng = np.random.default_rng(n)
    idx = np.concatenate([_boundaries(n, p), rng.integers(0, n, 200, dtype=np.uint64)])
    rng.shuffle(idx)
    for op in OPS:
        full = oracle_mod.all_reduce(xs, dt, op)[0]
        assert_bits_equal(oracle_mod.reduce_at(xs, idx, dt, op=op), full[idx.astype(np.int64)])


@pytest.mark.parametrize("p,n", [(2, 64), (4, 4096), (8, 8192), (16, 2048)])
def test_reduce_at_matches_reduce_scatter_cast(oracle_mod, p, n):
    """fp32 gradients -> bf16 with scale 1/p (the fused reduce_scatter of the
    FSDP step): the sampled values equal the reduce_scatter's shards."""
    xs = rc_inputs.normal(p, n, seed=40 + p, sigma=1e-3)
    rs = np.concatenate(oracle_mod.reduce_scatter(xs, "f32", "bf16", "sum", 1.0 / p))
    idx = np.concatenate([_boundaries(n, p), np.arange(0, n, 3, dtype=np.uint64)])
    got = oracle_mod.reduce_at(xs, idx, "f32", "bf16", "sum", 1.0 / p)
    assert_bits_equal(got, rs[idx.astype(np.int64)])
    # and every index at once, in order
    assert_bits_equal(oracle_mod.reduce_at(xs, np.arange(n, dtype=np.uint64), "f32", "bf16", "sum",
                                           1.0 / p), rs)


def test_reduce_at_index_range(oracle_mod):
    """Index n is past the end and is rejected; n - 1 and no index at all are fine."""
    p, n = 4, 10
    xs = rc_inputs.uniform(p, n, seed=0)
    full = oracle_mod.all_reduce(xs)[0]
    assert_bits_equal(oracle_mod.reduce_at(xs, np.array([n - 1], np.uint64)), full[-1:])
    assert oracle_mod.reduce_at(xs, np.zeros(0, np.uint64)).size == 0
    with pytest.raises(oracle_mod.OracleError):
        oracle_mod.reduce_at(xs, np.array([0, n], np.uint64))
    with pytest.raises(oracle_mod.OracleError):
        oracle_mod.reduce_at(xs, np.array([1], np.uint64), op="max", scale=0.5)
