"""GPU parity: every collective of the CUDA library against the CPU oracle on
the same seeded inputs, compared bit for bit (the fold order, fp32
accumulation and bf16 rounding are part of the contract, so "within
tolerance" would hide a broken kernel).  Hierarchical vs flat all-reduce are
two different orders and are compared with the fold bound
|err| <= p * 2^-24 * sum_r |x_r| (plus one bf16 ulp for bf16 outputs).

Sizes: small cases the oracle runs in full (several tiles, ragged tails),
and the configs' full sizes -- compared in full where the oracle finishes in
seconds, else on sampled indices (chunk boundaries included).
"""
import numpy as np
import pytest
import torch

import oracle
import rc_inputs
from util import assert_bits, check_canary, empty_dev, to_dev, to_host

pytestmark = pytest.mark.gpu

DTS = ["f32", "bf16", "i32"]
OPS = ["sum", "max", "min"]
ESZ = {"f32": 4, "bf16": 2, "i32": 4}


@pytest.fixture(scope="module")
def rc():
    import collective_rc_all_b200 as m
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return m


def _data(p, n, dt, seed):
    if dt == "i32":
        return rc_inputs.int_uniform(p, n, seed)
    return rc_inputs.uniform(p, n, seed, dt)


def _sync(rc):
    torch.cuda.synchronize()
    rc.rc_stream_status()


# ------------------------------------------------------------ worked example
def test_worked_example(rc):
    xs = rc_inputs.worked_example()
    d, _ = to_dev(xs, "f32")
    y, _ = empty_dev(4, "f32", 4)
    rc.rc_all_reduce(d, y)
    rs, _ = empty_dev(1, "f32", 4)
    rc.rc_reduce_scatter(d, rs)
    ag, _ = empty_dev(4, "f32", 4)
    rc.rc_all_gather(rs, ag)
    ring, _ = empty_dev(4, "f32", 4)
    rc.rc_ring_all_reduce(d, ring)
    _sync(rc)
    for r in range(4):
        assert to_host(y[r], "f32").tolist() == [6, 10, 14, 18]
        assert to_host(rs[r], "f32").tolist() == [[6], [10], [14], [18]][r]
        assert to_host(ag[r], "f32").tolist() == [6, 10, 14, 18]
        assert to_host(ring[r], "f32").tolist() == [6, 10, 14, 18]


def test_ring_order_golden(rc):
    """Hand-derived ring-order case: the ring order gives 0, any other gives 2."""
    from conftest import golden
    g = golden("ring_order_fp32.json")
    xs = [np.array(v, np.float32) for v in g["inputs"]]
    d, _ = to_dev(xs, "f32")
    y, _ = empty_dev(4, "f32", 4)
    rc.rc_all_reduce(d, y)
    yr, _ = empty_dev(4, "f32", 4)
    rc.rc_ring_all_reduce(d, yr)
    _sync(rc)
    for r in range(4):
        assert to_host(y[r], "f32").tolist() == g["all_reduce_sum"]
        assert to_host(yr[r], "f32").tolist() == g["all_reduce_sum"]


# ------------------------------------------------------------ flat collectives
CASES = [(1, 37), (2, 64), (3, 1001), (4, 65536), (5, 3), (7, 7777), (8, 65536 + 8 * 13),
         (8, 2 * 2048 * 8 + 40), (16, 4096 * 16), (16, 33)]


@pytest.mark.parametrize("p,n", CASES)
@pytest.mark.parametrize("dt", DTS)
def test_all_reduce_reduce_broadcast(rc, p, n, dt):
    xs = _data(p, n, dt, seed=1000 + p * 7 + n)
    d, _ = to_dev(xs, dt)
    for op in OPS:
        want = oracle.all_reduce(xs, dt, op)
        y, back = empty_dev(n, dt, p)
        rc.rc_all_reduce(d, y, op=op)
        root = (p * 3 + 1) % p
        yr, back_r = empty_dev(n, dt, 1)
        rc.rc_reduce(d, yr[0], root=root, op=op)
        _sync(rc)
        for r in range(p):
            assert_bits(to_host(y[r], dt), want[r], f"all_reduce {dt} {op} rank {r}")
        assert_bits(to_host(yr[0], dt), want[0], f"reduce {dt} {op}")
        check_canary(back, n * ESZ[dt])
        check_canary(back_r, n * ESZ[dt])
    # broadcast of rank `root`'s input
    root = p - 1
    yb, back_b = empty_dev(n, dt, p)
    rc.rc_broadcast(d[root], yb, root=root)
    _sync(rc)
    for r in range(p):
        assert_bits(to_host(yb[r], dt), xs[root], f"broadcast {dt} rank {r}")
    check_canary(back_b, n * ESZ[dt])


@pytest.mark.parametrize("p,n", [(1, 40), (2, 64), (3, 999), (4, 65536), (8, 8 * 4104),
                                 (16, 16 * 2048 + 16 * 3), (5, 5)])
@pytest.mark.parametrize("in_dt,out_dt", [("f32", "f32"), ("bf16", "bf16"), ("i32", "i32"),
                                          ("f32", "bf16"), ("bf16", "f32")])
def test_reduce_scatter_all_gather(rc, p, n, in_dt, out_dt):
    xs = _data(p, n, in_dt, seed=2000 + p + n)
    d, _ = to_dev(xs, in_dt)
    m = n // p
    for op in OPS:
        scale = (1.0 / p) if (op == "sum" and in_dt != "i32") else 1.0
        want = oracle.reduce_scatter(xs, in_dt, out_dt, op, scale)
        y, back = empty_dev(m, out_dt, p)
        rc.rc_reduce_scatter(d, y, op=op, scale=scale)
        _sync(rc)
        for r in range(p):
            assert_bits(to_host(y[r], out_dt), want[r], f"reduce_scatter {in_dt}->{out_dt} {op} r{r}")
        check_canary(back, m * ESZ[out_dt])
        # all_gather of the shards restores the all-reduce (same dtype)
        ag, back_ag = empty_dev(n, out_dt, p)
        rc.rc_all_gather(y, ag)
        _sync(rc)
        want_ag = oracle.all_gather(want, out_dt)
        for r in range(p):
            assert_bits(to_host(ag[r], out_dt), want_ag[r], f"all_gather {out_dt} r{r}")
        check_canary(back_ag, n * ESZ[out_dt])


def test_identity_all_reduce_equals_rs_plus_ag(rc):
    p, n = 8, 8 * 40960
    xs = rc_inputs.normal(p, n, seed=5, sigma=1.0)
    d, _ = to_dev(xs, "f32")
    ar, _ = empty_dev(n, "f32", p)
    rs, _ = empty_dev(n // p, "f32", p)
    ag, _ = empty_dev(n, "f32", p)
    rc.rc_all_reduce(d, ar)
    rc.rc_reduce_scatter(d, rs)
    rc.rc_all_gather(rs, ag)
    _sync(rc)
    for r in range(p):
        assert_bits(to_host(ag[r], "f32"), to_host(ar[r], "f32"), "AR vs RS+AG")


# ------------------------------------------------------------ literal ring
# RC_RING_KERNEL value and RC_RING_XSMEM value of each ring kernel: the link
# kernel with its inputs staged in shared memory (default) or held in
# registers, the chain kernel, the element kernel
RING_KERNELS = {"link": ("2", "1"), "link_regs": ("2", "0"), "chain": ("1", "1"), "element": ("0", "1")}


def _ring_kernel(monkeypatch, kernel):
    k, xs = RING_KERNELS[kernel]
    monkeypatch.setenv("RC_RING_KERNEL", k)
    monkeypatch.setenv("RC_RING_XSMEM", xs)


@pytest.mark.parametrize("p,n", [(2, 64), (3, 1001), (3, 840), (4, 65536), (5, 12), (8, 8 * 1024 + 24),
                                 (8, 8 * 2112), (12, 760), (16, 16 * 512), (16, 120), (16, 100)])
@pytest.mark.parametrize("dt", DTS)
@pytest.mark.parametrize("kernel", sorted(RING_KERNELS))
def test_ring_literal(rc, p, n, dt, kernel, monkeypatch):
    """Every kernel that executes the ring's steps (selected with
    RC_RING_KERNEL; aligned vector paths where the chunk length allows,
    element-wise otherwise): ragged chunks ((12, 760): a short last chunk;
    (16, 120): an empty one), several tiles with a ragged last tile."""
    _ring_kernel(monkeypatch, kernel)
    xs = _data(p, n, dt, seed=3000 + p + n)
    d, _ = to_dev(xs, dt)
    for op in OPS:
        scale = 0.125 if (op == "sum" and dt != "i32") else 1.0
        want = oracle.ring_all_reduce(xs, dt, op, scale)
        y, back = empty_dev(n, dt, p)
        rc.rc_ring_all_reduce(d, y, op=op, scale=scale, variant="literal")
        _sync(rc)
        for r in range(p):
            assert_bits(to_host(y[r], dt), want[r], f"ring {dt} {op} r{r}")
        check_canary(back, n * ESZ[dt])


def test_ring_and_oneshot_p8_8mib_full_size(rc, monkeypatch):
    """8 ranks x 2,097,152 fp32 ~N(0, 1e-2), seed 1: literal 14-step ring (the
    link kernel, and the chain kernel) and one-shot, all bit-identical to the
    oracle's ring simulation."""
    cfg = rc_inputs.config("ring_p8_2m_f32")
    xs = rc_inputs.draw(cfg)
    p, n = cfg["p"], cfg["n"]
    want = oracle.ring_all_reduce(xs, "f32")
    d, _ = to_dev(xs, "f32")
    for variant, kernel in (("literal", "2"), ("literal", "1"), ("oneshot", "2")):
        monkeypatch.setenv("RC_RING_KERNEL", kernel)
        y, back = empty_dev(n, "f32", p)
        rc.rc_ring_all_reduce(d, y, variant=variant)
        _sync(rc)
        for r in range(p):
            assert_bits(to_host(y[r], "f32"), want[r], f"ring p8 8MiB {variant} kernel {kernel} r{r}")
        check_canary(back, n * 4)


def test_ring_bf16_p8_8mib_full_size(rc):
    """The same ring workload in bf16 (8 ranks x 4,194,304 bf16 ~N(0, 1),
    8 MiB per rank): fp32 partials between steps, one rounding at the end,
    bit-identical to the oracle's ring simulation."""
    p, n = 8, 4194304
    xs = rc_inputs.normal(p, n, seed=1, sigma=1.0, dt="bf16")
    want = oracle.ring_all_reduce(xs, "bf16")
    d, _ = to_dev(xs, "bf16")
    y, back = empty_dev(n, "bf16", p)
    rc.rc_ring_all_reduce(d, y)
    _sync(rc)
    for r in range(p):
        assert_bits(to_host(y[r], "bf16"), want[r], f"bf16 ring p8 8MiB r{r}")
    check_canary(back, n * 2)


@pytest.mark.parametrize("kernel", sorted(RING_KERNELS))
def test_ring_in_place(rc, kernel, monkeypatch):
    _ring_kernel(monkeypatch, kernel)
    p, n = 8, 8 * 4096
    for dt in DTS:
        xs = _data(p, n, dt, seed=77)
        want = oracle.ring_all_reduce(xs, dt)
        d, _ = to_dev(xs, dt)
        rc.rc_ring_all_reduce(d, d)
        _sync(rc)
        for r in range(p):
            assert_bits(to_host(d[r], dt), want[r], f"ring in place {dt} r{r}")


# ------------------------------------------------------------ hierarchical
@pytest.mark.parametrize("p,G,n", [(8, 4, 8 * 1024), (8, 2, 1000), (4, 2, 65536), (16, 4, 4096),
                                   (6, 3, 999), (8, 1, 512), (8, 8, 512), (2, 2, 10),
                                   (16, 8, 16 * 2048), (16, 2, 16 * 1024 + 64)])
@pytest.mark.parametrize("dt", DTS)
def test_hier(rc, p, G, n, dt):
    xs = _data(p, n, dt, seed=4000 + p * G + n)
    d, _ = to_dev(xs, dt)
    for op in OPS:
        scale = 0.125 if (op == "sum" and dt != "i32") else 1.0
        want = oracle.hier_all_reduce(xs, G, dt, op, scale)
        for variant in ("fused", "staged"):
            y, back = empty_dev(n, dt, p)
            rc.rc_hier_all_reduce(d, y, G, op=op, scale=scale, variant=variant)
            _sync(rc)
            for r in range(p):
                assert_bits(to_host(y[r], dt), want[r], f"hier {variant} {dt} {op} r{r}")
            check_canary(back, n * ESZ[dt])


def test_hier_2x4_bf16_full_size(rc):
    """2 groups x 4 ranks, bf16 4,194,304 per rank ~N(0,1), seed 2: fused and
    staged bit-identical to the oracle's 3-phase simulation; within the fold
    bound (+1 bf16 ulp) of the flat all-reduce."""
    cfg = rc_inputs.config("hier_2x4_4m_bf16")
    xs = rc_inputs.draw(cfg)
    p, n, G = cfg["p"], cfg["n"], cfg["group"]
    want = oracle.hier_all_reduce(xs, G, "bf16")
    d, _ = to_dev(xs, "bf16")
    for variant in ("fused", "staged"):
        y, back = empty_dev(n, "bf16", p)
        rc.rc_hier_all_reduce(d, y, G, variant=variant)
        _sync(rc)
        for r in range(p):
            assert_bits(to_host(y[r], "bf16"), want[r], f"hier 2x4 bf16 {variant} r{r}")
        check_canary(back, n * 2)
    flat, _ = empty_dev(n, "bf16", 1)
    rc.rc_reduce(d, flat[0])
    _sync(rc)
    hf = oracle.bf16_to_f32(want[0]).astype(np.float64)
    ff = oracle.bf16_to_f32(to_host(flat[0], "bf16")).astype(np.float64)
    xa = sum(np.abs(oracle.bf16_to_f32(x).astype(np.float64)) for x in xs)
    assert np.all(np.abs(hf - ff) <= p * 2.0 ** -24 * xa + np.abs(ff) * 2.0 ** -7 + 2.0 ** -133)


# ------------------------------------------------------------ ZeRO-3 layer step
def test_llama_layer_all_gather_bulk_copy(rc, monkeypatch):
    """The bulk-copy fan-out (RC_FANOUT_BULK=1: tiles loaded once into the
    block's shared memory, written to every rank by bulk stores) on the
    Llama-2-7B layer's all-gather, compared in full."""
    monkeypatch.setenv("RC_FANOUT_BULK", "1")
    p = 8
    N = rc_inputs.LLAMA2_7B_LAYER_ELEMS
    shards = rc_inputs.draw(rc_inputs.config("llama_layer_param_shards_bf16"))
    d, _ = to_dev(shards, "bf16")
    full, back = empty_dev(N, "bf16", p, pad_bytes=16)
    rc.rc_all_gather(d, full)
    _sync(rc)
    want = torch.from_numpy(np.concatenate(shards).view(np.int16)).cuda()
    for r in range(p):
        assert torch.equal(full[r].view(torch.int16), want), f"bulk all_gather rank {r}"
    check_canary(back, N * 2, fill=0x5A)
    del full, d, want
    torch.cuda.empty_cache()


def test_llama_layer_zero3_collectives(rc):
    """Llama-2-7B decoder layer (202,375,168 elements), 8 ranks: all_gather of
    bf16 parameter shards, then reduce_scatter of fp32 gradients ~N(0, 1e-3)
    with scale 1/8 to bf16; both compared in full (every element of every
    rank) with the oracle."""
    p = 8
    N = rc_inputs.LLAMA2_7B_LAYER_ELEMS
    m = N // p
    shards = rc_inputs.draw(rc_inputs.config("llama_layer_param_shards_bf16"))
    d, _ = to_dev(shards, "bf16")
    full, _ = empty_dev(N, "bf16", p, pad_bytes=16)
    rc.rc_all_gather(d, full)
    _sync(rc)
    want = np.concatenate(shards)
    for r in range(p):
        assert_bits(to_host(full[r], "bf16"), want, f"llama layer all_gather r{r}")
    del full, d, want
    torch.cuda.empty_cache()

    grads = rc_inputs.draw(rc_inputs.config("llama_layer_grads_f32"))
    g, _ = to_dev(grads, "f32")
    y, back = empty_dev(m, "bf16", p)
    rc.rc_reduce_scatter(g, y, in_dtype="f32", out_dtype="bf16", scale=1.0 / p)
    _sync(rc)
    ref = oracle.reduce_scatter(grads, "f32", "bf16", "sum", 1.0 / p)
    for r in range(p):
        assert_bits(to_host(y[r], "bf16"), ref[r], f"llama layer reduce_scatter shard {r}")
    check_canary(back, m * 2)


# ------------------------------------------------------------ edge cases
@pytest.mark.parametrize("dt", DTS)
def test_misaligned_buffers(rc, dt):
    """Buffers that start off a 16-byte boundary take the scalar path and
    give the same bits."""
    p, n = 4, 4 * 1000
    xs = _data(p, n, dt, seed=9)
    off = 2 if dt == "bf16" else 4
    d, _ = to_dev(xs, dt, offset_bytes=off)
    want = oracle.all_reduce(xs, dt)
    y, back = empty_dev(n, dt, p, offset_bytes=off)
    rc.rc_all_reduce(d, y)
    rs, _ = empty_dev(n // p, dt, p, offset_bytes=off)
    rc.rc_reduce_scatter(d, rs)
    ag, _ = empty_dev(n, dt, p, offset_bytes=off)
    rc.rc_all_gather(rs, ag)
    ring, _ = empty_dev(n, dt, p, offset_bytes=off)
    rc.rc_ring_all_reduce(d, ring)
    hier, _ = empty_dev(n, dt, p, offset_bytes=off)
    rc.rc_hier_all_reduce(d, hier, 2)
    _sync(rc)
    want_h = oracle.hier_all_reduce(xs, 2, dt)
    for r in range(p):
        assert_bits(to_host(y[r], dt), want[r], "misaligned all_reduce")
        assert_bits(to_host(ag[r], dt), want[r], "misaligned rs+ag")
        assert_bits(to_host(ring[r], dt), want[r], "misaligned ring")
        assert_bits(to_host(hier[r], dt), want_h[r], "misaligned hier")
    check_canary(back, off + n * ESZ[dt])


@pytest.mark.parametrize("dt", ["f32", "bf16"])
def test_special_values(rc, dt):
    p, n = 8, 8 * 512
    xs = rc_inputs.special_values(p, n, seed=3, dt=dt)
    d, _ = to_dev(xs, dt)
    for op in OPS:
        want = oracle.all_reduce(xs, dt, op)
        y, _ = empty_dev(n, dt, p)
        rc.rc_all_reduce(d, y, op=op)
        yr, _ = empty_dev(n, dt, p)
        rc.rc_ring_all_reduce(d, yr, op=op)
        _sync(rc)
        for r in range(p):
            assert_bits(to_host(y[r], dt), want[r], f"special {dt} {op}")
            assert_bits(to_host(yr[r], dt), want[r], f"special ring {dt} {op}")


def test_special_int32_wraps(rc):
    p, n = 4, 4 * 256
    xs = rc_inputs.special_values(p, n, seed=4, dt="i32")
    d, _ = to_dev(xs, "i32")
    for op in OPS:
        want = oracle.all_reduce(xs, "i32", op)
        y, _ = empty_dev(n, "i32", p)
        rc.rc_all_reduce(d, y, op=op)
        _sync(rc)
        for r in range(p):
            assert_bits(to_host(y[r], "i32"), want[r], f"int32 {op}")


def test_in_place_variants(rc):
    p, n = 4, 4 * 2048
    xs = rc_inputs.uniform(p, n, seed=21)
    want = oracle.all_reduce(xs)
    d, _ = to_dev(xs, "f32")
    rc.rc_all_reduce(d, d)                                   # all-reduce in place
    _sync(rc)
    for r in range(p):
        assert_bits(to_host(d[r], "f32"), want[r], "in-place all_reduce")
    # reduce_scatter whose output is the rank's own slice of its input
    d2, _ = to_dev(xs, "f32")
    m = n // p
    outs = [d2[r][r * m:(r + 1) * m] for r in range(p)]
    rc.rc_reduce_scatter(d2, outs)
    _sync(rc)
    for r in range(p):
        assert_bits(to_host(outs[r], "f32"), want[r][r * m:(r + 1) * m], "in-place reduce_scatter")
    # all_gather whose input is the rank's own slot of its output
    full, _ = to_dev([np.zeros(n, np.float32) for _ in range(p)], "f32")
    for r in range(p):
        full[r][r * m:(r + 1) * m].copy_(torch.from_numpy(want[0][r * m:(r + 1) * m]).cuda())
    rc.rc_all_gather([full[r][r * m:(r + 1) * m] for r in range(p)], full)
    # reduce into the root's own input, broadcast from a root that is in place
    d3, _ = to_dev(xs, "f32")
    rc.rc_reduce(d3, d3[1], root=1)
    rc.rc_broadcast(d3[1], d3, root=1)
    # hierarchical in place
    d4, _ = to_dev(xs, "f32")
    rc.rc_hier_all_reduce(d4, d4, 2, variant="staged")
    _sync(rc)
    want_h = oracle.hier_all_reduce(xs, 2)
    for r in range(p):
        assert_bits(to_host(full[r], "f32"), want[0], "in-place all_gather")
        assert_bits(to_host(d3[r], "f32"), want[0], "in-place reduce+broadcast")
        assert_bits(to_host(d4[r], "f32"), want_h[r], "in-place hier staged")


def test_rejects_bad_buffers_without_launch(rc):
    from cuda.bindings import runtime as cudart
    p, n = 4, 1 << 20                 # 4 MiB per rank
    xs = rc_inputs.uniform(p, n, seed=1)
    d, _ = to_dev(xs, "f32")
    y, _ = empty_dev(n, "f32", p)
    err, base = cudart.cudaMalloc(4 << 20)
    assert err == cudart.cudaError_t.cudaSuccess
    try:
        short = int(base) + (2 << 20)  # only 2 MiB left in its allocation
        # the pure check must reject it before anything could be launched
        with pytest.raises(rc.RankCollError):
            rc.rc_check_buffer(short, n * 4)
        rc.rc_check_buffer(int(base), n * 4)          # the full allocation is fine
        before = rc.rc_launch_count()
        with pytest.raises(rc.RankCollError):         # output runs past its allocation
            rc.rc_all_reduce(d, [y[0], y[1], y[2], short], n=n)
        with pytest.raises(rc.RankCollError):         # outputs overlap
            rc.rc_all_reduce(d, [y[0], y[0], y[2], y[3]])
        with pytest.raises(rc.RankCollError):         # output overlaps another rank's input
            rc.rc_all_reduce(d, [y[0], d[0], y[2], y[3]])
        host = [np.zeros(n, np.float32) for _ in range(p)]
        with pytest.raises(rc.RankCollError):         # host memory
            rc.rc_all_reduce([h.ctypes.data for h in host], y, n=n, dtype="f32")
        _sync(rc)
        assert rc.rc_launch_count() == before
    finally:
        torch.cuda.synchronize()
        cudart.cudaFree(base)


def test_side_stream_and_launch_count(rc):
    p, n = 8, 8 * 8192
    xs = rc_inputs.uniform(p, n, seed=2)
    want = oracle.all_reduce(xs)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        d, _ = to_dev(xs, "f32")
        y, _ = empty_dev(n, "f32", p)
        before = rc.rc_launch_count()
        rc.rc_all_reduce(d, y)
        assert rc.rc_launch_count() == before + 1
    rc.rc_stream_status(s)
    for r in range(p):
        assert_bits(to_host(y[r], "f32"), want[r], "side stream")


def test_bf16_ring_workspace_across_streams(rc, monkeypatch):
    """The chain kernel's bf16 literal ring keeps fp32 partials in the library
    workspace; calls on two streams in a row see correct results (the second
    stream waits for the first user's work before reusing it)."""
    monkeypatch.setenv("RC_RING_KERNEL", "1")
    p, n = 8, 8 * 4096
    xs = rc_inputs.normal(p, n, seed=6, sigma=1.0, dt="bf16")
    want = oracle.ring_all_reduce(xs, "bf16")
    d, _ = to_dev(xs, "bf16")
    outs = []
    for s in (torch.cuda.Stream(), torch.cuda.Stream()):
        with torch.cuda.stream(s):
            y, _ = empty_dev(n, "bf16", p)
            rc.rc_ring_all_reduce(d, y)
            outs.append((s, y))
    for s, y in outs:
        rc.rc_stream_status(s)
        for r in range(p):
            assert_bits(to_host(y[r], "bf16"), want[r], "bf16 ring two streams")


def test_bounded_wait_reports_timeout_and_context_survives(rc):
    """A device wait that runs out returns an error status to the host; the
    context stays usable and the next collective is still correct."""
    rc.rc_stream_status()                       # clear anything earlier
    rc.rc_probe_bounded_wait(20_000_000)        # 20 ms, nothing will arrive
    with pytest.raises(rc.RankCollError) as e:
        rc.rc_stream_status()
    assert e.value.status == 4
    rc.rc_stream_status()                       # the flag was cleared
    p, n = 4, 4096
    xs = rc_inputs.uniform(p, n, seed=8)
    d, _ = to_dev(xs, "f32")
    y, _ = empty_dev(n, "f32", p)
    rc.rc_all_reduce(d, y)
    _sync(rc)
    want = oracle.all_reduce(xs)
    for r in range(p):
        assert_bits(to_host(y[r], "f32"), want[r], "after timeout")


@pytest.mark.parametrize("dt", DTS)
def test_register_path_matches_oracle(rc, dt, monkeypatch):
    """The register-only fold (used when the bulk-copy path is not eligible)
    gives the same bits as the oracle; forced here on aligned data."""
    monkeypatch.setenv("RC_NO_TMA_FOLD", "1")
    p, n = 8, 8 * 4096 + 8 * 24
    xs = _data(p, n, dt, seed=31)
    d, _ = to_dev(xs, dt)
    for op in OPS:
        y, _ = empty_dev(n, dt, p)
        rc.rc_all_reduce(d, y, op=op)
        rs, _ = empty_dev(n // p, dt, p)
        rc.rc_reduce_scatter(d, rs, op=op)
        h, _ = empty_dev(n, dt, p)
        rc.rc_hier_all_reduce(d, h, 4, op=op)
        _sync(rc)
        want = oracle.all_reduce(xs, dt, op)
        want_h = oracle.hier_all_reduce(xs, 4, dt, op)
        for r in range(p):
            assert_bits(to_host(y[r], dt), want[r], f"register all_reduce {dt} {op}")
            assert_bits(to_host(h[r], dt), want_h[r], f"register hier {dt} {op}")
        assert_bits(np.concatenate([to_host(t, dt) for t in rs]), want[0], f"register rs {dt} {op}")


@pytest.mark.parametrize("tile", ["4096", "16384", "register"])
def test_fanout_tile_sizes(rc, tile, monkeypatch):
    """The fan-out gives the same bytes with the bulk-copy kernel at any tile
    size and with the register kernel (ragged last tile)."""
    if tile != "register":
        monkeypatch.setenv("RC_FANOUT_BULK", "1")
        monkeypatch.setenv("RC_FANOUT_TILE", tile)
    p, m = 8, 12345 * 8
    shards = rc_inputs.uniform(p, m, seed=12, dt="bf16")
    d, _ = to_dev(shards, "bf16")
    y, back = empty_dev(p * m, "bf16", p)
    rc.rc_all_gather(d, y)
    b, back_b = empty_dev(m, "bf16", p)
    rc.rc_broadcast(d[3], b, root=3)
    _sync(rc)
    for r in range(p):
        assert_bits(to_host(y[r], "bf16"), np.concatenate(shards), "all_gather tile")
        assert_bits(to_host(b[r], "bf16"), shards[3], "broadcast tile")
    check_canary(back, p * m * 2)
    check_canary(back_b, m * 2)


@pytest.mark.parametrize("nbytes", [16, 1000, 1 << 20, (1 << 24) + 48])
def test_copy_kernel(rc, nbytes):
    a = torch.randint(0, 256, (nbytes,), dtype=torch.uint8, device="cuda")
    b = torch.zeros(nbytes + 64, dtype=torch.uint8, device="cuda")
    rc.rc_copy(a, b, nbytes)
    _sync(rc)
    assert torch.equal(a, b[:nbytes])
    assert int(b[nbytes:].sum()) == 0


@pytest.mark.parametrize("dt", DTS)
@pytest.mark.parametrize("p,G", [(8, 4), (8, 2), (16, 4), (4, 2)])
def test_staged_fold_paths_match_oracle(rc, dt, p, G, monkeypatch):
    """The shared-memory-staged fold, the alternative path of the all-reduce
    (RC_AR_FOLD=1) and of the fused hierarchical all-reduce (RC_HIER_FOLD=1),
    gives the oracle's bits too (ragged tail included)."""
    monkeypatch.setenv("RC_AR_FOLD", "1")
    monkeypatch.setenv("RC_HIER_FOLD", "1")
    n = p * 4096 + p * 24 + (8 if dt != "bf16" else 16)
    xs = _data(p, n, dt, seed=41 + p + G)
    d, _ = to_dev(xs, dt)
    for op in OPS:
        y, back = empty_dev(n, dt, p)
        rc.rc_all_reduce(d, y, op=op)
        h, _ = empty_dev(n, dt, p)
        rc.rc_hier_all_reduce(d, h, G, op=op)
        _sync(rc)
        want = oracle.all_reduce(xs, dt, op)
        want_h = oracle.hier_all_reduce(xs, G, dt, op)
        for r in (0, p - 1):
            assert_bits(to_host(y[r], dt), want[r], f"staged fold all_reduce {dt} {op}")
            assert_bits(to_host(h[r], dt), want_h[r], f"staged fold hier {dt} {op} G={G}")
        check_canary(back, n * (2 if dt == "bf16" else 4))


def test_workspace_kept_for_a_captured_graph(rc):
    """A graph that captured a call using the library workspace (the staged
    hierarchical all-reduce) still gives the oracle's bits when it is replayed
    after the workspace has grown: growth retires the captured block instead
    of freeing it, and rc_finalize frees it."""
    p, G, n = 8, 4, 8 * 4096
    xs = rc_inputs.normal(p, n, seed=52, sigma=1.0, dt="bf16")
    want = oracle.hier_all_reduce(xs, G, "bf16")
    d, _ = to_dev(xs, "bf16")
    y, _ = empty_dev(n, "bf16", p)
    torch.cuda.synchronize()
    rc.rc_finalize()
    need = (p // G + 1) * n * 4
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        rc.rc_reserve_workspace(need)
        s.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            rc.rc_hier_all_reduce(d, y, G, variant="staged")
        rc.rc_reserve_workspace(4 * need)                     # grows: the captured block is retired
        live, retired = rc.rc_workspace_bytes()
        assert live >= 4 * need and retired >= need
        other = rc_inputs.normal(p, n, seed=53, sigma=1.0, dt="bf16")
        d2, _ = to_dev(other, "bf16")
        y2, _ = empty_dev(n, "bf16", p)
        rc.rc_hier_all_reduce(d2, y2, G, variant="staged")   # uses the new block
        g.replay()
    s.synchronize()
    rc.rc_stream_status(s)
    for r in range(p):
        assert_bits(to_host(y[r], "bf16"), want[r], f"replayed graph after growth r{r}")
    want2 = oracle.hier_all_reduce(other, G, "bf16")
    for r in range(p):
        assert_bits(to_host(y2[r], "bf16"), want2[r], f"call on the grown workspace r{r}")
    del g
    torch.cuda.synchronize()
    rc.rc_finalize()
    assert rc.rc_workspace_bytes() == (0, 0)


def test_ordinary_launches_match_oracle():
    """With programmatic dependent launch turned off (RC_PDL=0, read once per
    process, so in a child process) every collective of the bench step still
    gives the oracle's bits, launched back to back on one stream."""
    import os
    import subprocess
    import sys
    code = r"""
import numpy as np, torch, sys
sys.path.insert(0, %r)
sys.path.insert(0, %r)
import collective_rc_all_b200 as rc, oracle, rc_inputs
from util import to_dev, empty_dev, to_host, assert_bits
p, n = 8, 8 * 4096
xs = rc_inputs.normal(p, n, seed=61, sigma=1.0)
d, _ = to_dev(xs, "f32")
y, _ = empty_dev(n, "f32", p); rs, _ = empty_dev(n // p, "bf16", p); ag, _ = empty_dev(n, "bf16", p)
ring, _ = empty_dev(n, "f32", p); h, _ = empty_dev(n, "f32", p)
rc.rc_all_reduce(d, y); rc.rc_reduce_scatter(d, rs, out_dtype="bf16", scale=1.0 / p)
rc.rc_all_gather(rs, ag); rc.rc_ring_all_reduce(d, ring); rc.rc_hier_all_reduce(d, h, 4)
torch.cuda.synchronize(); rc.rc_stream_status()
want = oracle.all_reduce(xs); want_rs = oracle.reduce_scatter(xs, "f32", "bf16", "sum", 1.0 / p)
want_h = oracle.hier_all_reduce(xs, 4)
for r in range(p):
    assert_bits(to_host(y[r], "f32"), want[r], "all_reduce")
    assert_bits(to_host(ring[r], "f32"), want[r], "ring")
    assert_bits(to_host(h[r], "f32"), want_h[r], "hier")
    assert_bits(to_host(rs[r], "bf16"), want_rs[r], "reduce_scatter")
    assert_bits(to_host(ag[r], "bf16"), np.concatenate(want_rs), "all_gather")
print("ok")
""" % (os.path.dirname(os.path.dirname(os.path.abspath(__file__))), os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, RC_PDL="0")
    r = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0 and r.stdout.strip().endswith("ok"), r.stdout[-2000:] + r.stderr[-2000:]


@pytest.mark.parametrize("p,n", [(12, 760), (16, 120), (3, 840)])
def test_link_ring_in_place_ragged(rc, p, n):
    """The link kernel in place with ragged chunks (a short or an empty last
    chunk): every input is read before its thread's first store."""
    for dt in DTS:
        if dt == "bf16" and (-(-n // p)) % 8:
            continue   # the chunk length must keep 16-byte vectors for the link kernel
        xs = _data(p, n, dt, seed=p + n)
        want = oracle.ring_all_reduce(xs, dt)
        d, _ = to_dev(xs, dt)
        rc.rc_ring_all_reduce(d, d)
        _sync(rc)
        for r in range(p):
            assert_bits(to_host(d[r], dt), want[r], f"link ring in place p={p} n={n} {dt} r{r}")


def test_link_ring_captures_without_workspace(rc):
    """The default bf16 literal ring keeps its partials on chip: it can be
    captured into a CUDA graph with no library workspace reserved, allocates
    none, and replays to the oracle's bits."""
    p, n = 8, 8 * 4096
    xs = rc_inputs.normal(p, n, seed=71, sigma=1.0, dt="bf16")
    want = oracle.ring_all_reduce(xs, "bf16")
    d, _ = to_dev(xs, "bf16")
    y, _ = empty_dev(n, "bf16", p)
    torch.cuda.synchronize()
    rc.rc_finalize()
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            rc.rc_ring_all_reduce(d, y)
        g.replay()
    s.synchronize()
    rc.rc_stream_status(s)
    assert rc.rc_workspace_bytes() == (0, 0)
    for r in range(p):
        assert_bits(to_host(y[r], "bf16"), want[r], f"captured bf16 ring r{r}")
    del g
