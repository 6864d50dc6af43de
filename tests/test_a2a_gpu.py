"""GPU parity of the all-to-all entry points (rc_all_to_all, rc_all_to_all_v)
against the CPU oracle, bit for bit: equal splits for every dtype and p, split
counts with empty and skewed blocks, unaligned blocks and buffers, dispatch
followed by combine, the MoE-sized exchange in full, and the host-side
rejection of overlapping buffers."""
import numpy as np
import pytest
import torch

import oracle
import rc_inputs
from util import assert_bits, check_canary, empty_dev, to_dev, to_host

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def rc():
    import collective_rc_all_b200 as m
    assert torch.cuda.is_available()
    return m


def _sync(rc):
    torch.cuda.synchronize()
    rc.rc_stream_status()


def _data(p, n, dt, seed):
    return rc_inputs.sweep_data(p, n, seed, dt)


@pytest.mark.parametrize("p", [2, 4, 8, 16])
@pytest.mark.parametrize("dt", ["f32", "bf16", "i32"])
@pytest.mark.parametrize("m", [1, 1001, 4096 + 8])
def test_equal_splits(rc, p, dt, m):
    n = p * m
    xs = _data(p, n, dt, seed=p * 7 + m)
    d, _ = to_dev(xs, dt)
    y, back = empty_dev(n, dt, p)
    rc.rc_all_to_all(d, y)
    _sync(rc)
    want = oracle.all_to_all(xs)
    esz = 2 if dt == "bf16" else 4
    for q in range(p):
        assert_bits(to_host(y[q], dt), want[q], f"a2a p={p} {dt} m={m} rank {q}")
    check_canary(back, n * esz)


def _counts(p, seed, skew=False, zeros=True, scale=3000):
    r = np.random.default_rng(seed)
    if skew:  # a few hot destinations (popular experts)
        w = 1.0 / np.arange(1, p + 1) ** 1.5
        w = w / w.sum()
        c = np.stack([r.multinomial(scale * p, w[r.permutation(p)]) for _ in range(p)])
    else:
        c = r.integers(0, scale, (p, p))
    if zeros:
        c[r.integers(0, p), :] = 0
        c[:, r.integers(0, p)] = 0
        c[r.integers(0, p), r.integers(0, p)] = 0
    return c.astype(np.int64)


@pytest.mark.parametrize("p,seed,skew", [(2, 1, False), (3, 2, False), (8, 3, False), (8, 4, True),
                                         (16, 5, True), (16, 6, False)])
@pytest.mark.parametrize("dt", ["f32", "bf16"])
def test_split_counts(rc, p, seed, skew, dt):
    counts = _counts(p, seed, skew)
    sends = _data(p, int(counts.sum(axis=1).max()) + 1, dt, seed)
    sends = [x[: int(counts[r].sum())] for r, x in enumerate(sends)]
    want = oracle.all_to_all_v(sends, counts)
    d, _ = to_dev([s if s.size else np.zeros(1, s.dtype) for s in sends], dt)
    esz = 2 if dt == "bf16" else 4
    y, back = [], []
    for q in range(p):
        t, b = empty_dev(max(1, int(counts[:, q].sum())), dt, 1)
        y += t
        back += b
    rc.rc_all_to_all_v(d, y, counts)
    _sync(rc)
    for q in range(p):
        k = int(counts[:, q].sum())
        assert_bits(to_host(y[q], dt)[:k], want[q], f"a2a_v p={p} seed={seed} rank {q}")
        check_canary([back[q]], max(1, k) * esz)


def test_dispatch_then_combine_restores(rc):
    p = 8
    counts = _counts(p, 11, skew=True, zeros=False)
    sends = _data(p, int(counts.sum(axis=1).max()), "bf16", 12)
    sends = [x[: int(counts[r].sum())] for r, x in enumerate(sends)]
    d, _ = to_dev(sends, "bf16")
    mid = [torch.empty(int(counts[:, q].sum()), dtype=torch.bfloat16, device="cuda") for q in range(p)]
    back = [torch.empty(int(counts[r].sum()), dtype=torch.bfloat16, device="cuda") for r in range(p)]
    rc.rc_all_to_all_v(d, mid, counts)
    rc.rc_all_to_all_v(mid, back, counts.T)
    _sync(rc)
    for r in range(p):
        assert_bits(to_host(back[r], "bf16"), sends[r], f"combine(dispatch) rank {r}")


@pytest.mark.parametrize("dt,off", [("f32", 4), ("bf16", 2)])
def test_unaligned_buffers(rc, dt, off):
    p, m = 4, 2048
    xs = _data(p, p * m, dt, 21)
    d, _ = to_dev(xs, dt, offset_bytes=off)
    y, back = empty_dev(p * m, dt, p, offset_bytes=off)
    rc.rc_all_to_all(d, y)
    _sync(rc)
    want = oracle.all_to_all(xs)
    for q in range(p):
        assert_bits(to_host(y[q], dt), want[q], f"a2a unaligned {dt} rank {q}")
    check_canary(back, off + p * m * (2 if dt == "bf16" else 4))


def test_moe_dispatch_balanced_full_size(rc):
    """t = 4096 tokens per rank, top-2, h = 4096, bf16, EP group of 8: 64 MiB
    per rank and phase, 8 MiB per (source, destination) pair."""
    p, t, k, h = 8, 4096, 2, 4096
    n = t * k * h
    g = torch.Generator(device="cpu")
    g.manual_seed(31)
    xs = [torch.randint(0, 1 << 16, (n,), generator=g, dtype=torch.int32).to(torch.int16).numpy().view(np.uint16)
          for _ in range(p)]
    d, _ = to_dev(xs, "bf16")
    y = [torch.empty(n, dtype=torch.bfloat16, device="cuda") for _ in range(p)]
    rc.rc_all_to_all(d, y)
    _sync(rc)
    tr = [0, 0]
    want = oracle.all_to_all(xs, traffic=tr)
    assert tr[1] == p * t * k * h * 2 * (p - 1) // p
    for q in range(p):
        assert_bits(to_host(y[q], "bf16"), want[q], f"MoE dispatch rank {q}")


def test_overlapping_send_and_recv_rejected(rc):
    p, m = 4, 256
    buf = torch.zeros(p * p * m, dtype=torch.float32, device="cuda")
    send = [buf[r * p * m:(r + 1) * p * m] for r in range(p)]
    before = rc.rc_launch_count()
    with pytest.raises(rc.RankCollError):
        rc.rc_all_to_all(send, send)  # in place is not an all-to-all
    other = [torch.empty(p * m, device="cuda") for _ in range(p)]
    with pytest.raises(rc.RankCollError):
        rc.rc_all_to_all(send, [other[0]] * p)  # receivers overlap one another
    assert rc.rc_launch_count() == before


def test_single_rank_is_a_copy(rc):
    xs = _data(1, 1000, "f32", 77)
    d, _ = to_dev(xs, "f32")
    y, back = empty_dev(1000, "f32", 1)
    rc.rc_all_to_all(d, y)
    _sync(rc)
    assert_bits(to_host(y[0], "f32"), xs[0], "a2a p=1")
    check_canary(back, 4000)
