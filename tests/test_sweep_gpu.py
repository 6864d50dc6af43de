"""The sweep workload on the GPU: p in {2, 4, 8, 16}, per-rank sizes from
1 KiB to 1 GiB in powers of 4, fp32 / bf16 / int32 (floats uniform[-1, 1),
ints uniform[-2^20, 2^20)), ops sum and max, all_reduce / reduce_scatter /
all_gather.

* up to 16 MiB per rank: seeded random data drawn on the host, every output
  element of every rank compared bit for bit with the CPU oracle;
* 64 MiB .. 1 GiB per rank, all 12 (p, dtype) pairs: seeded random data of
  the same distributions drawn on the device (fold-order sensitive, so the
  ring order of "LLM Parallelism 基础", section "Ring AllReduce", decides the
  bits), sum and max, every rank of the all-reduce and every shard of the
  reduce-scatter compared with the oracle at 100,000 random indices plus
  every chunk boundary +-one vector and the ragged end; the all-gather is a
  copy and is compared in full;
* the largest sizes also once with integer-valued inputs x_r[i] = (i mod
  1021) + r, exact in every dtype and fold order, every element checked
  against that closed form (on the device, with torch).
"""
import numpy as np
import pytest
import torch

import oracle
import rc_inputs
from util import assert_bits, empty_dev, to_dev, to_host

pytestmark = pytest.mark.gpu

ESZ = {"f32": 4, "bf16": 2, "i32": 4}
TORCH = {"f32": torch.float32, "bf16": torch.bfloat16, "i32": torch.int32}
SMALL = [1 << 10, 1 << 12, 1 << 14, 1 << 16, 1 << 18, 1 << 20, 1 << 22, 1 << 24]
LARGE = [1 << 26, 1 << 28, 1 << 30]


@pytest.fixture(scope="module")
def rc():
    import collective_rc_all_b200 as m
    assert torch.cuda.is_available()
    return m


@pytest.mark.parametrize("p", [2, 4, 8, 16])
@pytest.mark.parametrize("nbytes", SMALL)
@pytest.mark.parametrize("dt", ["f32", "bf16", "i32"])
def test_sweep_random_vs_oracle(rc, p, nbytes, dt):
    n = nbytes // ESZ[dt]
    xs = rc_inputs.sweep_data(p, n, seed=100 + p * 97 + nbytes % 9973, dt=dt)
    d, _ = to_dev(xs, dt)
    for op in ("sum", "max"):
        want = oracle.all_reduce(xs, dt, op)
        y, _ = empty_dev(n, dt, p, pad_bytes=16)
        rc.rc_all_reduce(d, y, op=op)
        rs, _ = empty_dev(n // p, dt, p, pad_bytes=16)
        rc.rc_reduce_scatter(d, rs, op=op)
        torch.cuda.synchronize()
        rc.rc_stream_status()
        for r in range(p):
            assert_bits(to_host(y[r], dt), want[r], f"AR p={p} {nbytes}B {dt} {op} rank {r}")
        assert_bits(np.concatenate([to_host(t, dt) for t in rs]), want[0],
                    f"RS p={p} {nbytes}B {dt} {op}")
    # all_gather of rank-specific shards
    shards = [x[: n // p] for x in xs]
    ag, _ = empty_dev(n, dt, p, pad_bytes=16)
    sd, _ = to_dev(shards, dt)
    rc.rc_all_gather(sd, ag)
    torch.cuda.synchronize()
    want_ag = np.concatenate(shards)
    for r in range(p):
        assert_bits(to_host(ag[r], dt), want_ag, f"AG p={p} {nbytes}B {dt} rank {r}")


def _closed_form_inputs(p, n, dt, dev="cuda"):
    base = torch.remainder(torch.arange(n, device=dev, dtype=torch.int64), 1021)
    return base, [(base + r).to(TORCH[dt]) for r in range(p)]


@pytest.mark.parametrize("p,nbytes,dt", [
    (2, LARGE[0], "bf16"), (4, LARGE[0], "i32"), (8, LARGE[1], "f32"), (16, LARGE[1], "bf16"),
    (16, LARGE[2], "f32"), (4, LARGE[2], "i32")])
def test_sweep_large_closed_form(rc, p, nbytes, dt):
    """Every element of the largest sweep sizes against the exact closed form
    (values stay exact in bf16: p*(1020) + p(p-1)/2 < 2^15 and bf16 holds the
    integers up to 256 exactly only, so bf16 cases use max and a small sum)."""
    n = nbytes // ESZ[dt]
    base, xs = _closed_form_inputs(p, n, dt)
    torch.cuda.synchronize()
    ops = ("max",) if dt == "bf16" else ("sum", "max")
    for op in ops:
        want = (base * p + p * (p - 1) // 2) if op == "sum" else (base + p - 1)
        want = want.to(TORCH[dt])
        y = [torch.empty(n, dtype=TORCH[dt], device="cuda") for _ in range(p)]
        rc.rc_all_reduce(xs, y, op=op)
        torch.cuda.synchronize()
        rc.rc_stream_status()
        for r in range(p):
            assert torch.equal(y[r], want), f"AR closed form p={p} {nbytes}B {dt} {op} r{r}"
        del y
        rs = [torch.empty(n // p, dtype=TORCH[dt], device="cuda") for _ in range(p)]
        rc.rc_reduce_scatter(xs, rs, op=op)
        torch.cuda.synchronize()
        for r in range(p):
            assert torch.equal(rs[r], want[r * (n // p):(r + 1) * (n // p)]), f"RS closed form r{r}"
        # all_gather the reduce-scatter shards back to the full vector
        y = [torch.empty(n, dtype=TORCH[dt], device="cuda") for _ in range(p)]
        rc.rc_all_gather(rs, y)
        torch.cuda.synchronize()
        for r in range(p):
            assert torch.equal(y[r], want), f"AG closed form p={p} {nbytes}B {dt} r{r}"
        del y, rs, want
    del xs, base
    torch.cuda.empty_cache()


def _sample_indices(n, p, vec, seed, k=100_000):
    """k random indices plus every chunk boundary +-vec (and +-1) and the ragged end."""
    C = -(-n // p)
    rng = np.random.default_rng(seed)
    edge = []
    for c in range(p + 1):
        for d in (-vec, -1, 0, 1, vec):
            if 0 <= c * C + d < n:
                edge.append(c * C + d)
    edge += [0, 1, n - vec, n - 2, n - 1]
    return np.unique(np.concatenate([rng.integers(0, n, k), np.array(edge)])).astype(np.int64)


def _sparse_host_inputs(xs, dt, idx):
    """Host arrays of the full length n that hold the device inputs' values at
    idx and zeros elsewhere (np.zeros maps untouched pages, so an n-element
    array costs only the pages idx touches).  reduce_at reads x_r[idx] and
    nothing else, so it sees exactly the inputs the GPU saw."""
    ti = torch.from_numpy(idx).cuda()
    out = []
    for x in xs:
        h = np.zeros(x.numel(), dtype={"f32": np.float32, "bf16": np.uint16, "i32": np.int32}[dt])
        h[idx] = to_host(x.index_select(0, ti), dt)
        out.append(h)
    return out


LARGE_POINTS = [(p, nbytes, dt) for nbytes in LARGE for p in (2, 4, 8, 16) for dt in ("f32", "bf16", "i32")]


@pytest.mark.parametrize("p,nbytes,dt", LARGE_POINTS)
def test_sweep_large_random_sampled(rc, p, nbytes, dt):
    n = nbytes // ESZ[dt]
    m = n // p
    vec = 16 // ESZ[dt]
    seed = 100 + p * 97 + nbytes % 9973
    xs = rc_inputs.sweep_data_device(p, n, seed=seed, dt=dt)
    idx = _sample_indices(n, p, vec, seed)
    hx = _sparse_host_inputs(xs, dt, idx)
    ti = torch.from_numpy(idx).cuda()
    for op in ("sum", "max"):
        want = oracle.reduce_at(hx, idx.astype(np.uint64), dt, dt, op)
        y = [torch.empty(n, dtype=TORCH[dt], device="cuda") for _ in range(p)]
        rc.rc_all_reduce(xs, y, op=op)
        torch.cuda.synchronize()
        rc.rc_stream_status()
        for r in range(p):
            assert_bits(to_host(y[r].index_select(0, ti), dt), want,
                        f"AR p={p} {nbytes}B {dt} {op} rank {r} (sampled)")
        del y
        rs = [torch.empty(m, dtype=TORCH[dt], device="cuda") for _ in range(p)]
        rc.rc_reduce_scatter(xs, rs, op=op)
        torch.cuda.synchronize()
        rc.rc_stream_status()
        got = to_host(torch.cat(rs).index_select(0, ti), dt)
        assert_bits(got, want, f"RS p={p} {nbytes}B {dt} {op} (sampled, every shard)")
        del rs
    # all_gather of rank-specific shards: a copy, compared in full on the device
    shards = [x[:m] for x in xs]
    ag = [torch.empty(n, dtype=TORCH[dt], device="cuda") for _ in range(p)]
    rc.rc_all_gather(shards, ag)
    torch.cuda.synchronize()
    rc.rc_stream_status()
    want_ag = torch.cat(shards)
    for r in range(p):
        assert torch.equal(ag[r].view(torch.int16 if dt == "bf16" else TORCH[dt]),
                           want_ag.view(torch.int16 if dt == "bf16" else TORCH[dt])), \
            f"AG p={p} {nbytes}B {dt} rank {r}"
    del ag, want_ag, shards, xs
    torch.cuda.empty_cache()
