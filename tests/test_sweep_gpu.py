"""The sweep workload on the GPU: p in {2, 4, 8, 16}, per-rank sizes from
1 KiB to 1 GiB in powers of 4, fp32 / bf16 / int32 (floats uniform[-1, 1),
ints uniform[-2^20, 2^20)), ops sum and max, all_reduce / reduce_scatter /
all_gather.

* up to 16 MiB per rank: seeded random data, every output element compared
  bit for bit with the CPU oracle;
* 64 MiB .. 1 GiB per rank: integer-valued inputs x_r[i] = (i mod 1021) + r,
  for which sum = p*(i mod 1021) + p(p-1)/2 and max = (i mod 1021) + p - 1
  are exact in every dtype and every fold order; every element is checked
  against that closed form (on the device, with torch);
* one 256 MiB-per-rank random case checked against the oracle at sampled
  indices (chunk boundaries included).
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
        assert_bits(to_host(y[0], dt), want[0], f"AR p={p} {nbytes}B {dt} {op} rank 0")
        assert_bits(to_host(y[p - 1], dt), want[p - 1], f"AR p={p} {nbytes}B {dt} {op} rank p-1")
        assert_bits(np.concatenate([to_host(t, dt) for t in rs]), want[0],
                    f"RS p={p} {nbytes}B {dt} {op}")
    # all_gather of rank-specific shards
    shards = [x[: n // p] for x in xs]
    ag, _ = empty_dev(n, dt, p, pad_bytes=16)
    sd, _ = to_dev(shards, dt)
    rc.rc_all_gather(sd, ag)
    torch.cuda.synchronize()
    want_ag = np.concatenate(shards)
    for r in (0, p - 1):
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
        for r in (0, p - 1):
            assert torch.equal(y[r], want), f"AR closed form p={p} {nbytes}B {dt} {op}"
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
        for r in (0, p - 1):
            assert torch.equal(y[r], want), f"AG closed form p={p} {nbytes}B {dt}"
        del y, rs, want
    del xs, base
    torch.cuda.empty_cache()


def test_sweep_256mib_random_sampled(rc):
    p, dt = 8, "f32"
    n = (1 << 28) // 4
    xs = rc_inputs.sweep_data(p, n, seed=777, dt=dt)
    d, _ = to_dev(xs, dt)
    y = [torch.empty(n, dtype=torch.float32, device="cuda") for _ in range(p)]
    rc.rc_all_reduce(d, y)
    rs = [torch.empty(n // p, dtype=torch.float32, device="cuda") for _ in range(p)]
    rc.rc_reduce_scatter(d, rs, op="max")
    torch.cuda.synchronize()
    rc.rc_stream_status()
    m = n // p
    rng = np.random.default_rng(5)
    idx = np.unique(np.concatenate([rng.integers(0, n, 100_000),
                                    np.array([c * m + o for c in range(p) for o in (0, 1, 3, 4, m - 5, m - 1)])]))
    ti = torch.from_numpy(idx.astype(np.int64)).cuda()
    got = y[3].index_select(0, ti).cpu().numpy()
    assert_bits(got, oracle.reduce_at(xs, idx.astype(np.uint64), dt, dt, "sum"), "AR 256MiB sampled")
    full = torch.cat(rs).index_select(0, ti).cpu().numpy()
    assert_bits(full, oracle.reduce_at(xs, idx.astype(np.uint64), dt, dt, "max"), "RS max 256MiB sampled")
