"""bench.py on the GPU, short runs: the JSON line keeps the keys the driver
reads (metric, value, unit, n_gpus, steps, warmup, ms_per_step, roofline with
its peak and frac, cpu_baseline, e2e with its byte counts, gpu_launches,
clocks), and the ZeRO-1 and all-to-all modes print their lines."""
import contextlib
import io
import json

import pytest
import torch

pytestmark = pytest.mark.gpu


def _run(argv):
    import bench
    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        rc = bench.main(argv)
    assert rc == 0
    lines = [l for l in buf.getvalue().splitlines() if l.startswith("{")]
    assert lines, buf.getvalue()[-2000:]
    return json.loads(lines[-1])


def test_step_line_has_the_driver_keys():
    assert torch.cuda.is_available()
    d = _run(["--steps", "3", "--warmup", "3", "--cpu-seconds", "1", "--no-copy-peak"])
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
              "scaling", "vs_baseline", "dtype", "data", "config", "roofline", "cpu_baseline", "e2e",
              "gpu_launches", "clocks"):
        assert k in d, k
    assert d["n_gpus"] == 1 and d["steps"] == 3 and d["warmup"] >= 3
    assert d["value"] > 0 and d["ms_per_step"] > 0
    r = d["roofline"]
    assert r["bound"] == "hbm" and r["peak"] > 0 and 0 < r["frac"] < 2 and r["unit"] == "GB/s"
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] == 1
    e = d["e2e"]
    assert e["value"] > 0 and e["h2d_bytes_per_step"] > 0 and e["d2h_bytes_per_step"] > 0
    assert d["gpu_launches"] >= 7 * 3
    assert set(d["per_op"]) == {"all_reduce", "reduce_scatter", "all_gather", "reduce", "broadcast",
                                "ring_all_reduce", "hier_all_reduce"}


def test_zero1_and_a2a_modes():
    z = _run(["--zero1", "--zero1-elems", str(8 * 4096 * 16), "--steps", "2", "--warmup", "3"])
    assert set(z["variants"]) == {"fused_bf16", "fused_f32", "unfused_f32", "owner_f32"}
    assert z["variants"]["fused_bf16"]["launches_per_step"] == 1
    a = _run(["--a2a", "--steps", "2", "--warmup", "3"])
    assert a["variants"]["balanced"]["cross_rank_bytes_per_phase"] == 8 * 4096 * 2 * 4096 * 2 * 7 // 8
