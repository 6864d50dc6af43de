"""GPU parity of the optimizer entry points against the CPU oracle, bit for bit:
rc_adamw_step (AdamW on one array) and rc_zero1_step (the ZeRO-1 step fused
with its reduce-scatter and all-gather), plus the identity of the fused step
with the unfused chain of library calls, and the full-size Llama-2-7B layer
(sampled)."""
import numpy as np
import pytest
import torch

import oracle
import rc_inputs
from util import assert_bits, check_canary, empty_dev, to_dev, to_host

pytestmark = pytest.mark.gpu

HP = rc_inputs.ZERO1_ADAMW


@pytest.fixture(scope="module")
def rc():
    import collective_rc_all_b200 as m
    assert torch.cuda.is_available()
    return m


def _sync(rc):
    torch.cuda.synchronize()
    rc.rc_stream_status()


def _grads(p, n, dt, seed):
    g = rc_inputs.normal(p, n, seed, sigma=1e-3, dt="f32")
    return g if dt == "f32" else [oracle.f32_to_bf16(x) for x in g]


@pytest.mark.parametrize("n,grad_dt,offset,goffset", [(4099, "f32", 0, 0), (4096, "bf16", 0, 0),
                                                      (777, "f32", 4, 4), (1 << 16, "bf16", 4, 2),
                                                      (8, "f32", 0, 0)])
@pytest.mark.parametrize("step", [1, 1000])
def test_adamw_step_matches_oracle(rc, n, grad_dt, offset, goffset, step):
    master, ea, es = rc_inputs.adam_state(1, n, seed=11 + n)
    g = _grads(1, n, grad_dt, seed=12 + n)[0]
    hp = dict(HP, step=step)
    want = oracle.adamw(master[0], ea[0], es[0], g, grad_dt, **hp)
    dev = [to_dev([a], "f32", offset_bytes=offset, pad_bytes=64) for a in (master[0], ea[0], es[0])]
    gd, _ = to_dev([g], grad_dt, offset_bytes=goffset)
    th, mm, vv = (d[0][0] for d in dev)
    rc.rc_adamw_step(th, mm, vv, gd[0], grad_dtype=grad_dt, **hp)
    _sync(rc)
    for got, w, name in zip((th, mm, vv), want, ("theta", "exp_avg", "exp_avg_sq")):
        assert_bits(to_host(got, "f32"), w, f"adamw {name} n={n} {grad_dt} step={step}")
    for d in dev:  # nothing written past the end
        b = d[1][0][offset + n * 4:offset + n * 4 + 64].cpu().numpy()
        assert np.all(b == 0xA5)


def _zero1_case(rc, p, n, grad_dt, param_dt, seed, offset=0, steps=1):
    m = n // p
    grads = _grads(p, n, grad_dt, seed)
    master, ea, es = rc_inputs.adam_state(p, n, seed + 1)
    gd, _ = to_dev(grads, grad_dt, offset_bytes=offset)
    md, _ = to_dev(master, "f32", offset_bytes=offset)
    ad, _ = to_dev(ea, "f32", offset_bytes=offset)
    sd, _ = to_dev(es, "f32", offset_bytes=offset)
    pd, back = empty_dev(n, param_dt, p, offset_bytes=offset)
    ref = (master, ea, es)
    for t in range(1, steps + 1):
        hp = dict(HP, step=t)
        rc.rc_zero1_step(gd, pd, md, ad, sd, grad_dtype=grad_dt, param_dtype=param_dt, **hp)
        params, *ref = oracle.zero1_step(grads, *ref, grad_dt=grad_dt, param_dt=param_dt, **hp)
    _sync(rc)
    esz = 4 if param_dt == "f32" else 2
    for q in range(p):
        assert_bits(to_host(pd[q], param_dt), params[q], f"zero1 params rank {q}")
    for r in range(p):
        for got, w, name in zip((md[r], ad[r], sd[r]), ref, ("master", "exp_avg", "exp_avg_sq")):
            assert_bits(to_host(got, "f32"), w[r], f"zero1 {name} shard {r}")
    check_canary(back, offset + n * esz)


@pytest.mark.parametrize("p", [2, 4, 8, 16])
@pytest.mark.parametrize("grad_dt,param_dt", [("f32", "bf16"), ("f32", "f32"), ("bf16", "bf16"),
                                              ("bf16", "f32")])
def test_zero1_step_matches_oracle(rc, p, grad_dt, param_dt):
    # several tiles per shard and a ragged last tile (m = 3 * 2048 + 40)
    _zero1_case(rc, p, p * (3 * 2048 + 40), grad_dt, param_dt, seed=40 + p)


@pytest.mark.parametrize("p,param_dt", [(8, "bf16"), (3, "bf16"), (8, "f32")])
def test_zero1_odd_vector_count_per_shard(rc, p, param_dt):
    """m = 4 * 1001: an odd number of 16-byte vectors per shard, so every other
    shard starts off a 16-byte boundary of the bf16 parameters and the last
    thread of a shard holds a single vector."""
    _zero1_case(rc, p, p * 4 * 1001, "f32", param_dt, seed=60 + p)


@pytest.mark.parametrize("p,n,offset", [(8, 8 * 1001, 0), (4, 4 * 6, 0), (8, 8 * 512, 4), (3, 3 * 333, 0)])
def test_zero1_element_path(rc, p, n, offset):
    """Shard lengths that are not whole vectors, and buffers off a 16-byte
    boundary (4-byte offset: still aligned to their elements), take the
    element path: same bits."""
    _zero1_case(rc, p, n, "f32", "bf16", seed=70 + n, offset=offset)


def test_zero1_three_steps_carry_state(rc):
    _zero1_case(rc, 8, 8 * 4096, "f32", "bf16", seed=90, steps=3)


def test_zero1_equals_unfused_library_chain(rc):
    """rc_zero1_step == rc_reduce_scatter (fp32, x 1/p) + rc_adamw_step on each
    shard + rc_all_gather, bit for bit, on the GPU."""
    p, n = 8, 8 * 65536
    m = n // p
    grads = _grads(p, n, "f32", 123)
    master, ea, es = rc_inputs.adam_state(p, n, 124)
    gd, _ = to_dev(grads, "f32")
    fused = [to_dev(x, "f32")[0] for x in (master, ea, es)]
    chain = [to_dev(x, "f32")[0] for x in (master, ea, es)]
    pf, _ = empty_dev(n, "bf16", p)
    pc, _ = empty_dev(n, "bf16", p)
    rc.rc_zero1_step(gd, pf, *fused, param_dtype="bf16", **HP)
    gs = [torch.empty(m, dtype=torch.float32, device="cuda") for _ in range(p)]
    rc.rc_reduce_scatter(gd, gs, out_dtype="f32", scale=1.0 / p)
    for r in range(p):
        rc.rc_adamw_step(chain[0][r], chain[1][r], chain[2][r], gs[r], **HP)
    shards = [t.to(torch.bfloat16) for t in chain[0]]  # RNE narrowing by torch, compared below
    rc.rc_all_gather(shards, pc)
    _sync(rc)
    for a, b in zip(fused, chain):
        for r in range(p):
            assert torch.equal(a[r], b[r])
    want_shards = [oracle.f32_to_bf16(to_host(t, "f32")) for t in chain[0]]
    for q in range(p):
        assert_bits(to_host(pf[q], "bf16"), np.concatenate(want_shards), f"fused params rank {q}")
        assert_bits(to_host(pc[q], "bf16"), np.concatenate(want_shards), f"chain params rank {q}")


def test_zero1_llama_layer_full(rc):
    """The full-size step: 8 ranks x 202,375,168 fp32 gradients ~N(0, 1e-3),
    bf16 parameters, fp32 shards of master weights and moments; every element
    of the new state and of every rank's parameters against the oracle's
    composition (reduce_scatter x 1/p, AdamW per shard, all_gather)."""
    p = 8
    N = rc_inputs.LLAMA2_7B_LAYER_ELEMS
    grads = rc_inputs.draw(rc_inputs.config("llama_layer_grads_f32"))
    master, ea, es = rc_inputs.draw(rc_inputs.config("zero1_state"))
    gd, _ = to_dev(grads, "f32")
    md, _ = to_dev(master, "f32")
    ad, _ = to_dev(ea, "f32")
    sd, _ = to_dev(es, "f32")
    pd = [torch.empty(N, dtype=torch.bfloat16, device="cuda") for _ in range(p)]
    rc.rc_zero1_step(gd, pd, md, ad, sd, param_dtype="bf16", **HP)
    _sync(rc)
    del gd
    torch.cuda.empty_cache()
    want_p, w_th, w_m, w_v = oracle.zero1_step(grads, master, ea, es, "f32", "bf16", **HP)
    del grads, master, ea, es
    for r in range(p):
        assert_bits(to_host(md[r], "f32"), w_th[r], f"llama zero1 master shard {r}")
        assert_bits(to_host(ad[r], "f32"), w_m[r], f"llama zero1 exp_avg shard {r}")
        assert_bits(to_host(sd[r], "f32"), w_v[r], f"llama zero1 exp_avg_sq shard {r}")
    want = torch.from_numpy(want_p[0].view(np.int16)).cuda()
    for q in range(p):
        assert_bits(want_p[q], want_p[0], f"oracle params rank {q}")
        assert torch.equal(pd[q].view(torch.int16), want), f"llama zero1 params rank {q}"


def test_sharded_owner_broadcast_variant(rc):
    """The ShardedOptimizer form through library calls: every gradient tensor
    all-reduced with scale 1/p, AdamW by the owner (tensor t % p) on its fp32
    master copy, the result broadcast from the owner; against the oracle."""
    p, sizes = 4, [5, 4096, 1, 333, 8, 1 << 14]
    r = np.random.default_rng(31)
    grads = [[(r.standard_normal(s) * 1e-3).astype(np.float32) for _ in range(p)] for s in sizes]
    master = [r.uniform(-1, 1, s).astype(np.float32) for s in sizes]
    ea = [(r.standard_normal(s) * 1e-3).astype(np.float32) for s in sizes]
    es = [np.square(r.standard_normal(s) * 1e-3).astype(np.float32) for s in sizes]
    want, w_m, w_a, w_s = oracle.sharded_owner_step(grads, master, ea, es, param_dt="f32", **HP)
    for t, s in enumerate(sizes):
        owner = t % p
        gd, _ = to_dev(grads[t], "f32")
        rc.rc_all_reduce(gd, gd, scale=1.0 / p)  # in place, like dist.all_reduce(AVG)
        (th,), _ = to_dev([master[t]], "f32")
        (mm,), _ = to_dev([ea[t]], "f32")
        (vv,), _ = to_dev([es[t]], "f32")
        rc.rc_adamw_step(th, mm, vv, gd[owner], **HP)
        out, _ = empty_dev(s, "f32", p)
        out[owner] = th  # the owner's own copy is the updated master (broadcast in place)
        rc.rc_broadcast(th, out, root=owner)
        _sync(rc)
        assert_bits(to_host(th, "f32"), w_m[t], f"owner master t={t}")
        assert_bits(to_host(mm, "f32"), w_a[t], f"owner exp_avg t={t}")
        assert_bits(to_host(vv, "f32"), w_s[t], f"owner exp_avg_sq t={t}")
        for q in range(p):
            assert_bits(to_host(out[q], "f32"), want[t][q], f"owner broadcast t={t} rank {q}")


def test_zero1_single_rank(rc):
    """p = 1: no reduction partner; the step is AdamW on the whole vector (x scale)."""
    _zero1_case(rc, 1, 4096 + 4, "f32", "bf16", seed=99)
