"""Pins for the oracle's optimizer step (oracle/rc_oracle.c rco_adamw and the
ZeRO-1 / ShardedOptimizer compositions in oracle/__init__.py).

What fixes the answer independently of the oracle's own code:
  * closed forms: with binary-exact hyperparameters (beta1 = 1/2, beta2 = 3/4,
    lr and weight decay powers of two, eps = 0) the first step from zero
    moments is exactly theta*(1 - lr*wd) - lr*sign(g), m = g/2, v = g^2/4;
    a zero gradient leaves the moments at zero and only decays theta;
  * a library routine: torch.optim.AdamW (float64, one step from the same
    fp32 state) agrees within the rounding bound of the binary32 evaluation;
  * identities: the ZeRO-1 step (reduce_scatter -> AdamW on each shard ->
    all_gather) gives bit for bit the unsharded AdamW step on the averaged
    gradient, and the ShardedOptimizer form gives every rank the owner's
    update of each tensor.
"""
import numpy as np
import pytest
import torch

import oracle

U = 2.0 ** -24


def _rng(seed):
    return np.random.default_rng(seed)


def test_first_step_closed_form_exact_hyperparameters():
    g = np.array([1.0, -2.0, 0.5, -0.25, 3.0, -1e-3, 7.5, -64.0], np.float32)
    theta = np.array([1.0, 1.0, -2.0, 0.5, 4.0, -1.0, 0.25, 8.0], np.float32)
    lr, wd = 2.0 ** -10, 2.0 ** -3
    th, m, v = oracle.adamw(theta, np.zeros(8, np.float32), np.zeros(8, np.float32), g,
                            lr=lr, beta1=0.5, beta2=0.75, eps=0.0, weight_decay=wd, step=1)
    want = theta.astype(np.float64) * (1 - lr * wd) - lr * np.sign(g)
    assert np.array_equal(th, want.astype(np.float32))
    assert np.array_equal(th.astype(np.float64), want)  # every value is exact in binary32
    assert np.array_equal(m, g * 0.5)
    assert np.array_equal(v, (g.astype(np.float64) ** 2 * 0.25).astype(np.float32))


def test_zero_gradient_only_decays():
    theta = _rng(1).standard_normal(64).astype(np.float32)
    th, m, v = oracle.adamw(theta, np.zeros(64, np.float32), np.zeros(64, np.float32),
                            np.zeros(64, np.float32), lr=0.01, weight_decay=0.1, step=3)
    assert np.array_equal(th, theta * np.float32(1 - 0.01 * 0.1))
    assert not m.any() and not v.any()


def test_zero_gradient_no_decay_is_identity():
    theta = _rng(2).standard_normal(33).astype(np.float32)
    th, _, _ = oracle.adamw(theta, np.zeros(33, np.float32), np.zeros(33, np.float32),
                            np.zeros(33, np.float32), lr=0.5, weight_decay=0.0, step=1)
    assert np.array_equal(th, theta)


def test_bias_correction_second_step_closed_form():
    # step 2 with beta1 = beta2 = 1/2, eps = 0, wd = 0, constant gradient g:
    # m = 3g/4, v = 3g^2/4, bias corrections 3/4 -> mhat = g, vhat = g^2,
    # so the update is again exactly lr*sign(g)
    g = np.array([2.0, -0.5, 4.0, -8.0], np.float32)
    th1, m1, v1 = oracle.adamw(np.zeros(4, np.float32), np.zeros(4, np.float32),
                               np.zeros(4, np.float32), g, lr=0.25, beta1=0.5, beta2=0.5, eps=0.0, step=1)
    th2, m2, v2 = oracle.adamw(th1, m1, v1, g, lr=0.25, beta1=0.5, beta2=0.5, eps=0.0, step=2)
    assert np.array_equal(th2, -0.5 * np.sign(g).astype(np.float32))
    assert np.array_equal(m2, 0.75 * g)


def _torch64_step(theta, m, v, g, step, **hp):
    """torch.optim.AdamW in float64, one step from the given state."""
    p = torch.nn.Parameter(torch.from_numpy(theta.astype(np.float64)))
    opt = torch.optim.AdamW([p], lr=hp["lr"], betas=(hp["beta1"], hp["beta2"]), eps=hp["eps"],
                            weight_decay=hp["weight_decay"], foreach=False)
    p.grad = torch.from_numpy(g.astype(np.float64))
    st = opt.state[p]
    st["step"] = torch.tensor(float(step - 1), dtype=torch.float64)
    st["exp_avg"] = torch.from_numpy(m.astype(np.float64))
    st["exp_avg_sq"] = torch.from_numpy(v.astype(np.float64))
    opt.step()
    return p.detach().numpy(), st["exp_avg"].numpy(), st["exp_avg_sq"].numpy()


HPS = [
    dict(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.01),
    dict(lr=0.1, beta1=0.8, beta2=0.95, eps=1e-3, weight_decay=0.5),   # eps and decay matter
    dict(lr=3e-4, beta1=0.9, beta2=0.98, eps=1e-6, weight_decay=0.0),
]


@pytest.mark.parametrize("hp", range(len(HPS)))
@pytest.mark.parametrize("step", [1, 2, 7, 1000])
def test_against_torch_adamw_float64(hp, step):
    # the oracle takes binary32 hyperparameters: give torch the same values
    hpd = {k: float(np.float32(v)) for k, v in HPS[hp].items()}
    r = _rng(10 + hp * 31 + step)
    n = 4096
    theta = r.standard_normal(n).astype(np.float32)
    g = (r.standard_normal(n) * 10.0 ** r.uniform(-4, 0, n)).astype(np.float32)
    if step == 1:
        m = np.zeros(n, np.float32)
        v = np.zeros(n, np.float32)
    else:
        m = (r.standard_normal(n) * 1e-2).astype(np.float32)
        v = (r.uniform(0, 1, n) * 10.0 ** r.uniform(-8, -2, n)).astype(np.float32)
    th, mm, vv = oracle.adamw(theta, m, v, g, step=step, **hpd)
    th_t, m_t, v_t = _torch64_step(theta, m, v, g, step, **hpd)
    b1, b2, lr = hpd["beta1"], hpd["beta2"], hpd["lr"]
    # binary32 evaluation bounds (a few roundings per line, the scalars rounded once)
    tol_m = 4 * U * (np.abs(b1 * m.astype(np.float64)) + np.abs((1 - b1) * g.astype(np.float64))) + 1e-45
    tol_v = 4 * U * (np.abs(b2 * v.astype(np.float64)) + np.abs((1 - b2) * g.astype(np.float64) ** 2)) + 1e-45
    assert np.all(np.abs(mm - m_t) <= tol_m)
    assert np.all(np.abs(vv - v_t) <= tol_v)
    upd = np.abs(th_t - theta.astype(np.float64) * (1 - lr * hpd["weight_decay"]))
    tol_th = 2 * U * (np.abs(theta) + np.abs(th_t)) + 16 * U * upd + 1e-45
    err = np.abs(th.astype(np.float64) - th_t)
    assert np.all(err <= tol_th), float(np.max(err / tol_th))


def test_bf16_gradient_is_widened_exactly():
    r = _rng(5)
    g32 = r.standard_normal(256).astype(np.float32)
    gb = oracle.f32_to_bf16(g32)
    theta = r.standard_normal(256).astype(np.float32)
    z = np.zeros(256, np.float32)
    a = oracle.adamw(theta, z, z, gb, grad_dt="bf16", lr=1e-2, step=1)
    b = oracle.adamw(theta, z, z, oracle.bf16_to_f32(gb), grad_dt="f32", lr=1e-2, step=1)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)


@pytest.mark.parametrize("p,n,param_dt,grad_dt", [(4, 64, "f32", "f32"), (8, 4096, "bf16", "f32"),
                                                   (2, 10, "bf16", "bf16"), (8, 8 * 33, "f32", "bf16")])
def test_zero1_equals_unsharded_adamw_on_averaged_gradient(p, n, param_dt, grad_dt):
    r = _rng(100 + p + n)
    g32 = [(r.standard_normal(n) * 1e-3).astype(np.float32) for _ in range(p)]
    grads = g32 if grad_dt == "f32" else [oracle.f32_to_bf16(x) for x in g32]
    m = n // p
    master = r.standard_normal(n).astype(np.float32)
    ea = (r.standard_normal(n) * 1e-3).astype(np.float32)
    es = (r.uniform(0, 1e-6, n)).astype(np.float32)
    hp = dict(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.1, step=5)
    sh = lambda a: [a[k * m:(k + 1) * m] for k in range(p)]
    params, mas, ea2, es2 = oracle.zero1_step(grads, sh(master), sh(ea), sh(es), grad_dt=grad_dt,
                                              param_dt=param_dt, **hp)
    # unsharded: all_reduce of the (exactly widened) gradients with the same
    # scale, kept in fp32, then AdamW on the full vector
    g_f32 = grads if grad_dt == "f32" else [oracle.bf16_to_f32(x) for x in grads]
    gfull = oracle.all_reduce(g_f32, "f32", "sum", 1.0 / p)[0]
    th, mm, vv = oracle.adamw(master, ea, es, gfull, "f32", **hp)
    assert np.array_equal(np.concatenate(mas), th)
    assert np.array_equal(np.concatenate(ea2), mm)
    assert np.array_equal(np.concatenate(es2), vv)
    want = th if param_dt == "f32" else oracle.f32_to_bf16(th)
    for q in range(p):
        assert np.array_equal(params[q], want)


def test_sharded_owner_step_every_rank_gets_the_owner_update():
    r = _rng(7)
    p, sizes = 4, [5, 16, 1, 33, 8]
    grads = [[(r.standard_normal(s) * 1e-2).astype(np.float32) for _ in range(p)] for s in sizes]
    master = [r.standard_normal(s).astype(np.float32) for s in sizes]
    ea = [np.zeros(s, np.float32) for s in sizes]
    es = [np.zeros(s, np.float32) for s in sizes]
    hp = dict(lr=1e-2, beta1=0.9, beta2=0.99, eps=1e-8, weight_decay=0.0, step=1)
    params, mas, _, _ = oracle.sharded_owner_step(grads, master, ea, es, param_dt="f32", **hp)
    for t, s in enumerate(sizes):
        g = oracle.all_reduce(grads[t], "f32", "sum", 1.0 / p)[t % p]
        th, _, _ = oracle.adamw(master[t], ea[t], es[t], g, **hp)
        assert np.array_equal(mas[t], th)
        for q in range(p):
            assert np.array_equal(params[t][q], th)
