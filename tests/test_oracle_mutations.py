"""Planted mistakes: each case copies the oracle's C source, plants one
plausible slip, builds the copy, and runs the pin tests against it.  Every
slip must make the pins fail -- otherwise the pins could not tell a wrong
oracle from a right one.  CPU only; the real oracle is never modified.
"""
import concurrent.futures
import os
import subprocess
import sys
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "rc_oracle.c")

MUTANTS = {
    "fold_starts_at_own_chunk_rank": [
        ("int r = (int)((c + 1) % (size_t)q);", "int r = (int)(c % (size_t)q);"),
        ("r = (int)((c + 1 + (size_t)k) % (size_t)q);", "r = (int)((c + (size_t)k) % (size_t)q);"),
    ],
    "fold_in_ascending_rank_order": [
        ("int r = (int)((c + 1) % (size_t)q);", "int r = 0;"),
        ("r = (int)((c + 1 + (size_t)k) % (size_t)q);", "r = k;"),
    ],
    "dropped_last_rank": [
        ("for (int k = 1; k < q; ++k) {\n        r = (int)", "for (int k = 1; k < q - 1; ++k) {\n        r = (int)"),
    ],
    "sum_sign_flipped": [("acc.f = acc.f + v.f;", "acc.f = acc.f - v.f;")],
    "max_ties_take_new_operand": [("acc.f = (v.f > acc.f) ? v.f : acc.f;", "acc.f = (v.f >= acc.f) ? v.f : acc.f;")],
    "scale_ignored": [("float y = acc.f * scale;", "float y = acc.f;")],
    "reduce_scatter_wrong_slice": [("size_t i = (size_t)r * m + j;", "size_t i = (size_t)((r + 1) % p) * m + j;")],
    "bf16_ties_round_up": [("if (lo > 0x8000u || (lo == 0x8000u && (hi & 1u) != 0u))", "if (lo >= 0x8000u)")],
    "ring_receiver_operands_swapped": [("combine(msg[r][i - b], w[d][i], is_int, op)", "combine(w[d][i], msg[r][i - b], is_int, op)")],
    "ring_allgather_wrong_chunk": [("size_t c = (size_t)(((r - k) % p + p) % p);", "size_t c = (size_t)(((r - k - 1) % p + p) % p);")],
    "hier_leader_sum_starts_at_own_group": [("int g = (int)((c + 1) % (size_t)ng);", "int g = (int)(c % (size_t)ng);"),
                                            ("g = (int)((c + 1 + (size_t)k) % (size_t)ng);",
                                             "g = (int)((c + (size_t)k) % (size_t)ng);")],
    "ring_reduce_scatter_chunk_shifted": [("size_t c = (size_t)(((r - k - 1) % q + q) % q);",
                                           "size_t c = (size_t)(((r - k) % q + q) % q);")],
    "hier_group_drops_a_rank": [("ring_core(send + (size_t)g * (size_t)G, G,", "ring_core(send + (size_t)g * (size_t)G, G > 1 ? G - 1 : G,")],
    "adamw_no_first_bias_correction": [("float mhat = mi / bc1;", "float mhat = mi;")],
    "adamw_eps_inside_sqrt": [("float den = sqrtf(vhat) + eps;", "float den = sqrtf(vhat + eps);")],
    "adamw_decay_after_update": [("float th = theta[i] * decay;", "float th = theta[i];"),
                                 ("th = th - lr * (mhat / den);", "th = (th - lr * (mhat / den)) * decay;")],
    "adamw_second_moment_of_g_not_g2": [("float vi = beta2 * v[i] + omb2 * (gi * gi);",
                                         "float vi = beta2 * v[i] + omb2 * gi;")],
    "adamw_update_sign_flipped": [("th = th - lr * (mhat / den);", "th = th + lr * (mhat / den);")],
    "adamw_betas_swapped": [("float mi = beta1 * m[i] + omb1 * gi;", "float mi = beta2 * m[i] + omb2 * gi;")],
    "a2a_recv_offset_by_destination": [("for (int k = 0; k < r; ++k)\n                roff += counts[(size_t)k * p + q];",
                                        "for (int k = 0; k < q; ++k)\n                roff += counts[(size_t)r * p + k];")],
    "a2a_send_offset_off_by_one": [("for (int k = 0; k < q; ++k)\n                soff += counts[(size_t)r * p + k];",
                                    "for (int k = 0; k <= q && k < p - 1; ++k)\n                soff += counts[(size_t)r * p + k];")],
    "a2a_transposed_count": [("uint64_t c = counts[(size_t)r * p + q];", "uint64_t c = counts[(size_t)q * p + r];")],
    "a2a_traffic_swapped": [("traffic[r == q ? 0 : 1] += c * (uint64_t)esz;", "traffic[r == q ? 1 : 0] += c * (uint64_t)esz;")],
    "reduce_at_chunk_from_index_count": [("acc_t a = fold_ring_order(send, p, n, (size_t)idx[j], in_dt, op);",
                                          "acc_t a = fold_ring_order(send, p, k, (size_t)idx[j], in_dt, op);")],
    "reduce_at_scale_dropped": [("store_result(out, j, out_dt, a, scale);", "store_result(out, j, out_dt, a, 1.0f);")],
    "reduce_at_accepts_index_n": [("if (idx[j] >= n)\n            return RCO_EINVAL;",
                                   "if (idx[j] > n)\n            return RCO_EINVAL;")],
    "int_sum_saturates": [("acc.i = (int32_t)((uint32_t)acc.i + (uint32_t)v.i);",
                           "{ long long t = (long long)acc.i + v.i; acc.i = t > 2147483647LL ? 2147483647 : (t < -2147483648LL ? (int32_t)-2147483648LL : (int32_t)t); }")],
}


def _run_mutant(name):
    """Build one mutant and run the pins against it; returns (returncode, tail of output)."""
    src = open(SRC).read()
    for old, new in MUTANTS[name]:
        if src.count(old) < 1:
            return None, f"mutation anchor not found: {old!r}"
        src = src.replace(old, new)
    with tempfile.TemporaryDirectory() as d:
        c = os.path.join(d, "mutant.c")
        so = os.path.join(d, "libmutant.so")
        open(c, "w").write(src)
        subprocess.run(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off",
                        "-o", so, c, "-lm"], check=True)
        env = dict(os.environ, RC_ORACLE_LIB=so)
        # the pin file that covers the mutated function runs first, so that a
        # caught mutant stops at its first failure
        pins = ["test_oracle_pins.py", "test_oracle_optim.py", "test_oracle_a2a.py"]
        first = ("test_oracle_optim.py" if name.startswith("adamw") else
                 "test_oracle_a2a.py" if name.startswith("a2a") else "test_oracle_pins.py")
        pins.remove(first)
        r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider"] +
                           [os.path.join(ROOT, "tests", f) for f in [first] + pins],
                           cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    return r.returncode, r.stdout[-2000:]


@pytest.fixture(scope="module")
def mutant_results():
    """All mutants, built and checked in parallel (independent processes)."""
    workers = max(1, min(8, (os.cpu_count() or 2)))
    with concurrent.futures.ThreadPoolExecutor(max_workers=workers) as ex:
        futs = {n: ex.submit(_run_mutant, n) for n in MUTANTS}
        return {n: f.result() for n, f in futs.items()}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistake(name, mutant_results):
    rc, out = mutant_results[name]
    assert rc is not None, out
    assert rc != 0, f"pins did not catch mutant {name}:\n{out}"
