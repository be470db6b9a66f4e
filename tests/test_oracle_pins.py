"""The fp64 oracle against the facts the pages print and mathematics fixes."""
import os
import shutil
import subprocess

import numpy as np
import pytest

import oracle_pins as P
from oracle import build_oracle, kda_oracle


@pytest.mark.parametrize("pin", P.ALL_PINS, ids=lambda p: p.__name__)
def test_pin(pin):
    pin(kda_oracle.recurrent)


def test_brute_force_matches_closed_forms():
    # The brute force itself, at beta = 0 (pure decay) and alpha = 1, beta = 1
    # with orthonormal keys (exact recall), without going through the recurrence.
    rng = np.random.default_rng(21)
    q, k, v, la, _, s0 = P.rand_case(rng, 6, 4, 3)
    o, S = kda_oracle.brute_force(q, k, v, la, np.zeros(6), s0)
    g = np.cumsum(la, 0)
    assert np.allclose(S, np.exp(g[-1])[:, None] * s0, atol=1e-13)
    assert np.allclose(o, (np.exp(g) * q) @ s0, atol=1e-13)
    Qm, _ = np.linalg.qr(rng.standard_normal((4, 4)))
    keys = Qm.T[[0, 1, 2, 1]]
    vals = rng.standard_normal((4, 3))
    o, S = kda_oracle.brute_force(keys, keys, vals, np.zeros((4, 4)),
                                  np.ones(4), None)
    assert np.allclose(o, vals, atol=1e-12)


def test_forward_substitution_inverse():
    rng = np.random.default_rng(22)
    A = np.tril(rng.standard_normal((9, 9)), -1) * 0.3
    X = kda_oracle._forward_substitution_inverse(A)
    assert np.allclose(X @ (np.eye(9) + A), np.eye(9), atol=1e-12)


def test_bad_offsets_rejected():
    z = np.zeros((4, 1, 2))
    with pytest.raises(ValueError):
        kda_oracle.recurrent(z, z, z, z, np.zeros((4, 1)), seq_offsets=[0, 3])


# Each entry plants one plausible mistake in a copy of the oracle's C source.
MUTANTS = {
    "error_sign": ("bt * kt[c] * (vt[j] - e[j])", "bt * kt[c] * (vt[j] + e[j])"),
    "gate_not_exponentiated": ("const double a = exp(lt[c]);",
                               "const double a = 1.0 + lt[c];"),
    "error_from_undecayed_state": ("e[j] += S[c * dv + j] * kt[c];",
                                   "e[j] += S[c * dv + j] * kt[c] / exp(lt[c]);"),
    "output_before_write": (
        "ot[j] += S[c * dv + j] * qt[c];",
        "ot[j] += (S[c * dv + j] - bt * kt[c] * (vt[j] - e[j])) * qt[c];"),
    "beta_dropped": ("S[c * dv + j] += bt * kt[c]", "S[c * dv + j] += kt[c]"),
    "decay_on_value_columns": ("S[c * dv + j] *= a;",
                               "S[c * dv + j] *= exp(lt[j % dk]);"),
    "output_reads_key": ("ot[j] += S[c * dv + j] * qt[c];",
                         "ot[j] += S[c * dv + j] * kt[c];"),
}


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistake(name, tmp_path):
    old, new = MUTANTS[name]
    with open(build_oracle.SRC) as f:
        src = f.read()
    assert src.count(old) >= 1, name
    mutant_c = tmp_path / f"{name}.c"
    mutant_c.write_text(src.replace(old, new))
    lib = str(tmp_path / f"lib_{name}.so")
    subprocess.check_call(["gcc", "-O1", "-std=c11", "-fopenmp", "-fPIC",
                           "-shared", "-o", lib, str(mutant_c), "-lm"])

    def rec(*a, **kw):
        return kda_oracle.recurrent(*a, library=lib, **kw)

    failed = P.failing_pins(rec)
    assert failed, f"no pin caught the planted mistake {name!r}"
    os.remove(lib)


def test_prologue_closed_forms():
    # logsigmoid: 0 -> -log 2; large positive -> 0; large negative -> x;
    # L2 normalisation gives unit (or q_scale) norms and keeps direction.
    rng = np.random.default_rng(30)
    q = rng.standard_normal((3, 5, 2, 8))
    k = rng.standard_normal((3, 5, 2, 8))
    g = np.array([0.0, 40.0, -40.0, 1.0])
    qn, kn, la = kda_oracle.prologue(q, k, g, q_scale=0.25, gate_scale=0.5)
    assert np.allclose(np.linalg.norm(qn, axis=-1), 0.25)
    assert np.allclose(np.linalg.norm(kn, axis=-1), 1.0)
    assert np.allclose(np.sum(kn * k, axis=-1), np.linalg.norm(k, axis=-1))
    assert np.isclose(la[0], -0.5 * np.log(2.0))
    assert abs(la[1]) < 1e-15 and np.isclose(la[2], -20.0)
    assert np.isclose(la[3], 0.5 * np.log(1.0 / (1.0 + np.exp(-1.0))))
    # no normalisation: only the scale; no logits: the gate passes through
    q2, k2, la2 = kda_oracle.prologue(q, k, g, normalize_qk=False, q_scale=2.0,
                                      gate_logits=False)
    assert np.allclose(q2, 2.0 * q) and np.allclose(k2, k) and np.allclose(la2, g)
