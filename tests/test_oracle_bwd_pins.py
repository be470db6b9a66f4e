"""Pins of the oracle's backward pass (``kda_oracle.recurrent_bwd``).

The gradients are checked against central finite differences of the forward
oracle ``recurrent`` (itself pinned by the forward pins), which involve no
differentiation at all; against a closed form (no write and no decay); and
against the linearity of a gradient in the incoming gradients.  Planted
mistakes in a copy of the backward's C source must each be caught.
"""
import os
import shutil
import subprocess

import numpy as np
import pytest

from oracle import build_oracle, kda_oracle

EPS = 1e-6
TOL = 1e-6


def case(rng, lead, H, dk, dv, n_states):
    q = rng.normal(size=lead + (H, dk))
    k = rng.normal(size=lead + (H, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.normal(size=lead + (H, dv))
    la = np.log(rng.uniform(0.6, 1.0, size=lead + (H, dk)))
    b = rng.uniform(0.1, 0.9, size=lead + (H,))
    s0 = rng.normal(size=(n_states, H, dk, dv)) * 0.3
    do = rng.normal(size=lead + (H, dv))
    dsT = rng.normal(size=(n_states, H, dk, dv))
    return [q, k, v, la, b, s0], do, dsT


def fd_error(inputs, do, dsT, offs=None, library=None):
    """Worst relative difference between the backward's gradients and central
    finite differences of L = <do, out> + <dsT, final> over every input."""
    grads = kda_oracle.recurrent_bwd(*inputs, do, dsT, seq_offsets=offs,
                                     library=library)

    def loss(args):
        o, f = kda_oracle.recurrent(*args, seq_offsets=offs)
        return float((o * do).sum() + (f * dsT).sum())

    worst = 0.0
    for i, (x, g) in enumerate(zip(inputs, grads)):
        num = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            plus = [a.copy() for a in inputs]
            minus = [a.copy() for a in inputs]
            plus[i][idx] += EPS
            minus[i][idx] -= EPS
            num[idx] = (loss(plus) - loss(minus)) / (2 * EPS)
        scale = max(1.0, float(np.abs(num).max()))
        worst = max(worst, float(np.abs(num - g).max()) / scale)
    return worst


def test_backward_matches_finite_differences_small():
    rng = np.random.default_rng(40)
    inputs, do, dsT = case(rng, (2, 5), 2, 3, 2, 2)
    assert fd_error(inputs, do, dsT) < TOL


def test_backward_matches_finite_differences_across_blocks():
    # 70 tokens: the reverse pass re-runs the forward in blocks of 64
    rng = np.random.default_rng(41)
    inputs, do, dsT = case(rng, (1, 70), 1, 2, 2, 1)
    assert fd_error(inputs, do, dsT) < TOL


def test_backward_matches_finite_differences_packed():
    rng = np.random.default_rng(42)
    lengths = [3, 0, 4]
    offs = np.concatenate([[0], np.cumsum(lengths)])
    inputs, do, dsT = case(rng, (sum(lengths),), 2, 2, 3, len(lengths))
    assert fd_error(inputs, do, dsT, offs) < TOL
    # the empty sequence passes its state gradient straight through
    grads = kda_oracle.recurrent_bwd(*inputs, do, dsT, seq_offsets=offs)
    assert np.array_equal(grads[5][1], dsT[1])


def test_backward_closed_form_without_write_or_decay():
    # beta = 0 and alpha = 1: S_t = S_0 and o_t = S_0^T q_t, so
    # dq_t = S_0 dO_t, dv = dk = 0 (nothing is written), and
    # dS_0 = sum_t q_t dO_t^T + dS_T.
    rng = np.random.default_rng(43)
    (q, k, v, la, b, s0), do, dsT = case(rng, (1, 6), 1, 3, 2, 1)
    la = np.zeros_like(la)
    b = np.zeros_like(b)
    dq, dk, dv, dla, db, ds0 = kda_oracle.recurrent_bwd(q, k, v, la, b, s0, do,
                                                        dsT)
    np.testing.assert_allclose(dq[0, :, 0], do[0, :, 0] @ s0[0, 0].T, atol=1e-12)
    np.testing.assert_allclose(dv, 0.0, atol=1e-12)
    np.testing.assert_allclose(dk, 0.0, atol=1e-12)
    np.testing.assert_allclose(ds0[0, 0], q[0, :, 0].T @ do[0, :, 0] + dsT[0, 0],
                               atol=1e-12)
    # dlog_alpha_t = rowsum(D' .* S_0) with D' the gradient of S_t
    D = dsT[0, 0].copy()
    for t in range(5, -1, -1):
        D = D + np.outer(q[0, t, 0], do[0, t, 0])
        np.testing.assert_allclose(dla[0, t, 0], (D * s0[0, 0]).sum(axis=1),
                                   atol=1e-12)


def test_backward_is_linear_in_incoming_gradients():
    rng = np.random.default_rng(44)
    inputs, do1, ds1 = case(rng, (1, 9), 2, 3, 3, 1)
    _, do2, ds2 = case(rng, (1, 9), 2, 3, 3, 1)
    g1 = kda_oracle.recurrent_bwd(*inputs, do1, ds1)
    g2 = kda_oracle.recurrent_bwd(*inputs, do2, ds2)
    g12 = kda_oracle.recurrent_bwd(*inputs, do1 + 2 * do2, ds1 + 2 * ds2)
    for a, b_, c in zip(g1, g2, g12):
        np.testing.assert_allclose(c, a + 2 * b_, rtol=1e-10, atol=1e-10)


# Each entry plants one plausible mistake in the backward of a copy of the
# oracle's C source.
BWD_MUTANTS = {
    "state_gradient_not_decayed": ("D[c * dv + j] *= a;", "D[c * dv + j] *= 1.0;"),
    "error_gradient_sign": ("de[j] = -bt * dd[j];", "de[j] = bt * dd[j];"),
    "query_gradient_reads_old_state": ("acc += S_t[c * dv + j] * dot[j];",
                                       "acc += S_prev[c * dv + j] * dot[j];"),
    "gate_gradient_undecayed": ("acc += D[c * dv + j] * Sp[c * dv + j];",
                                "acc += D[c * dv + j] * S_prev[c * dv + j];"),
    "beta_gradient_without_error": ("db += dd[j] * (vt[j] - e[j]);",
                                    "db += dd[j] * vt[j];"),
}


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
@pytest.mark.parametrize("name", sorted(BWD_MUTANTS))
def test_backward_pins_catch_planted_mistake(name, tmp_path):
    old, new = BWD_MUTANTS[name]
    with open(build_oracle.SRC) as f:
        src = f.read()
    assert src.count(old) == 1, name
    mutant_c = tmp_path / f"{name}.c"
    mutant_c.write_text(src.replace(old, new))
    lib = str(tmp_path / f"lib_{name}.so")
    subprocess.check_call(["gcc", "-O1", "-std=c11", "-fopenmp", "-fPIC",
                           "-shared", "-o", lib, str(mutant_c), "-lm"])
    rng = np.random.default_rng(45)
    inputs, do, dsT = case(rng, (1, 6), 1, 3, 2, 1)
    assert fd_error(inputs, do, dsT, library=lib) > 1e-3, name
    os.remove(lib)


@pytest.mark.parametrize("T,C", [(150, 64), (150, 32), (37, 16), (1, 16)])
def test_chunked_backward_model_matches_oracle(T, C):
    # the chunkwise backward algebra (the GPU backward's recipe) against the
    # token-level gradients
    rng = np.random.default_rng(50 + T + C)
    (q, k, v, la, b, s0), do, dsT = case(rng, (1, T), 1, 6, 5, 1)
    ref = kda_oracle.recurrent_bwd(q, k, v, la, b, s0, do, dsT)
    got = kda_oracle.chunked_bwd_debug(q[0, :, 0], k[0, :, 0], v[0, :, 0],
                                       la[0, :, 0], b[0, :, 0], s0[0, 0],
                                       do[0, :, 0], dsT[0, 0], chunk=C)
    refs = [r[0, :, 0] for r in ref[:5]] + [ref[5][0, 0]]
    for g, r in zip(got, refs):
        np.testing.assert_allclose(g, r, rtol=1e-10, atol=1e-10)
