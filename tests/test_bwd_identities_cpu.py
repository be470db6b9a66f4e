"""Two identities the backward kernels rely on, checked in fp64 against the
token-level oracle (no GPU):

1. The state leaving a chunk is Diag(gam) (S_0 + Kb^T Delta) with gam =
   exp(g_C): the token recurrence's state at each chunk boundary equals that
   expression built from the chunk's own factors.  The reverse chain
   therefore reads gam * d gam = rowsum(S_next * dS_C) from the next chunk's
   stored start state (or the final state) instead of forming Kb^T Delta.

2. rowsum(dA * M) = rowsum((dA Kb) * Kt) for a strictly lower dA, with M the
   strictly lower part of Kt Kb^T: the final d beta sum uses the right-hand
   side, so M is never stored.

A planted mistake in either (the decay left out, Kb and Kt swapped) must
fail."""
import numpy as np
import pytest

from oracle import kda_oracle


def inputs(rng, T, dk, dv):
    q = rng.normal(size=(1, T, 1, dk))
    k = rng.normal(size=(1, T, 1, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.normal(size=(1, T, 1, dv))
    la = np.log(rng.uniform(0.6, 1.0, size=(1, T, 1, dk)))
    b = rng.uniform(0.1, 0.9, size=(1, T, 1))
    s0 = rng.normal(size=(1, 1, dk, dv)) * 0.3
    return q, k, v, la, b, s0


@pytest.mark.parametrize("T,C", [(70, 16), (64, 32), (50, 64)])
def test_state_leaving_a_chunk(T, C):
    rng = np.random.default_rng(T + C)
    q, k, v, la, b, s0 = inputs(rng, T, 5, 4)
    rec = kda_oracle.chunked_debug(q[0, :, 0], k[0, :, 0], v[0, :, 0],
                                   la[0, :, 0], b[0, :, 0], s0[0, 0], chunk=C)
    starts = list(range(0, T, C))
    for n, c0 in enumerate(starts):
        c1 = min(T, c0 + C)
        # the state after token c1 - 1, from the token recurrence
        _, s_tok = kda_oracle.recurrent(q[:, :c1], k[:, :c1], v[:, :c1],
                                        la[:, :c1], b[:, :c1], s0)
        g = rec["g"][n]
        kc = k[0, c0:c1, 0]
        Kb = kc * np.exp(-g)
        delta = rec["U"][n] - rec["W"][n] @ rec["S_start"][n]
        s_next = np.exp(g[-1])[:, None] * (rec["S_start"][n] + Kb.T @ delta)
        np.testing.assert_allclose(s_next, s_tok[0, 0], rtol=1e-10, atol=1e-10)
        # and without the decay the identity fails
        wrong = rec["S_start"][n] + Kb.T @ delta
        assert np.abs(wrong - s_tok[0, 0]).max() > 1e-3


@pytest.mark.parametrize("L,dk", [(64, 128), (37, 32), (16, 8)])
def test_beta_row_sum_identity(L, dk):
    rng = np.random.default_rng(L * dk)
    k = rng.normal(size=(L, dk))
    g = np.cumsum(np.log(rng.uniform(0.8, 1.0, size=(L, dk))), axis=0)
    Kt, Kb = k * np.exp(g), k * np.exp(-g)
    M = np.tril(Kt @ Kb.T, -1)
    dA = np.tril(rng.normal(size=(L, L)), -1)
    lhs = (dA * M).sum(axis=1)
    rhs = ((dA @ Kb) * Kt).sum(axis=1)
    np.testing.assert_allclose(rhs, lhs, rtol=1e-10, atol=1e-10)
    # swapping the two factors breaks it
    wrong = ((dA @ Kt) * Kb).sum(axis=1)
    assert np.abs(wrong - lhs).max() > 1e-6
