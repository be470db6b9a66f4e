"""The algebra behind the sequence split (kda_chunk_fwd_split), checked with
the fp64 oracle alone.  The state update is affine in the state, so inside a
segment entered with state S_in:
    S_t = M_t S_in + S_t|0,      o_t = o_t|0 + S_in^T (M_t^T q_t),
where |0 is the evaluation from zero and M_t (the product of the token
transitions) is the state of the same recurrence run with v = 0 from the
identity, M_t^T q_t its output.  Segments joined by the scan S_in(j+1) =
M_end(j) S_in(j) + S_end|0(j) must reproduce the unsplit recurrence; planted
mistakes in the join must not."""
import numpy as np
import pytest

from oracle import kda_oracle


def case(rng, T, H, dk, dv):
    q = rng.normal(size=(1, T, H, dk))
    k = rng.normal(size=(1, T, H, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.normal(size=(1, T, H, dv))
    la = np.log(rng.uniform(0.7, 1.0, size=(1, T, H, dk)))
    b = rng.uniform(0.1, 0.9, size=(1, T, H))
    s0 = rng.normal(size=(1, H, dk, dv)) * 0.3
    return q, k, v, la, b, s0


def split_eval(q, k, v, la, b, s0, bounds, mistake=None):
    """The split's four steps on the oracle: value runs, transition runs,
    scan, correction.  ``bounds`` are the segment start tokens plus T."""
    H, dk = q.shape[2], q.shape[3]
    outs, s_in = [], s0[0]
    for j in range(len(bounds) - 1):
        sl = slice(bounds[j], bounds[j + 1])
        seg = [x[:, sl] for x in (q, k, v, la, b)]
        if j == 0:  # segment 0 from the true start state
            o, e = kda_oracle.recurrent(*seg, s0)
            outs.append(o)
            s_in = e[0]
            continue
        o0, e0 = kda_oracle.recurrent(*seg, None)            # value run
        ident = np.broadcast_to(np.eye(dk), (1, H, dk, dk)).copy()
        zero_v = np.zeros(seg[0].shape)                       # d_v = d_k
        X, M = kda_oracle.recurrent(seg[0], seg[1], zero_v, seg[3], seg[4],
                                    ident)                     # transition run
        corr = np.einsum("thc,hcj->thj", X[0], s_in)          # S_in^T x_t
        if mistake == "no_correction":
            corr = 0 * corr
        outs.append(o0 + corr[None])
        Mj = M[0]
        if mistake == "transposed_transition":
            Mj = np.swapaxes(Mj, -1, -2)
        if mistake == "transition_dropped":  # S_in + S_end|0, no M_end
            s_in = s_in + e0[0]
        else:
            s_in = np.einsum("hcd,hde->hce", Mj, s_in) + e0[0]
    return np.concatenate(outs, axis=1), s_in[None]


@pytest.mark.parametrize("bounds", [[0, 16, 40], [0, 10, 20, 33, 40], [0, 1, 40]])
def test_split_reproduces_the_recurrence(bounds):
    rng = np.random.default_rng(7 + len(bounds))
    q, k, v, la, b, s0 = case(rng, 40, 2, 4, 3)
    ref_o, ref_s = kda_oracle.recurrent(q, k, v, la, b, s0)
    o, s = split_eval(q, k, v, la, b, s0, bounds)
    np.testing.assert_allclose(o, ref_o, rtol=1e-11, atol=1e-11)
    np.testing.assert_allclose(s, ref_s, rtol=1e-11, atol=1e-11)


def test_transition_run_is_the_transition_product():
    # with v = 0 and the identity start, the final state is the product of
    # (I - beta k k^T) Diag(alpha) over the tokens, built here by brute force
    rng = np.random.default_rng(3)
    q, k, v, la, b, s0 = case(rng, 9, 1, 3, 2)
    ident = np.eye(3)[None, None]
    _, M = kda_oracle.recurrent(q, k, np.zeros_like(q), la, b, ident)
    P = np.eye(3)
    for t in range(9):
        kt = k[0, t, 0]
        A = (np.eye(3) - b[0, t, 0] * np.outer(kt, kt)) @ np.diag(np.exp(la[0, t, 0]))
        P = A @ P
    np.testing.assert_allclose(M[0, 0], P, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("mistake", ["no_correction", "transposed_transition",
                                     "transition_dropped"])
def test_split_mistakes_are_caught(mistake):
    rng = np.random.default_rng(11)
    q, k, v, la, b, s0 = case(rng, 40, 2, 4, 3)
    ref_o, ref_s = kda_oracle.recurrent(q, k, v, la, b, s0)
    o, s = split_eval(q, k, v, la, b, s0, [0, 10, 20, 33, 40], mistake=mistake)
    err = max(np.abs(o - ref_o).max(), np.abs(s - ref_s).max())
    assert err > 1e-3, (mistake, err)
