"""Pins of the fp64 oracle to facts fixed by the pages and by mathematics.

Each ``pin_*`` takes the oracle's ``recurrent`` callable (so the same checks can
be run against deliberately broken builds of the oracle source) and raises
AssertionError when the pinned fact does not hold.  Facts printed on the pages
come from ``tests/golden/*.json`` (each file names its source).
"""
import json
import os

import numpy as np

from oracle import kda_oracle

GOLD = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def gold(name):
    with open(os.path.join(GOLD, name)) as f:
        return json.load(f)


def one(rec, q, k, v, la, b, s0=None):
    """Run one (sequence, head) given as [T, d] arrays; returns (o [T, d_v],
    S_T [d_k, d_v])."""
    q, k, v, la = (np.asarray(x, dtype=np.float64) for x in (q, k, v, la))
    b = np.asarray(b, dtype=np.float64)
    out, fin = rec(q[None, :, None, :], k[None, :, None, :], v[None, :, None, :],
                   la[None, :, None, :], b[None, :, None],
                   None if s0 is None else np.asarray(s0, np.float64)[None, None])
    return out[0, :, 0], fin[0, 0]


def rand_case(rng, T, dk, dv, unit_k=True, with_state=True, gate_scale=0.3):
    q = rng.standard_normal((T, dk))
    k = rng.standard_normal((T, dk))
    if unit_k:
        k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((T, dv))
    la = -gate_scale * rng.random((T, dk))
    b = rng.random(T)
    s0 = rng.standard_normal((dk, dv)) if with_state else None
    return q, k, v, la, b, s0


# T1 -- per-channel decay worked example: a = [0.9, 0.2] on [10, 10] -> [9, 2].
def pin_per_channel_decay(rec):
    g = gold("per_channel_decay.json")
    a = np.array(g["alpha"])
    s0 = np.array(g["memory"])[:, None]                      # d_k = 2, d_v = 1
    _, S = one(rec, [[0.3, -0.7]], [[0.6, 0.8]], [[5.0]], [np.log(a)], [0.0], s0)
    assert np.allclose(S[:, 0], g["expected"], rtol=0, atol=1e-12), S[:, 0]


# T2 -- printed half-lives 6.6 and 0.43 tokens, ratio 15x.
def pin_half_lives(rec):
    g = gold("half_lives.json")
    a = np.array(g["alpha"])
    s0 = np.ones((2, 1))
    # Measure the per-token factor the oracle applies to each channel.
    _, S = one(rec, [[0.0, 0.0]], [[1.0, 0.0]], [[0.0]], [np.log(a)], [0.0], s0)
    factor = S[:, 0]
    with np.errstate(all="ignore"):
        half = np.log(0.5) / np.log(factor)
    for h, printed, dec in zip(half, g["half_life_tokens_printed"],
                               g["printed_decimals"]):
        assert round(float(h), dec) == printed, (h, printed)
    assert round(float(half[0] / half[1])) == g["ratio_printed"]
    # Whole tokens: channel 1 falls below half between tokens 6 and 7,
    # channel 2 within its first token.
    _, S6 = one(rec, np.zeros((6, 2)), np.tile([1.0, 0.0], (6, 1)),
                np.zeros((6, 1)), np.tile(np.log(a), (6, 1)), np.zeros(6), s0)
    _, S7 = one(rec, np.zeros((7, 2)), np.tile([1.0, 0.0], (7, 1)),
                np.zeros((7, 1)), np.tile(np.log(a), (7, 1)), np.zeros(7), s0)
    assert S6[0, 0] > 0.5 > S7[0, 0] and factor[1] < 0.5


# T5 -- delta-correction trace: beta = 1 on channel 2 gives exactly [4, 4];
# two 0.2-gate steps later 0.160.
def pin_delta_correction(rec):
    g = gold("delta_correction_trace.json")
    gate = np.log(np.array(g["gate"]))
    prior = np.array([[1.5, -2.0], [3.0, 7.0]])
    for corr_gate in (gate, np.zeros(2)):
        q = np.zeros((3, 2))
        k = np.array([[0.0, 1.0], [0.0, 1.0], [0.0, 1.0]])
        v = np.array([g["value"], [0.0, 0.0], [0.0, 0.0]])
        la = np.stack([corr_gate, gate, gate])
        b = np.array([1.0, 0.0, 0.0])
        _, S1 = one(rec, q[:1], k[:1], v[:1], la[:1], b[:1], prior)
        assert np.allclose(S1[1], g["after_correction_row2"], rtol=0, atol=1e-12)
        assert np.allclose(S1[0], np.exp(corr_gate[0]) * prior[0], atol=1e-12)
        _, S3 = one(rec, q, k, v, la, b, prior)
        assert np.allclose(S3[1], g["after_two_gate_steps_row2"], atol=1e-12)


# T6 -- a new key: the error is just v, the write is linear attention's.
def pin_new_key(rec):
    rng = np.random.default_rng(6)
    dk, dv = 5, 3
    q, k, v = rng.standard_normal((1, dk)), rng.standard_normal((1, dk)), \
        rng.standard_normal((1, dv))
    k /= np.linalg.norm(k)
    la, b = -0.2 * rng.random((1, dk)), np.array([0.7])
    o, S = one(rec, q, k, v, la, b, None)                    # empty memory
    assert np.allclose(S, b[0] * np.outer(k[0], v[0]), atol=1e-14)
    assert np.allclose(o[0], b[0] * (k[0] @ q[0]) * v[0], atol=1e-14)
    # Memory holding keys on channels 0, 1 only; the new key is channel 3.
    s0 = np.zeros((dk, dv))
    s0[0], s0[1] = rng.standard_normal(dv), rng.standard_normal(dv)
    e3 = np.eye(dk)[3][None]
    _, S = one(rec, q, e3, v, la, b, s0)
    expect = np.exp(la[0])[:, None] * s0 + b[0] * np.outer(e3[0], v[0])
    assert np.allclose(S, expect, atol=1e-14)


# T7 -- overwrite widget: three associations, then overwrite one.
def pin_overwrite_widget(rec):
    rng = np.random.default_rng(7)
    dk, dv = 8, 4
    Qm, _ = np.linalg.qr(rng.standard_normal((dk, dk)))
    k1, k2, k3 = Qm[:, 0], Qm[:, 1], Qm[:, 2]
    v1, v2, v3, v2n = (rng.standard_normal(dv) for _ in range(4))
    keys = np.stack([k1, k2, k3, k2, k1, k1, k1])
    vals = np.stack([v1, v2, v3, v2n, np.zeros(dv), np.zeros(dv), np.zeros(dv)])
    qs = np.stack([k1, k1, k1, k1, k1, k2, k3])
    b = np.array([1, 1, 1, 1, 0, 0, 0], dtype=float)
    o, _ = one(rec, qs, keys, vals, np.zeros((7, dk)), b, None)
    assert np.allclose(o[4], v1, atol=1e-12)
    assert np.allclose(o[5], v2n, atol=1e-12)                # the clean value
    assert np.allclose(o[6], v3, atol=1e-12)
    additive = np.outer(k1, v1) + np.outer(k2, v2) + np.outer(k3, v3) \
        + np.outer(k2, v2n)
    assert np.allclose(additive.T @ k2, v2 + v2n)            # the corrupted sum
    assert not np.allclose(o[5], v2 + v2n, atol=1e-3)


def _deltanet(q, k, v, b, s0, gates=None):
    """Textbook DeltaNet (gates None) / Gated DeltaNet (one scalar gate per
    token): S <- a S; S <- S + b k (v - S^T k)^T; o = S^T q."""
    S = np.array(s0, dtype=float, copy=True)
    out = []
    for t in range(len(k)):
        if gates is not None:
            S = gates[t] * S
        S = S + b[t] * np.outer(k[t], v[t] - S.T @ k[t])
        out.append(S.T @ q[t])
    return np.array(out), S


# T3 -- alpha = 1 is DeltaNet.
def pin_deltanet(rec):
    rng = np.random.default_rng(3)
    q, k, v, _, b, s0 = rand_case(rng, 40, 6, 4)
    o, S = one(rec, q, k, v, np.zeros_like(k), b, s0)
    o2, S2 = _deltanet(q, k, v, b, s0)
    assert np.allclose(o, o2, atol=1e-12) and np.allclose(S, S2, atol=1e-12)


# T4 -- a channel-uniform alpha is Gated DeltaNet.
def pin_gated_deltanet(rec):
    rng = np.random.default_rng(4)
    q, k, v, _, b, s0 = rand_case(rng, 40, 6, 4)
    a = np.exp(-0.5 * rng.random(40))
    la = np.repeat(np.log(a)[:, None], 6, axis=1)
    o, S = one(rec, q, k, v, la, b, s0)
    o2, S2 = _deltanet(q, k, v, b, s0, gates=a)
    assert np.allclose(o, o2, atol=1e-12) and np.allclose(S, S2, atol=1e-12)


# T8 -- brute-force unrolled products, T <= 8 (d_k != d_v to expose transposes).
def pin_brute_force(rec):
    rng = np.random.default_rng(8)
    for T, dk, dv, st, unit in ((1, 3, 2, True, True), (5, 5, 3, True, True),
                                (8, 4, 6, False, True), (8, 6, 5, True, False)):
        q, k, v, la, b, s0 = rand_case(rng, T, dk, dv, unit_k=unit,
                                       with_state=st, gate_scale=1.0)
        o, S = one(rec, q, k, v, la, b, s0)
        ob, Sb = kda_oracle.brute_force(q, k, v, la, b, s0)
        assert np.allclose(o, ob, atol=1e-12), np.abs(o - ob).max()
        assert np.allclose(S, Sb, atol=1e-12), np.abs(S - Sb).max()


# T9 -- beta = 0 is pure decay, in closed form.
def pin_pure_decay(rec):
    rng = np.random.default_rng(9)
    q, k, v, la, _, s0 = rand_case(rng, 30, 5, 3, gate_scale=0.5)
    o, S = one(rec, q, k, v, la, np.zeros(30), s0)
    g = np.cumsum(la, axis=0)
    assert np.allclose(S, np.exp(g[-1])[:, None] * s0, atol=1e-13)
    assert np.allclose(o, (np.exp(g) * q) @ s0, atol=1e-13)


# T10 -- exact recall: q = k, beta = 1, unit keys -> o_t = v_t exactly.
def pin_exact_recall(rec):
    rng = np.random.default_rng(10)
    _, k, v, la, _, s0 = rand_case(rng, 300, 16, 12, gate_scale=0.5)
    o, _ = one(rec, k, k, v, la, np.ones(300), s0)
    assert np.allclose(o, v, atol=1e-12), np.abs(o - v).max()


# T11 -- state hand-off: one call equals two calls joined by the state; the
# packed variable-length layout equals separate calls.
def pin_state_handoff(rec):
    rng = np.random.default_rng(11)
    H, dk, dv, T = 3, 6, 5, 50
    q = rng.standard_normal((1, T, H, dk))
    k = rng.standard_normal((1, T, H, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((1, T, H, dv))
    la = -0.3 * rng.random((1, T, H, dk))
    b = rng.random((1, T, H))
    s0 = rng.standard_normal((1, H, dk, dv))
    o, S = rec(q, k, v, la, b, s0)
    t1 = 17
    oa, Sa = rec(q[:, :t1], k[:, :t1], v[:, :t1], la[:, :t1], b[:, :t1], s0)
    ob, Sb = rec(q[:, t1:], k[:, t1:], v[:, t1:], la[:, t1:], b[:, t1:], Sa)
    assert np.allclose(np.concatenate([oa, ob], 1), o, atol=1e-12)
    assert np.allclose(Sb, S, atol=1e-12)
    offs = [0, 9, 9, 30, T]                    # includes an empty sequence
    s0v = rng.standard_normal((4, H, dk, dv))
    ov, Sv = rec(q[0], k[0], v[0], la[0], b[0], s0v, seq_offsets=offs)
    for s in range(4):
        a, e = offs[s], offs[s + 1]
        oo, SS = rec(q[:, a:e], k[:, a:e], v[:, a:e], la[:, a:e], b[:, a:e],
                     s0v[s:s + 1])
        assert np.allclose(ov[a:e], oo[0], atol=1e-12)
        assert np.allclose(Sv[s], SS[0], atol=1e-12)


# T12 -- the chunkwise rewrite reproduces the recurrence (any chunk size, a
# ragged last chunk) and, from a zero state, the output is linear in V.
def pin_chunked_model(rec):
    rng = np.random.default_rng(12)
    q, k, v, la, b, s0 = rand_case(rng, 200, 8, 6, gate_scale=0.2)
    o, S = one(rec, q, k, v, la, b, s0)
    for C in (16, 64, 7):
        r = kda_oracle.chunked_debug(q, k, v, la, b, s0, chunk=C)
        assert np.allclose(r["out"], o, atol=1e-10), (C, np.abs(r["out"] - o).max())
        assert np.allclose(r["final"], S, atol=1e-10)
    v2 = rng.standard_normal(v.shape)
    o1, _ = one(rec, q, k, v, la, b, None)
    o2, _ = one(rec, q, k, v2, la, b, None)
    o12, _ = one(rec, q, k, 2.0 * v - 3.0 * v2, la, b, None)
    assert np.allclose(o12, 2.0 * o1 - 3.0 * o2, atol=1e-10)


ALL_PINS = [pin_per_channel_decay, pin_half_lives, pin_delta_correction,
            pin_new_key, pin_overwrite_widget, pin_deltanet,
            pin_gated_deltanet, pin_brute_force, pin_pure_decay,
            pin_exact_recall, pin_state_handoff, pin_chunked_model]


def failing_pins(rec):
    """Names of the pins that ``rec`` fails."""
    bad = []
    for p in ALL_PINS:
        try:
            p(rec)
        except AssertionError:
            bad.append(p.__name__)
    return bad

