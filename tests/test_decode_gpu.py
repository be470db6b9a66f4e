"""kda_recurrent_step (token-by-token decode kernel) against the fp64 oracle."""
import numpy as np
import pytest
import torch

import kda_workloads as W
import parity as PY
from gated_delta_rule_156_b200 import kda as K
from oracle import kda_oracle

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _decode_case(N, H, dk, dv, T, io, seed, with_state=True):
    d = W.draw((N, T), H, dk, dv, io=io, n_states=N if with_state else None,
               device=DEV, seed=seed)
    state = d["initial_state"] if with_state else torch.zeros(
        (N, H, dk, dv), device=DEV)
    return d, state.clone()


@pytest.mark.parametrize("io", ["f32", "bf16"])
@pytest.mark.parametrize("dk,dv", [(32, 32), (64, 64), (128, 128), (32, 128),
                                   (128, 64), (64, 32)])
@pytest.mark.parametrize("T", [1, 5])
def test_small_vs_oracle(io, dk, dv, T):
    N, H = 3, 2
    d, state = _decode_case(N, H, dk, dv, T, io, seed=7 + dk + dv + T)
    s0 = state.clone()
    out = K.recurrent_step(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"],
                           state)
    torch.cuda.synchronize()
    ro, rs = kda_oracle.recurrent(PY.host64(d["q"]), PY.host64(d["k"]),
                                  PY.host64(d["v"]), PY.host64(d["log_alpha"]),
                                  PY.host64(d["beta"]), PY.host64(s0))
    tol = PY.TOL_F32 if io == "f32" else PY.TOL_BF16
    PY.check("out", PY.host64(out), ro, tol)
    PY.check("state", PY.host64(state), rs, tol)


def test_step_by_step_equals_multi_token():
    # T calls of one token each == one call of T tokens (state hand-off).
    N, H, dk, dv, T = 4, 3, 128, 128, 6
    d, state = _decode_case(N, H, dk, dv, T, "f32", seed=11)
    s_a, s_b = state.clone(), state.clone()
    out_a = K.recurrent_step(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"],
                             s_a)
    outs = []
    for t in range(T):
        sl = lambda x: x[:, t:t + 1].contiguous()  # noqa: E731
        outs.append(K.recurrent_step(sl(d["q"]), sl(d["k"]), sl(d["v"]),
                                     sl(d["log_alpha"]), sl(d["beta"]), s_b))
    torch.cuda.synchronize()
    assert torch.allclose(out_a, torch.cat(outs, 1), atol=1e-5, rtol=1e-5)
    assert torch.allclose(s_a, s_b, atol=1e-5, rtol=1e-5)


def test_exact_recall_property():
    # q = k, beta = 1, unit keys: o_t = v_t whatever the state (fp32 io).
    N, H, dk, dv = 8, 4, 128, 128
    d, state = _decode_case(N, H, dk, dv, 1, "f32", seed=12)
    out = K.recurrent_step(d["k"], d["k"], d["v"], d["log_alpha"],
                           torch.ones_like(d["beta"]), state)
    torch.cuda.synchronize()
    assert PY.rel_l2(PY.host64(out), PY.host64(d["v"])) < 1e-5


def test_zero_tokens_keeps_state():
    N, H, dk, dv = 2, 2, 64, 64
    d, state = _decode_case(N, H, dk, dv, 1, "bf16", seed=13)
    s0 = state.clone()
    e = lambda x: x[:, :0].contiguous()  # noqa: E731
    K.recurrent_step(e(d["q"]), e(d["k"]), e(d["v"]), e(d["log_alpha"]),
                     e(d["beta"]), state)
    torch.cuda.synchronize()
    assert torch.equal(state, s0)


def test_config4_full_size_every_element():
    """256 sequences x 32 heads, d = 128, 64 consecutive steps with the state
    updated in place (the benchmarked launch): every output of every step and
    the whole final state against the fp64 oracle run over all 8192
    (sequence, head) units (about a second on 16 host cores)."""
    d = W.make(4, device=DEV)
    cfg = d["cfg"]
    S = cfg["steps"]
    s0 = PY.host64(d["initial_state"])
    state = d["initial_state"]
    outs = []
    for s in range(S):
        outs.append(K.recurrent_step(d["q"][s][:, None], d["k"][s][:, None],
                                     d["v"][s][:, None],
                                     d["log_alpha"][s][:, None],
                                     d["beta"][s][:, None], state))
    torch.cuda.synchronize()
    out = torch.cat(outs, 1)                      # [N, S, H, dv]
    # the oracle sees each sequence's 64 steps as one 64-token sequence
    tr = lambda x: np.ascontiguousarray(np.swapaxes(PY.host64(x), 0, 1))  # noqa: E731
    ro, rs = kda_oracle.recurrent(tr(d["q"]), tr(d["k"]), tr(d["v"]),
                                  tr(d["log_alpha"]), tr(d["beta"]), s0)
    PY.check_units("out", PY.host64(out), ro, PY.TOL_BF16, unit_axes=(0, 2))
    PY.check_units("state", PY.host64(state), rs, PY.TOL_BF16, unit_axes=(0, 1))
