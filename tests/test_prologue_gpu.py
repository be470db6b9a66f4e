"""The in-kernel input prologue (kda_chunk_fwd_ex / kda_recurrent_step_ex):
q and k L2-normalised per token and head, q scaled, and the gate given as raw
logits with log(alpha) = scale * logsigmoid(x).  Checked against the fp64
oracle's plain prologue followed by the recurrence."""
import math

import pytest
import torch

import parity as PY
from gated_delta_rule_156_b200 import kda as K
from oracle import kda_oracle

pytestmark = pytest.mark.gpu
DEV = "cuda"


def raw_inputs(B, T, H, dk, dv, io, gate, seed, states=True):
    g = torch.Generator(device=DEV).manual_seed(seed)
    dt = torch.bfloat16 if io == "bf16" else torch.float32
    r = lambda *s: torch.randn(s, generator=g, device=DEV)  # noqa: E731
    d = dict(q=(2.0 * r(B, T, H, dk)).to(dt), k=(0.5 * r(B, T, H, dk)).to(dt),
             v=r(B, T, H, dv).to(dt), beta=torch.sigmoid(r(B, T, H)),
             initial_state=0.1 * r(B, H, dk, dv) if states else None)
    d["gate"] = (r(B, T, H, dk) if gate == "channel" else
                 r(B, T, H) if gate == "head" else None)
    return d


def reference(d, pro, gate):
    qn, kn, la = kda_oracle.prologue(
        PY.host64(d["q"]), PY.host64(d["k"]),
        None if d["gate"] is None else PY.host64(d["gate"]),
        normalize_qk=pro["normalize_qk"], q_scale=pro["q_scale"],
        gate_logits=pro["gate_logits"], gate_scale=pro["gate_scale"])
    if la is None:
        la = torch.zeros(d["q"].shape, dtype=torch.float64).numpy()
    elif gate == "head":
        la = la[..., None].repeat(qn.shape[-1], axis=-1)
    return kda_oracle.recurrent(qn, kn, PY.host64(d["v"]), la,
                                PY.host64(d["beta"]),
                                None if d["initial_state"] is None
                                else PY.host64(d["initial_state"]))


PRO = dict(normalize_qk=True, q_scale=1 / math.sqrt(128), gate_logits=True,
           gate_scale=1 / 16)


@pytest.mark.parametrize("gate", ["channel", "head", "none"])
@pytest.mark.parametrize("io,dk,C,staged", [("bf16", 128, 64, False),
                                            ("bf16", 64, 64, False),
                                            ("bf16", 128, 64, True),
                                            ("f32", 64, 32, True)])
def test_chunk_prologue(gate, io, dk, C, staged):
    d = raw_inputs(2, 140, 2, dk, dk, io, gate, seed=dk + C)
    pro = dict(PRO, q_scale=1 / math.sqrt(dk))
    out, fin = K.chunk_fwd(d["q"], d["k"], d["v"], d["gate"], d["beta"],
                           d["initial_state"], None, chunk=C, staged=staged,
                           gate=gate, prologue=pro)
    torch.cuda.synchronize()
    ro, rs = reference(d, pro, gate)
    tol = PY.TOL_F32 if io == "f32" else PY.TOL_BF16
    PY.check("out", PY.host64(out), ro, tol)
    PY.check("final", PY.host64(fin), rs, tol)


@pytest.mark.parametrize("pro", [dict(normalize_qk=False, q_scale=0.5,
                                      gate_logits=False, gate_scale=1.0),
                                 dict(normalize_qk=True, q_scale=1.0,
                                      gate_logits=False, gate_scale=1.0)])
def test_chunk_prologue_partial_options(pro):
    d = raw_inputs(1, 100, 2, 128, 128, "bf16", "channel", seed=3)
    d["gate"] = torch.nn.functional.logsigmoid(d["gate"]) / 16  # log(alpha)
    if not pro["normalize_qk"]:  # keep the keys unit-norm: a valid KDA input
        d["k"] = (d["k"].float() / d["k"].float().norm(dim=-1, keepdim=True)
                  ).to(torch.bfloat16)
    out, fin = K.chunk_fwd(d["q"], d["k"], d["v"], d["gate"], d["beta"],
                           d["initial_state"], None, chunk=64, prologue=pro)
    torch.cuda.synchronize()
    ro, rs = reference(d, pro, "channel")
    PY.check("out", PY.host64(out), ro, PY.TOL_BF16)
    PY.check("final", PY.host64(fin), rs, PY.TOL_BF16)


@pytest.mark.parametrize("gate", ["channel", "head"])
@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_decode_prologue(gate, io):
    d = raw_inputs(4, 3, 2, 128, 128, io, gate, seed=11)
    pro = dict(PRO)
    state = d["initial_state"].clone()
    out = K.recurrent_step(d["q"], d["k"], d["v"], d["gate"], d["beta"], state,
                           gate=gate, prologue=pro)
    torch.cuda.synchronize()
    ro, rs = reference(d, pro, gate)
    tol = PY.TOL_F32 if io == "f32" else PY.TOL_BF16
    PY.check("out", PY.host64(out), ro, tol)
    PY.check("state", PY.host64(state), rs, tol)
