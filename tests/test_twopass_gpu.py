"""kda_chunk_fwd_twopass (a parallel factorisation pass over every
(chunk, head), then the chain kernel) against the fp64 oracle: ragged and
packed inputs with empty sequences, both key widths and both value widths,
every gate layout, the input prologue, strong gates, and the B=2, T=8192,
H=32, d=128 layer in full; and against the one-kernel path."""
import math

import numpy as np
import pytest
import torch

import kda_workloads as W
import parity as PY
from gated_delta_rule_156_b200 import kda as K
from oracle import kda_oracle

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.mark.parametrize("dk,dv,T", [(128, 128, 333), (64, 64, 200),
                                     (64, 128, 64), (128, 64, 130),
                                     (128, 128, 5)])
def test_twopass_ragged_dense(dk, dv, T):
    d = W.draw((2, T), 3, dk, dv, io="bf16", n_states=2, device=DEV,
               seed=dk + dv + T)
    out, fin = K.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"],
                           d["initial_state"], None, chunk=64, twopass=True)
    assert K.device_status() == 0
    ro, rs = PY.oracle_dense(d)
    PY.check("out", PY.host64(out), ro, PY.TOL_BF16)
    PY.check("final", PY.host64(fin), rs, PY.TOL_BF16)
    # the one-kernel path agrees closely (same bf16 operands, other order)
    o1, f1 = K.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"],
                         d["initial_state"], None, chunk=64)
    PY.check("vs fused out", PY.host64(out), PY.host64(o1), 2e-3)
    PY.check("vs fused final", PY.host64(fin), PY.host64(f1), 2e-3)


def test_twopass_packed_with_empty_and_ragged():
    lengths = [300, 0, 77, 1, 200, 64]
    d = W.draw((1, sum(lengths)), 2, 128, 128, io="bf16",
               n_states=len(lengths), device=DEV, seed=31)
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lengths)]),
                      dtype=torch.int32, device=DEV)
    out, fin = K.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"],
                           d["initial_state"], cu, chunk=64, twopass=True)
    assert K.device_status() == 0
    offs = [0] + list(np.cumsum(lengths))
    ro, rs = kda_oracle.recurrent(*(PY.host64(d[n][0]) for n in
                                    ("q", "k", "v", "log_alpha", "beta")),
                                  PY.host64(d["initial_state"]),
                                  seq_offsets=offs)
    PY.check("out", PY.host64(out[0]), ro, PY.TOL_BF16)
    PY.check("final", PY.host64(fin), rs, PY.TOL_BF16)


@pytest.mark.parametrize("path", ["twopass", "paired"])
def test_prefill_is_deterministic(path):
    # two calls on the same packed input agree bit for bit (both prefill
    # paths reduce in a fixed order; a difference can only come from a race)
    lengths = [300, 0, 77, 1, 200, 64, 650]
    d = W.draw((1, sum(lengths)), 4, 128, 128, io="bf16",
               n_states=len(lengths), device=DEV, seed=33)
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lengths)]),
                      dtype=torch.int32, device=DEV)
    runs = []
    for _ in range(3):
        out, fin = K.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"],
                               d["beta"], d["initial_state"], cu, chunk=64,
                               **{path: True})
        torch.cuda.synchronize()
        runs.append((out.clone(), fin.clone()))
    assert K.device_status() == 0
    for o, f in runs[1:]:
        assert torch.equal(o, runs[0][0]) and torch.equal(f, runs[0][1])


@pytest.mark.parametrize("mode", ["head", "none"])
def test_twopass_gate_layouts(mode):
    d = W.draw((2, 150), 3, 128, 128, io="bf16", n_states=2, device=DEV, seed=5)
    if mode == "none":
        lg, la_full = None, torch.zeros_like(d["log_alpha"])
    else:
        g = torch.Generator(device=DEV).manual_seed(6)
        lg = (torch.nn.functional.logsigmoid(
            torch.randn(d["beta"].shape, generator=g, device=DEV)) / 16).contiguous()
        la_full = lg[..., None].expand_as(d["log_alpha"]).contiguous()
    out, fin = K.chunk_fwd(d["q"], d["k"], d["v"], lg, d["beta"],
                           d["initial_state"], None, chunk=64, gate=mode,
                           twopass=True)
    ro, rs = kda_oracle.recurrent(*(PY.host64(x) for x in (
        d["q"], d["k"], d["v"], la_full, d["beta"], d["initial_state"])))
    PY.check("out", PY.host64(out), ro, PY.TOL_BF16)
    PY.check("final", PY.host64(fin), rs, PY.TOL_BF16)


def test_twopass_prologue_and_strong_gate():
    g = torch.Generator(device=DEV).manual_seed(8)
    B, T, H, d = 1, 300, 2, 128
    q = torch.randn((B, T, H, d), generator=g, device=DEV).bfloat16()
    k = torch.randn((B, T, H, d), generator=g, device=DEV).bfloat16()
    v = torch.randn((B, T, H, d), generator=g, device=DEV).bfloat16()
    x = torch.randn((B, T, H, d), generator=g, device=DEV)
    beta = torch.sigmoid(torch.randn((B, T, H), generator=g, device=DEV))
    s0 = torch.randn((B, H, d, d), generator=g, device=DEV) * 0.1
    pro = dict(normalize_qk=True, q_scale=d ** -0.5, gate_logits=True,
               gate_scale=1.0)   # undivided logsigmoid: a strong gate
    out, fin = K.chunk_fwd(q, k, v, x, beta, s0, None, chunk=64,
                           prologue=pro, twopass=True)
    assert K.device_status() == 0
    qn, kn, la = kda_oracle.prologue(PY.host64(q), PY.host64(k), PY.host64(x),
                                     normalize_qk=True, q_scale=d ** -0.5,
                                     gate_logits=True, gate_scale=1.0)
    ro, rs = kda_oracle.recurrent(qn, kn, PY.host64(v), la, PY.host64(beta),
                                  PY.host64(s0))
    PY.check("out", PY.host64(out), ro, PY.TOL_BF16)
    PY.check("final", PY.host64(fin), rs, PY.TOL_BF16)
    # the pages' 0.2 gate held on a channel for 160 tokens
    dd = W.draw((1, 400), 2, 128, 128, io="bf16", n_states=1, device=DEV,
                seed=9, gate_divisor=1.0)
    dd["log_alpha"][0, 50:210, :, 4] = math.log(0.2)
    out, fin = K.chunk_fwd(dd["q"], dd["k"], dd["v"], dd["log_alpha"],
                           dd["beta"], dd["initial_state"], None, chunk=64,
                           twopass=True)
    assert K.device_status() == 0
    ro, rs = PY.oracle_dense(dd)
    PY.check("alpha 0.2 out", PY.host64(out), ro, PY.TOL_BF16)
    PY.check("alpha 0.2 final", PY.host64(fin), rs, PY.TOL_BF16)


def test_twopass_config2_every_element():
    d = W.make(2, device=DEV)
    out, fin = K.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"],
                           None, None, chunk=64, twopass=True)
    torch.cuda.synchronize()
    assert K.device_status() == 0
    ro, rs = PY.oracle_dense(d)
    PY.check_units("out", PY.host64(out), ro, PY.TOL_BF16, unit_axes=(0, 2))
    PY.check_units("final", PY.host64(fin), rs, PY.TOL_BF16, unit_axes=(0, 1))


def test_twopass_unsupported_shapes_rejected():
    d = W.draw((1, 64), 1, 32, 32, io="bf16", n_states=1, device=DEV, seed=1)
    with pytest.raises(K.KdaError):
        K.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"],
                    d["initial_state"], None, chunk=64, twopass=True)


@pytest.mark.gpu
def test_pass_event_times_the_two_passes_apart():
    """kda_profile_pass_event: an event recorded between the factorisation
    pass and the chain kernel splits the call's time into two positive
    parts that add up to the whole."""
    d = W.make(2, device="cuda")
    out = torch.empty(d["v"].shape, dtype=torch.bfloat16, device="cuda")
    fin = torch.empty((2, 32, 128, 128), dtype=torch.float32, device="cuda")
    e0, mid, e1 = (torch.cuda.Event(enable_timing=True) for _ in range(3))
    mid.record()
    K.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], None, None,
                chunk=64, out=out, final_state=fin)
    e0.record()
    K.profile_pass_event(mid)
    try:
        K.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], None,
                    None, chunk=64, out=out, final_state=fin)
    finally:
        K.profile_pass_event(None)
    e1.record()
    torch.cuda.synchronize()
    a, b, whole = e0.elapsed_time(mid), mid.elapsed_time(e1), e0.elapsed_time(e1)
    assert a > 0 and b > 0
    assert abs(a + b - whole) <= 1e-3 * whole + 1e-3
    with pytest.raises(ValueError):
        K.profile_pass_event(torch.cuda.Event())  # never recorded
