"""The per-head forget gate (Gated DeltaNet) and no gate (DeltaNet) layouts of
kda_chunk_fwd_gated / kda_recurrent_step_gated, against the fp64 oracle run
on the equivalent per-channel gate (broadcast over d_k, or zeros)."""
import pytest
import torch

import kda_workloads as W
import parity as PY
from gated_delta_rule_156_b200 import kda as K
from oracle import kda_oracle

pytestmark = pytest.mark.gpu
DEV = "cuda"


def gates(d, mode, seed):
    """(gate tensor for the call, equivalent per-channel log(alpha))."""
    shape_h = d["beta"].shape
    if mode == "none":
        return None, torch.zeros_like(d["log_alpha"])
    g = torch.Generator(device=DEV).manual_seed(seed)
    lh = torch.nn.functional.logsigmoid(
        torch.randn(shape_h, generator=g, device=DEV)) / 16
    return lh.contiguous(), lh[..., None].expand_as(d["log_alpha"]).contiguous()


def oracle_of(d, la_full):
    return kda_oracle.recurrent(PY.host64(d["q"]), PY.host64(d["k"]),
                                PY.host64(d["v"]), PY.host64(la_full),
                                PY.host64(d["beta"]),
                                None if d["initial_state"] is None
                                else PY.host64(d["initial_state"]))


@pytest.mark.parametrize("mode", ["head", "none"])
@pytest.mark.parametrize("io,dk,dv,C,staged", [
    ("bf16", 128, 128, 64, False), ("bf16", 64, 64, 64, False),
    ("bf16", 128, 64, 64, True), ("f32", 64, 64, 32, True),
    ("f32", 32, 32, 16, False)])
def test_chunk_gate_modes(mode, io, dk, dv, C, staged):
    d = W.draw((2, 150), 3, dk, dv, io=io, n_states=2, device=DEV, seed=dk + C)
    lg, la_full = gates(d, mode, seed=5)
    out, fin = K.chunk_fwd(d["q"], d["k"], d["v"], lg, d["beta"],
                           d["initial_state"], None, chunk=C, staged=staged,
                           gate=mode)
    torch.cuda.synchronize()
    ro, rs = oracle_of(d, la_full)
    tol = PY.TOL_F32 if io == "f32" else PY.TOL_BF16
    PY.check("out", PY.host64(out), ro, tol)
    PY.check("final", PY.host64(fin), rs, tol)
    # the same kernels fed the broadcast per-channel gate agree closely
    o2, f2 = K.chunk_fwd(d["q"], d["k"], d["v"], la_full, d["beta"],
                         d["initial_state"], None, chunk=C, staged=staged)
    torch.cuda.synchronize()
    PY.check("vs channel gate", PY.host64(out), PY.host64(o2), 1e-3)
    PY.check("vs channel gate state", PY.host64(fin), PY.host64(f2), 1e-3)


@pytest.mark.parametrize("mode", ["head", "none"])
def test_chunk_gate_modes_packed(mode):
    lengths = [100, 0, 64, 7]
    T = sum(lengths)
    d = W.draw((1, T), 2, 128, 128, io="bf16", n_states=4, device=DEV, seed=77)
    lg, la_full = gates(d, mode, seed=6)
    offs = [0]
    for n in lengths:
        offs.append(offs[-1] + n)
    cu = torch.tensor(offs, dtype=torch.int32, device=DEV)
    out, fin = K.chunk_fwd(d["q"], d["k"], d["v"], lg, d["beta"],
                           d["initial_state"], cu, chunk=64, gate=mode)
    torch.cuda.synchronize()
    ro, rs = kda_oracle.recurrent(PY.host64(d["q"][0]), PY.host64(d["k"][0]),
                                  PY.host64(d["v"][0]), PY.host64(la_full[0]),
                                  PY.host64(d["beta"][0]),
                                  PY.host64(d["initial_state"]), seq_offsets=offs)
    PY.check("out", PY.host64(out[0]), ro, PY.TOL_BF16)
    PY.check("final", PY.host64(fin), rs, PY.TOL_BF16)


@pytest.mark.parametrize("mode", ["head", "none"])
@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_decode_gate_modes(mode, io):
    d = W.draw((4, 3), 2, 128, 128, io=io, n_states=4, device=DEV, seed=9)
    lg, la_full = gates(d, mode, seed=7)
    state = d["initial_state"].clone()
    out = K.recurrent_step(d["q"], d["k"], d["v"], lg, d["beta"], state,
                           gate=mode)
    torch.cuda.synchronize()
    ro, rs = oracle_of(d, la_full)
    tol = PY.TOL_F32 if io == "f32" else PY.TOL_BF16
    PY.check("out", PY.host64(out), ro, tol)
    PY.check("state", PY.host64(state), rs, tol)


def test_kimi_layer_head_gate_full_size_sampled():
    """The Kimi-Linear-shaped workload with a per-head gate on the fused path,
    sampled units against the oracle."""
    d = W.make(2, device=DEV)
    lg, _ = gates(d, "head", seed=8)
    out, fin = K.chunk_fwd(d["q"], d["k"], d["v"], lg, d["beta"], None, None,
                           chunk=64, gate="head")
    torch.cuda.synchronize()
    units = [(0, 0), (1, 31), (0, 17)]
    la = lg[..., None].expand_as(d["log_alpha"])
    ref = PY.oracle_units(d["q"], d["k"], d["v"], la, d["beta"], None, units)
    for (s, h), (o, f) in ref.items():
        PY.check(f"out[{s},{h}]", PY.host64(out[s, :, h]), o, PY.TOL_BF16)
        PY.check(f"final[{s},{h}]", PY.host64(fin[s, h]), f, PY.TOL_BF16)
