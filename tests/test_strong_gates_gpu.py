"""Strong forget gates on every chunkwise path, against the fp64 oracle.

The chunkwise form factorises the decay inside a chunk into one factor per
row and one per column.  Gates far stronger than the named configs' (whose
decay over a 64-token chunk is about 3 per channel) must still give the
recurrence's result:
  - the undivided logsigmoid(N(0, 1)) gate: about 52 per channel over a
    64-token chunk;
  - the per-channel decay worked example's strong gate, alpha = 0.2 ("Teacher
    guide - Kimi Delta Attention", section 12.1 and the Misconceptions table:
    the gate that flushes a channel), held on a few channels for 160 tokens:
    about 103 over a chunk;
  - alpha = exp(-2.4) held for a whole chunk: 153.6, just inside the
    supported range.
A decay beyond the range (192 over one chunk, e.g. alpha = exp(-3) for 64
tokens) is not supported; the call must not fault and kda_device_status must report
KDA_ERR_RANGE."""
import math

import numpy as np
import pytest
import torch

import kda_workloads as W
import parity as PY
from gated_delta_rule_156_b200 import kda as K

pytestmark = pytest.mark.gpu
DEV = "cuda"
KDA_OK, KDA_ERR_RANGE = 0, 6

# (io, dk, dv, chunk, staged): the fused kernels (cluster pair at d_v = 128,
# single CTA at d_v = 64) and the four-stage pipeline, fp32 and bf16
PATHS = [("bf16", 128, 128, 64, False), ("bf16", 64, 64, 64, False),
         ("bf16", 64, 128, 64, False), ("bf16", 128, 64, 64, False),
         ("bf16", 128, 128, 64, True), ("f32", 64, 64, 64, True),
         ("f32", 32, 32, 16, True), ("f32", 64, 32, 32, True)]


def inputs(kind, io, dk, dv, seed, chunk=64):
    d = W.draw((2, 300), 2, dk, dv, io=io, n_states=2, device=DEV, seed=seed,
               gate_divisor=1.0 if kind == "logsigmoid" else 16.0)
    la = d["log_alpha"]
    if kind == "alpha0.2":
        # channels 0, 5 and dk - 1 of every head forget at 0.2 per token for
        # tokens 40 .. 199 (across chunk boundaries) of both sequences
        for c in (0, 5, dk - 1):
            la[:, 40:200, :, c] = math.log(0.2)
    elif kind == "edge":
        # one channel at exp(-2.4) for tokens 64 .. 127: 153.6 in one chunk
        la[:, 64:128, :, 3] = -2.4
    elif kind == "beyond":
        # 192 per chunk at any chunk length: tokens 64 .. 127 hold whole chunks
        la[:, 64:128, :, 3] = -192.0 / chunk
    return d


@pytest.mark.parametrize("kind", ["logsigmoid", "alpha0.2", "edge"])
@pytest.mark.parametrize("io,dk,dv,C,staged", PATHS)
def test_strong_gates_match_oracle(kind, io, dk, dv, C, staged):
    if kind == "edge" and C != 64:
        pytest.skip("the edge case is one 64-token chunk")
    d = inputs(kind, io, dk, dv, seed=7 + dk + dv + C)
    assert K.device_status() == KDA_OK
    out, fin = K.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"],
                           d["initial_state"], None, chunk=C, staged=staged)
    assert K.device_status() == KDA_OK
    ro, rs = PY.oracle_dense(d)
    tol = PY.TOL_F32 if io == "f32" else PY.TOL_BF16
    PY.check(f"{kind} out", PY.host64(out), ro, tol)
    PY.check(f"{kind} final", PY.host64(fin), rs, tol)


@pytest.mark.parametrize("io,dk,dv,C,staged", PATHS)
def test_decay_beyond_range_is_reported(io, dk, dv, C, staged):
    d = inputs("beyond", io, dk, dv, seed=3, chunk=C)
    K.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"],
                d["initial_state"], None, chunk=C, staged=staged)
    assert K.device_status() == KDA_ERR_RANGE
    assert K.device_status() == KDA_OK  # reading the status cleared it
    # the context stays usable: an ordinary call matches the oracle
    d = W.draw((1, 130), 2, dk, dv, io=io, n_states=1, device=DEV, seed=4)
    out, fin = K.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"],
                           d["initial_state"], None, chunk=C, staged=staged)
    ro, rs = PY.oracle_dense(d)
    tol = PY.TOL_F32 if io == "f32" else PY.TOL_BF16
    PY.check("after out", PY.host64(out), ro, tol)
    assert K.device_status() == KDA_OK


def test_strong_gate_packed_and_split():
    # a packed batch and the sequence split with the strong gate
    lengths = [300, 0, 77, 200]
    d = W.draw((1, sum(lengths)), 2, 128, 128, io="bf16",
               n_states=len(lengths), device=DEV, seed=11, gate_divisor=1.0)
    d["log_alpha"][0, 10:150, :, 7] = math.log(0.2)
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lengths)]),
                      dtype=torch.int32, device=DEV)
    out, fin = K.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"],
                           d["initial_state"], cu, chunk=64)
    assert K.device_status() == KDA_OK
    offs = [0] + list(np.cumsum(lengths))
    ref = PY.oracle_units(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"],
                          d["initial_state"],
                          [(s, h) for s in range(len(lengths)) for h in range(2)],
                          offsets=offs)
    for (s, h), (ro, rs) in ref.items():
        if lengths[s]:
            PY.check(f"packed out {s},{h}",
                     PY.host64(out[0, offs[s]:offs[s + 1], h]), ro, PY.TOL_BF16)
        PY.check(f"packed final {s},{h}", PY.host64(fin[s, h]), rs, PY.TOL_BF16)
    ds = W.draw((1, 700), 2, 128, 128, io="bf16", n_states=1, device=DEV,
                seed=12, gate_divisor=1.0)
    ds["log_alpha"][0, 100:400, :, 1] = math.log(0.2)
    o2, f2 = K.chunk_fwd_split(ds["q"], ds["k"], ds["v"], ds["log_alpha"],
                               ds["beta"], ds["initial_state"], n_segments=3)
    assert K.device_status() == KDA_OK
    ro, rs = PY.oracle_dense(ds)
    PY.check("split out", PY.host64(o2), ro, PY.TOL_BF16)
    PY.check("split final", PY.host64(f2), rs, PY.TOL_BF16)


def test_backward_strong_gate_and_range():
    from oracle import kda_oracle
    # the undivided logsigmoid gate (|g_C| about 52) is inside the backward's
    # range; the 0.2 gate held for a chunk (about 103) is reported
    d = W.draw((1, 150), 2, 64, 64, io="f32", n_states=1, device=DEV, seed=21,
               gate_divisor=1.0)
    g = torch.Generator(device=DEV).manual_seed(22)
    do = torch.randn(d["v"].shape, generator=g, device=DEV)
    dsT = torch.randn(d["initial_state"].shape, generator=g, device=DEV)
    got = K.chunk_bwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"],
                      d["initial_state"], None, do, dsT, chunk=32)
    assert K.device_status() == KDA_OK
    ref = kda_oracle.recurrent_bwd(*(PY.host64(x) for x in (
        d["q"], d["k"], d["v"], d["log_alpha"], d["beta"],
        d["initial_state"], do, dsT)))
    for name, x, r in zip(("dq", "dk", "dv", "dla", "db", "ds0"), got, ref):
        PY.check(name, PY.host64(x).reshape(r.shape), r, PY.TOL_F32)
    d["log_alpha"][0, 0:64, :, 2] = math.log(0.2)
    K.chunk_bwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"],
                d["initial_state"], None, do, dsT, chunk=64)
    assert K.device_status() == KDA_ERR_RANGE
    assert K.device_status() == KDA_OK


def test_backward_tensor_core_path_strong_gate_and_range():
    from oracle import kda_oracle
    # bf16 inputs in 64-token chunks take the tensor-core backward (the
    # two-pass state pass, tf32 prep, chain and products): the undivided
    # logsigmoid gate against the oracle, and the 0.2 gate held for a chunk
    # reported as out of range
    d = W.draw((2, 150), 2, 128, 128, io="bf16", n_states=2, device=DEV,
               seed=23, gate_divisor=1.0)
    g = torch.Generator(device=DEV).manual_seed(24)
    do = torch.randn(d["v"].shape, generator=g, device=DEV).bfloat16()
    dsT = torch.randn(d["initial_state"].shape, generator=g, device=DEV)
    got = K.chunk_bwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"],
                      d["initial_state"], None, do, dsT, chunk=64)
    assert K.device_status() == KDA_OK
    ref = kda_oracle.recurrent_bwd(*(PY.host64(x) for x in (
        d["q"], d["k"], d["v"], d["log_alpha"], d["beta"],
        d["initial_state"], do, dsT)))
    for name, x, r in zip(("dq", "dk", "dv", "dla", "db", "ds0"), got, ref):
        PY.check(name, PY.host64(x).reshape(r.shape), r, PY.TOL_BF16)
    d["log_alpha"][0, 64:128, :, 5] = math.log(0.2)
    K.chunk_bwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"],
                d["initial_state"], None, do, dsT, chunk=64)
    assert K.device_status() == KDA_ERR_RANGE
    assert K.device_status() == KDA_OK
