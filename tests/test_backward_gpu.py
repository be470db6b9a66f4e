"""kda_chunk_bwd (the chunkwise backward pass) against the oracle's fp64
reverse-mode gradients of the token recurrence, for every gradient: dq, dk,
dv, dlog_alpha, dbeta and the initial-state gradient."""
import numpy as np
import pytest
import torch

import kda_workloads as W
import parity as PY
from gated_delta_rule_156_b200 import kda as K
from oracle import kda_oracle

pytestmark = pytest.mark.gpu
DEV = "cuda"
NAMES = ("dq", "dk", "dv", "dlog_alpha", "dbeta", "d_initial_state")


def grads_in(d, seed, with_final=True):
    g = torch.Generator(device=DEV).manual_seed(seed)
    do = torch.randn(d["v"].shape, generator=g, device=DEV).to(d["v"].dtype)
    dsT = None
    if with_final:
        n = d["initial_state"].shape[0] if d["initial_state"] is not None else \
            d["q"].shape[0]
        H, dk, dv = d["q"].shape[2], d["q"].shape[3], d["v"].shape[3]
        dsT = torch.randn((n, H, dk, dv), generator=g, device=DEV)
    return do, dsT


def compare(got, ref, tol):
    for name, x, r in zip(NAMES, got, ref):
        if x is None:
            continue
        PY.check(name, PY.host64(x).reshape(r.shape), r, tol)


@pytest.mark.parametrize("io", ["f32", "bf16"])
@pytest.mark.parametrize("dk,dv,C,T", [(32, 32, 16, 77), (64, 64, 32, 150),
                                       (128, 128, 64, 130), (64, 128, 64, 200),
                                       (128, 64, 64, 150), (64, 64, 64, 64),
                                       (128, 32, 16, 40)])
def test_backward_dense(io, dk, dv, C, T):
    d = W.draw((2, T), 2, dk, dv, io=io, n_states=2, device=DEV,
               seed=dk + dv + C + T)
    do, dsT = grads_in(d, seed=T)
    got = K.chunk_bwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"],
                      d["initial_state"], None, do, dsT, chunk=C)
    torch.cuda.synchronize()
    ref = kda_oracle.recurrent_bwd(*(PY.host64(d[n]) for n in
                                     ("q", "k", "v", "log_alpha", "beta",
                                      "initial_state")),
                                   PY.host64(do), PY.host64(dsT))
    compare(got, ref, PY.TOL_F32 if io == "f32" else PY.TOL_BF16)


@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_backward_packed_with_empty_and_short(io):
    lengths = [5, 0, 64, 1, 130, 63]
    T = sum(lengths)
    d = W.draw((1, T), 2, 64, 64, io=io, n_states=len(lengths), device=DEV,
               seed=77)
    offs = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)
    cu = torch.tensor(offs, dtype=torch.int32, device=DEV)
    do, dsT = grads_in(d, seed=78)
    got = K.chunk_bwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"],
                      d["initial_state"], cu, do, dsT, chunk=64)
    torch.cuda.synchronize()
    ref = kda_oracle.recurrent_bwd(*(PY.host64(d[n][0]) for n in
                                     ("q", "k", "v", "log_alpha", "beta")),
                                   PY.host64(d["initial_state"]),
                                   PY.host64(do[0]), PY.host64(dsT),
                                   seq_offsets=offs)
    compare(got, ref, PY.TOL_F32 if io == "f32" else PY.TOL_BF16)
    # the empty sequence passes its state gradient straight through
    assert torch.equal(got[5][1], dsT[1])


@pytest.mark.parametrize("io,C", [("f32", 32), ("bf16", 64)])
def test_backward_without_states(io, C):
    # no initial state (zeros) and no final-state gradient; bf16 in 64-token
    # chunks takes the tensor-core path
    d = W.draw((1, 100), 3, 64, 64, io=io, n_states=None, device=DEV, seed=5)
    do, _ = grads_in(d, seed=6, with_final=False)
    got = K.chunk_bwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], None,
                      None, do, None, chunk=C)
    torch.cuda.synchronize()
    ref = kda_oracle.recurrent_bwd(*(PY.host64(d[n]) for n in
                                     ("q", "k", "v", "log_alpha", "beta")),
                                   None, PY.host64(do), None)
    compare(got, ref, PY.TOL_F32 if io == "f32" else PY.TOL_BF16)


def test_backward_config2_sampled():
    # the Kimi-Linear-shaped layer (B=2, T=8192, H=32, d=128, bf16) on
    # sampled (sequence, head) units
    d = W.make(2, device=DEV)
    do, dsT = grads_in(d, seed=9)
    got = K.chunk_bwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], None,
                      None, do, dsT, chunk=64)
    torch.cuda.synchronize()
    for s, h in [(0, 0), (1, 31), (0, 17)]:
        def unit(x):  # one (sequence, head) of a [B, T, H, ...] tensor
            return x[s:s + 1, :, h:h + 1]
        ref = kda_oracle.recurrent_bwd(
            *(PY.host64(unit(d[n])) for n in ("q", "k", "v", "log_alpha", "beta")),
            None, PY.host64(unit(do)), PY.host64(dsT[s:s + 1, h:h + 1]))
        mine = [unit(x) for x in got[:5]] + [got[5][s:s + 1, h:h + 1]]
        compare(mine, ref, PY.TOL_BF16)


@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_backward_is_deterministic(io):
    # two calls on the same inputs agree bit for bit: every kernel of the
    # backward (the tensor-core ones included) reduces in a fixed order, so a
    # difference can only come from a race
    lengths = [130, 64, 5, 200]
    T = sum(lengths)
    d = W.draw((1, T), 3, 128, 128, io=io, n_states=len(lengths), device=DEV,
               seed=91)
    offs = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)
    cu = torch.tensor(offs, dtype=torch.int32, device=DEV)
    do, dsT = grads_in(d, seed=92)
    runs = []
    for _ in range(3):
        got = K.chunk_bwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"],
                          d["initial_state"], cu, do, dsT, chunk=64)
        torch.cuda.synchronize()
        runs.append([x.clone() for x in got if x is not None])
    for later in runs[1:]:
        for name, a, b in zip(NAMES, runs[0], later):
            assert torch.equal(a, b), f"{name} differs between two calls"
