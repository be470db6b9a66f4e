"""kda_chunk_fwd / kda_chunk_fwd_staged (chunkwise prefill) against the fp64
oracle: the small named configs in full, ragged and packed inputs, edge cases,
and the large configs on sampled (sequence, head) units."""
import numpy as np
import pytest
import torch

import kda_workloads as W
import parity as PY
from gated_delta_rule_156_b200 import kda as K
from oracle import kda_oracle

pytestmark = pytest.mark.gpu
DEV = "cuda"
PATHS = ["auto", "staged"]


def run(d, path, chunk, initial_state="from_d", cu=None, final_state=None):
    s0 = d["initial_state"] if initial_state == "from_d" else initial_state
    return K.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], s0,
                       cu, chunk=chunk, staged=(path == "staged"),
                       final_state=final_state)


def tol(d):
    return PY.TOL_F32 if d["q"].dtype == torch.float32 else PY.TOL_BF16


@pytest.mark.parametrize("path", PATHS)
def test_config0_tiny_fp32(path):
    d = W.make(0, device=DEV)
    out, fin = run(d, path, d["cfg"]["chunk"])
    torch.cuda.synchronize()
    ro, rs = PY.oracle_dense(d)
    PY.check("out", PY.host64(out), ro, PY.TOL_F32)
    PY.check("final", PY.host64(fin), rs, PY.TOL_F32)
    # the first 8 tokens also against the brute-force product form
    bo, bs = kda_oracle.brute_force(*(PY.host64(d[x][0, :8, 0]) for x in
                                      ("q", "k", "v", "log_alpha", "beta")))
    PY.check("out[:8] vs brute force", PY.host64(out[0, :8, 0]), bo, PY.TOL_F32)


@pytest.mark.parametrize("path", PATHS)
def test_config1_small_bf16(path):
    d = W.make(1, device=DEV)
    out, fin = run(d, path, d["cfg"]["chunk"])
    torch.cuda.synchronize()
    ro, rs = PY.oracle_dense(d)
    PY.check("out", PY.host64(out), ro, PY.TOL_BF16)
    PY.check("final", PY.host64(fin), rs, PY.TOL_BF16)


@pytest.mark.parametrize("path", PATHS)
@pytest.mark.parametrize("io", ["f32", "bf16"])
@pytest.mark.parametrize("dk,dv,C,T", [(32, 32, 16, 77), (64, 64, 64, 200),
                                       (128, 128, 64, 333), (64, 128, 32, 100),
                                       (128, 32, 16, 50), (128, 64, 64, 64)])
def test_ragged_dense(path, io, dk, dv, C, T):
    d = W.draw((2, T), 3, dk, dv, io=io, n_states=2, device=DEV,
               seed=dk * 7 + dv + C + T)
    out, fin = run(d, path, C)
    torch.cuda.synchronize()
    ro, rs = PY.oracle_dense(d)
    PY.check("out", PY.host64(out), ro, tol(d))
    PY.check("final", PY.host64(fin), rs, tol(d))


@pytest.mark.parametrize("path", PATHS)
@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_packed_varlen_with_empty_and_ragged(path, io):
    lengths = [5, 0, 64, 130, 1, 200, 63]
    H, dk, dv = 2, 64, 64
    T = sum(lengths)
    d = W.draw((1, T), H, dk, dv, io=io, n_states=len(lengths), device=DEV,
               seed=31)
    offs = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)
    cu = torch.tensor(offs, dtype=torch.int32, device=DEV)
    out = torch.full((1, T, H, dv), float("nan"), dtype=d["q"].dtype, device=DEV)
    out, fin = K.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"],
                           d["initial_state"], cu, chunk=64, out=out,
                           staged=(path == "staged"))
    torch.cuda.synchronize()
    ro, rs = kda_oracle.recurrent(PY.host64(d["q"][0]), PY.host64(d["k"][0]),
                                  PY.host64(d["v"][0]),
                                  PY.host64(d["log_alpha"][0]),
                                  PY.host64(d["beta"][0]),
                                  PY.host64(d["initial_state"]), seq_offsets=offs)
    PY.check("out", PY.host64(out[0]), ro, tol(d))
    PY.check("final", PY.host64(fin), rs, tol(d))
    # the empty sequence hands its initial state through unchanged
    assert torch.equal(fin[1], d["initial_state"][1])


@pytest.mark.parametrize("path", PATHS)
def test_zero_length_and_none_state(path):
    d = W.draw((2, 0), 2, 64, 64, io="bf16", n_states=2, device=DEV, seed=3)
    _, fin = run(d, path, 64)
    torch.cuda.synchronize()
    assert torch.equal(fin, d["initial_state"])
    d = W.draw((1, 0), 2, 64, 64, io="bf16", n_states=None, device=DEV, seed=3)
    _, fin = run(d, path, 64)
    torch.cuda.synchronize()
    assert torch.count_nonzero(fin) == 0


@pytest.mark.parametrize("path", PATHS)
def test_state_handoff_and_in_place(path):
    # one call over T == two calls joined by the state (T1 not a chunk
    # multiple; the second call updates the state in place)
    d = W.draw((1, 300), 2, 128, 128, io="bf16", n_states=1, device=DEV, seed=5)
    out, fin = run(d, path, 64)
    part = lambda x, a, b: x[:, a:b].contiguous()  # noqa: E731
    d1 = {k_: part(d[k_], 0, 137) for k_ in ("q", "k", "v", "log_alpha", "beta")}
    d2 = {k_: part(d[k_], 137, 300) for k_ in ("q", "k", "v", "log_alpha", "beta")}
    state = d["initial_state"].clone()
    o1, _ = K.chunk_fwd(d1["q"], d1["k"], d1["v"], d1["log_alpha"], d1["beta"],
                        state, None, chunk=64, final_state=state,
                        staged=(path == "staged"))
    o2, _ = K.chunk_fwd(d2["q"], d2["k"], d2["v"], d2["log_alpha"], d2["beta"],
                        state, None, chunk=64, final_state=state,
                        staged=(path == "staged"))
    torch.cuda.synchronize()
    ro, rs = PY.oracle_dense(d)
    split = PY.host64(torch.cat([o1, o2], 1))
    PY.check("split out vs oracle", split, ro, PY.TOL_BF16)
    PY.check("split state vs oracle", PY.host64(state), rs, PY.TOL_BF16)
    PY.check("one call out vs oracle", PY.host64(out), ro, PY.TOL_BF16)
    PY.check("split vs one call", split, PY.host64(out), PY.TOL_BF16)


@pytest.mark.parametrize("path", PATHS)
def test_chunk_size_invariance_fp32(path):
    d = W.draw((1, 256), 2, 64, 64, io="f32", n_states=1, device=DEV, seed=9)
    outs = [run(d, path, C) for C in (16, 32, 64)]
    torch.cuda.synchronize()
    for o, f in outs[1:]:
        PY.check("out", PY.host64(o), PY.host64(outs[0][0]), 1e-5)
        PY.check("final", PY.host64(f), PY.host64(outs[0][1]), 1e-5)


@pytest.mark.parametrize("path", PATHS)
def test_exact_recall_fp32(path):
    # q = k, beta = 1, unit keys: o_t = v_t at any size.
    d = W.draw((2, 512), 4, 128, 128, io="f32", n_states=2, device=DEV, seed=10)
    out, _ = K.chunk_fwd(d["k"], d["k"], d["v"], d["log_alpha"],
                         torch.ones_like(d["beta"]), d["initial_state"], None,
                         chunk=64, staged=(path == "staged"))
    torch.cuda.synchronize()
    PY.check("recall", PY.host64(out), PY.host64(d["v"]), 1e-4)


@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 64), (64, 128), (128, 64)])
def test_bf16_takes_fused_path(dk, dv):
    # the two-pass tensor-core evaluation: factorisation pass + chain kernel
    path, kernels, ws = K.chunk_fwd_plan(1, 128, 2, dk, dv, 64, torch.bfloat16)
    assert path == "twopass" and kernels == 2 and ws > 0
    d = W.draw((2, 130), 2, dk, dv, io="bf16", n_states=2, device=DEV, seed=dk + dv)
    out, fin = run(d, "auto", 64)
    assert K.device_status() == 0
    ro, rs = PY.oracle_dense(d)
    PY.check("out", PY.host64(out), ro, PY.TOL_BF16)
    PY.check("final", PY.host64(fin), rs, PY.TOL_BF16)


_ORACLE = {}


def _oracle_config2(d):
    """The fp64 oracle over the whole B=2, T=8192, H=32, d=128 input (about a
    second on 16 host cores), computed once for both paths."""
    if 2 not in _ORACLE:
        _ORACLE[2] = PY.oracle_dense(d)
    return _ORACLE[2]


@pytest.mark.parametrize("path", PATHS)
def test_config2_full_size_every_element(path):
    d = W.make(2, device=DEV)
    out, fin = run(d, path, 64)
    torch.cuda.synchronize()
    assert K.device_status() == 0
    ro, rs = _oracle_config2(d)
    # every element, bounded as a whole and per (sequence, head)
    PY.check_units("out", PY.host64(out), ro, PY.TOL_BF16, unit_axes=(0, 2))
    PY.check_units("final", PY.host64(fin), rs, PY.TOL_BF16, unit_axes=(0, 1))


def _oracle_config3(d):
    """The oracle over the whole packed batch (16 sequences + one of 131072
    tokens, H = 32, d = 128), in two groups of 16 heads to bound host memory;
    about 20 s on 16 host cores.  Computed once for both paths."""
    if 3 not in _ORACLE:
        offs = [0]
        for n in d["lengths"]:
            offs.append(offs[-1] + n)
        H = d["q"].shape[2]
        outs, fins = [], []
        for h0 in range(0, H, 16):
            sl = (0, slice(None), slice(h0, h0 + 16))
            o, f = kda_oracle.recurrent(
                PY.host64(d["q"][sl]), PY.host64(d["k"][sl]),
                PY.host64(d["v"][sl]), PY.host64(d["log_alpha"][sl]),
                PY.host64(d["beta"][sl]),
                PY.host64(d["initial_state"][:, h0:h0 + 16]), seq_offsets=offs)
            outs.append(o)
            fins.append(f)
        _ORACLE[3] = (np.concatenate(outs, axis=1), np.concatenate(fins, axis=1),
                      offs)
    return _ORACLE[3]


@pytest.mark.parametrize("path", PATHS)
def test_config3_packed_long_every_element(path):
    d = W.make(3, device=DEV)
    out, fin = run(d, path, 64, cu=d["cu_seqlens"])
    torch.cuda.synchronize()
    assert K.device_status() == 0
    ro, rs, offs = _oracle_config3(d)
    got = PY.host64(out[0])                       # [T_total, H, d_v]
    PY.check_units("out", got, ro, PY.TOL_BF16, unit_axes=(1,))
    # per (sequence, head) over every sequence's tokens, the long one too
    for s in range(len(offs) - 1):
        sl = slice(offs[s], offs[s + 1])
        PY.check_units(f"out seq {s}", got[sl], ro[sl], PY.TOL_BF16,
                       unit_axes=(1,))
    PY.check_units("final", PY.host64(fin), rs, PY.TOL_BF16, unit_axes=(0, 1))
