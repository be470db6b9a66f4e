"""kda_chunk_fwd_split (one long sequence as segments evaluated side by side,
joined by a scan of their state transitions) against the fp64 oracle: the
fused path (bf16, d = 64 / 128) and the four-stage path (fp32), every gate
layout, segment counts from 2 up to more than the sequence has chunks, a
ragged last chunk, and n_segments = 1, which must equal kda_chunk_fwd bit
for bit."""
import pytest
import torch

import kda_workloads as W
import parity as PY
from gated_delta_rule_156_b200 import kda as K

pytestmark = pytest.mark.gpu
DEV = "cuda"


def case(T, H, dk, dv, io, seed, state=True):
    return W.draw((1, T), H, dk, dv, io=io, n_states=1 if state else None,
                  device=DEV, seed=seed)


def against_oracle(d, out, fin, tol, la_full=None):
    dd = dict(d)
    if la_full is not None:
        dd["log_alpha"] = la_full
    ro, rs = PY.oracle_dense(dd)
    PY.check("out", PY.host64(out), ro, tol)
    PY.check("final", PY.host64(fin), rs, tol)


@pytest.mark.parametrize("n", [2, 3, 4, 7])
def test_split_fused_d128(n):
    # 1000 tokens = 15 full chunks and a ragged one
    d = case(1000, 2, 128, 128, "bf16", seed=10 + n)
    out, fin = K.chunk_fwd_split(d["q"], d["k"], d["v"], d["log_alpha"],
                                 d["beta"], d["initial_state"], n_segments=n)
    assert K.device_status() == 0
    against_oracle(d, out, fin, PY.TOL_BF16)


@pytest.mark.parametrize("dk,dv", [(64, 64), (64, 128), (128, 64)])
def test_split_fused_dims(dk, dv):
    d = case(777, 3, dk, dv, "bf16", seed=dk + dv)
    out, fin = K.chunk_fwd_split(d["q"], d["k"], d["v"], d["log_alpha"],
                                 d["beta"], d["initial_state"], n_segments=3)
    against_oracle(d, out, fin, PY.TOL_BF16)


@pytest.mark.parametrize("dk,dv,C", [(64, 64, 32), (32, 128, 16), (128, 32, 64)])
def test_split_staged_fp32(dk, dv, C):
    d = case(613, 2, dk, dv, "f32", seed=C + dk)
    out, fin = K.chunk_fwd_split(d["q"], d["k"], d["v"], d["log_alpha"],
                                 d["beta"], d["initial_state"], n_segments=4,
                                 chunk=C)
    against_oracle(d, out, fin, PY.TOL_F32)


@pytest.mark.parametrize("gate", ["head", "none"])
def test_split_gate_layouts(gate):
    d = case(700, 2, 128, 128, "bf16", seed=31)
    if gate == "none":
        lg, la_full = None, torch.zeros_like(d["log_alpha"])
    else:
        g = torch.Generator(device=DEV).manual_seed(5)
        lg = torch.nn.functional.logsigmoid(
            torch.randn(d["beta"].shape, generator=g, device=DEV)) / 16
        la_full = lg[..., None].expand_as(d["log_alpha"]).contiguous()
    out, fin = K.chunk_fwd_split(d["q"], d["k"], d["v"], lg, d["beta"],
                                 d["initial_state"], n_segments=3, gate=gate)
    against_oracle(d, out, fin, PY.TOL_BF16, la_full=la_full)


def test_split_one_segment_is_chunk_fwd():
    d = case(500, 2, 128, 128, "bf16", seed=2)
    o1, f1 = K.chunk_fwd_split(d["q"], d["k"], d["v"], d["log_alpha"],
                               d["beta"], d["initial_state"], n_segments=1)
    o2, f2 = K.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"],
                         d["initial_state"])
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(f1, f2)


def test_split_more_segments_than_chunks_and_short():
    # 3 chunks asked to split 10 ways: one-chunk segments, rounded up to the
    # 128-token tiles of the tensor-core correction (bf16, d = 64), so two
    # segments; a sequence shorter than one chunk is not split at all
    for T, n in ((150, 10), (40, 4)):
        d = case(T, 2, 64, 64, "bf16", seed=T)
        out, fin = K.chunk_fwd_split(d["q"], d["k"], d["v"], d["log_alpha"],
                                     d["beta"], d["initial_state"], n_segments=n)
        against_oracle(d, out, fin, PY.TOL_BF16)
    assert K.chunk_fwd_split_plan(150, 2, 64, 64, 64, torch.bfloat16, 10)[0] == 2
    assert K.chunk_fwd_split_plan(150, 2, 64, 64, 64, torch.float32, 10)[0] == 3
    assert K.chunk_fwd_split_plan(40, 2, 64, 64, 64, torch.bfloat16, 4)[0] == 1


def test_split_without_initial_state_long():
    # a longer single sequence, zero start state, 8 segments of 16 chunks
    d = case(8192, 2, 128, 128, "bf16", seed=8, state=False)
    out, fin = K.chunk_fwd_split(d["q"], d["k"], d["v"], d["log_alpha"],
                                 d["beta"], None, n_segments=8)
    against_oracle(d, out, fin, PY.TOL_BF16)
    # and it matches the unsplit prefill to the same tolerance
    o2, f2 = K.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"],
                         None)
    PY.check("out vs unsplit", PY.host64(out), PY.host64(o2), PY.TOL_BF16)
    PY.check("final vs unsplit", PY.host64(fin), PY.host64(f2), PY.TOL_BF16)


def test_split_auto_segment_count():
    # n_segments = 0: the library picks the count from the SM count (two
    # heads of d = 128 leave most SMs idle, so it splits)
    d = case(4000, 2, 128, 128, "bf16", seed=44)
    n_sms = torch.cuda.get_device_properties(0).multi_processor_count
    seg = K.chunk_fwd_split_plan(4000, 2, 128, 128, 64, torch.bfloat16, 0,
                                 num_sms=n_sms)[0]
    assert seg > 1
    out, fin = K.chunk_fwd_split(d["q"], d["k"], d["v"], d["log_alpha"],
                                 d["beta"], d["initial_state"], n_segments=0)
    assert K.device_status() == 0
    against_oracle(d, out, fin, PY.TOL_BF16)


@pytest.mark.parametrize("dk,dv,C", [(64, 128, 32), (32, 128, 16), (128, 32, 64)])
def test_split_bf16_other_paths(dk, dv, C):
    # bf16 io off the fused path (C < 64, or d = 32): the value and transition
    # runs take the four-stage pipeline; the correction runs on the tensor
    # cores when d_k, d_v are in {64, 128} (first case) and in fp32 otherwise
    d = case(613, 2, dk, dv, "bf16", seed=dk + dv + C)
    out, fin = K.chunk_fwd_split(d["q"], d["k"], d["v"], d["log_alpha"],
                                 d["beta"], d["initial_state"], n_segments=3,
                                 chunk=C)
    assert K.device_status() == 0
    against_oracle(d, out, fin, PY.TOL_BF16)
