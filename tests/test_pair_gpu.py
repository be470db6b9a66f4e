"""The tensor-core prefill paths on the chunk counts that exercise their
hand-overs: sequences with no chunk, one chunk, two and three chunks, and
longer ones with a ragged tail; for both key widths, every gate layout and
the input prologue, against the fp64 oracle.  Each test runs both
evaluations: the paired one-kernel path (kda_chunk_fwd_paired: the two
64-column tiles of a head run as a 2-CTA cluster and factorise alternate
chunks; the second CTA of a one-chunk sequence factorises nothing, and with
two or three chunks the first sends before the peer has anything to
release) and the two-pass default (kda_chunk_fwd: the factorisation pass
writes one package per (chunk, head), the chain kernel reads them)."""
import numpy as np
import pytest
import torch

import kda_workloads as W
import parity as PY
from gated_delta_rule_156_b200 import kda as K
from oracle import kda_oracle

pytestmark = pytest.mark.gpu
DEV = "cuda"
LENGTHS = [1, 63, 64, 65, 0, 127, 128, 129, 191, 192, 193, 320, 383, 2]


def packed(dk, seed, io="bf16"):
    T = sum(LENGTHS)
    d = W.draw((1, T), 3, dk, 128, io=io, n_states=len(LENGTHS), device=DEV,
               seed=seed)
    offs = np.concatenate([[0], np.cumsum(LENGTHS)]).astype(np.int64)
    d["offs"] = offs
    d["cu"] = torch.tensor(offs, dtype=torch.int32, device=DEV)
    return d


def oracle_packed(d, la_full):
    return kda_oracle.recurrent(PY.host64(d["q"][0]), PY.host64(d["k"][0]),
                                PY.host64(d["v"][0]), PY.host64(la_full[0]),
                                PY.host64(d["beta"][0]),
                                PY.host64(d["initial_state"]),
                                seq_offsets=d["offs"])


PATHS = ["paired", "twopass"]


def call(path, *args, **kw):
    return K.chunk_fwd(*args, paired=(path == "paired"), **kw)


@pytest.mark.parametrize("dk", [128, 64])
def test_default_path_is_twopass(dk):
    # order and chunk offsets of the packed layout, the factorisation pass,
    # the chain kernel
    path, kernels, ws = K.chunk_fwd_plan(1, sum(LENGTHS), 3, dk, 128, 64,
                                         torch.bfloat16, packed=True,
                                         n_seqs=len(LENGTHS))
    assert path == "twopass" and kernels == 4 and ws > 0


@pytest.mark.parametrize("path", PATHS)
@pytest.mark.parametrize("dk", [128, 64])
def test_pair_packed_chunk_counts(dk, path):
    d = packed(dk, seed=100 + dk)
    out, fin = call(path, d["q"], d["k"], d["v"], d["log_alpha"], d["beta"],
                    d["initial_state"], d["cu"], chunk=64)
    assert K.device_status() == 0
    ro, rs = oracle_packed(d, d["log_alpha"])
    PY.check("out", PY.host64(out[0]), ro, PY.TOL_BF16)
    PY.check("final", PY.host64(fin), rs, PY.TOL_BF16)
    # the empty sequence hands its state through untouched
    assert torch.equal(fin[4], d["initial_state"][4])


@pytest.mark.parametrize("path", PATHS)
@pytest.mark.parametrize("mode", ["head", "none"])
def test_pair_gate_layouts(mode, path):
    d = packed(128, seed=7)
    if mode == "none":
        lg, la_full = None, torch.zeros_like(d["log_alpha"])
    else:
        g = torch.Generator(device=DEV).manual_seed(11)
        lg = (torch.nn.functional.logsigmoid(
            torch.randn(d["beta"].shape, generator=g, device=DEV)) / 16)
        la_full = lg[..., None].expand_as(d["log_alpha"]).contiguous()
    out, fin = call(path, d["q"], d["k"], d["v"], lg, d["beta"],
                    d["initial_state"], d["cu"], chunk=64, gate=mode)
    assert K.device_status() == 0
    ro, rs = oracle_packed(d, la_full)
    PY.check("out", PY.host64(out[0]), ro, PY.TOL_BF16)
    PY.check("final", PY.host64(fin), rs, PY.TOL_BF16)


@pytest.mark.parametrize("path", PATHS)
def test_pair_prologue(path):
    # raw (unnormalised) q, k and gate logits; the kernel normalises, scales
    # q by 1/sqrt(d_k) and maps the logits to log(alpha) = logsigmoid(x) / 16
    d = packed(128, seed=21)
    g = torch.Generator(device=DEV).manual_seed(3)
    q_raw = (torch.randn(d["q"].shape, generator=g, device=DEV) * 3).to(torch.bfloat16)
    k_raw = (torch.randn(d["k"].shape, generator=g, device=DEV) * 3).to(torch.bfloat16)
    logits = torch.randn(d["log_alpha"].shape, generator=g, device=DEV)
    pro = dict(normalize_qk=True, q_scale=128 ** -0.5, gate_logits=True,
               gate_scale=1.0 / 16)
    out, fin = call(path, q_raw, k_raw, d["v"], logits, d["beta"],
                    d["initial_state"], d["cu"], chunk=64, prologue=pro)
    assert K.device_status() == 0
    qn, kn, la = kda_oracle.prologue(PY.host64(q_raw), PY.host64(k_raw),
                                     PY.host64(logits), normalize_qk=True,
                                     q_scale=128 ** -0.5, gate_logits=True,
                                     gate_scale=1.0 / 16)
    ro, rs = kda_oracle.recurrent(qn[0], kn[0], PY.host64(d["v"][0]), la[0],
                                  PY.host64(d["beta"][0]),
                                  PY.host64(d["initial_state"]),
                                  seq_offsets=d["offs"])
    PY.check("out", PY.host64(out[0]), ro, PY.TOL_BF16)
    PY.check("final", PY.host64(fin), rs, PY.TOL_BF16)


@pytest.mark.parametrize("path", PATHS)
@pytest.mark.parametrize("T", [64, 128, 192])
def test_pair_dense_short(T, path):
    # one, two and three chunks per sequence, no cu_seqlens
    d = W.draw((3, T), 2, 128, 128, io="bf16", n_states=3, device=DEV, seed=T)
    out, fin = call(path, d["q"], d["k"], d["v"], d["log_alpha"], d["beta"],
                    d["initial_state"], None, chunk=64)
    assert K.device_status() == 0
    ro, rs = PY.oracle_dense(d)
    PY.check("out", PY.host64(out), ro, PY.TOL_BF16)
    PY.check("final", PY.host64(fin), rs, PY.TOL_BF16)


@pytest.mark.parametrize("path", PATHS)
def test_pair_is_deterministic(path):
    # no atomics and a fixed hand-over order: two runs agree bit for bit
    d = packed(128, seed=5)
    runs = [call(path, d["q"], d["k"], d["v"], d["log_alpha"], d["beta"],
                 d["initial_state"], d["cu"], chunk=64) for _ in range(2)]
    torch.cuda.synchronize()
    assert torch.equal(runs[0][0], runs[1][0])
    assert torch.equal(runs[0][1], runs[1][1])
