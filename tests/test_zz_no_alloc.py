"""kda_chunk_fwd_staged_noalloc: the entry point for callers that must not
allocate device memory during a call (for example a plugin whose host engine
owns and pre-plans all device memory, or a serving loop that may not stall on
an allocator).  It runs the four-stage pipeline with its workspace in the
library's fixed device array; its results must equal those of
kda_chunk_fwd_staged, which allocates its workspace per call.

This file is collected last on purpose, so a stop-at-first-failure run has
already run every other test before these.  The size limit is checked on
the host; that check is exercised in fake_address_abi.py, in a process that
sees no GPU."""
import numpy as np
import pytest
import torch

import kda_workloads as W
import parity as PY
from gated_delta_rule_156_b200 import kda as K

DEV = "cuda"


def _cases():
    # (inputs, chunk, tolerance): the tiny fp32 config, the small bf16
    # config, and a packed batch with an empty and ragged sequences.
    yield "config0-fp32", W.make(0, device=DEV), 16, None, PY.TOL_F32
    yield "config1-bf16", W.make(1, device=DEV), 64, None, PY.TOL_BF16
    lengths = [70, 0, 128, 5]
    d = W.draw((1, sum(lengths)), 2, 64, 64, io="bf16", n_states=len(lengths),
               device=DEV, seed=77)
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lengths)]),
                      dtype=torch.int32, device=DEV)
    yield "packed-bf16", d, 64, cu, PY.TOL_BF16


@pytest.mark.gpu
def test_noalloc_matches_allocating_entry_point_twice():
    for name, d, C, cu, tol in _cases():
        ref_o, ref_s = K.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"],
                                   d["beta"], d["initial_state"], cu, chunk=C,
                                   staged=True)
        _, _, ws = K.chunk_fwd_plan(d["q"].shape[0], d["q"].shape[1],
                                    d["q"].shape[2], d["q"].shape[3],
                                    d["v"].shape[3], C, d["q"].dtype,
                                    packed=cu is not None,
                                    n_seqs=0 if cu is None else cu.numel() - 1,
                                    staged=True)
        assert ws <= K.NOALLOC_SCRATCH_BYTES, (name, ws)
        for call in range(2):  # two calls in a row share the scratch array
            out = torch.full_like(ref_o, float("nan"))
            fin = torch.full_like(ref_s, float("nan"))
            K.chunk_fwd_noalloc(d["q"], d["k"], d["v"], d["log_alpha"],
                                d["beta"], d["initial_state"], cu, chunk=C,
                                out=out, final_state=fin)
            torch.cuda.synchronize()
            PY.check(f"{name} call {call} out", PY.host64(out),
                     PY.host64(ref_o), tol)
            PY.check(f"{name} call {call} state", PY.host64(fin),
                     PY.host64(ref_s), tol)
