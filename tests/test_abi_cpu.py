"""The C-ABI library on the host: it loads without a GPU, exports every entry
point include/*.h declares, plans without touching a device, and rejects bad
arguments before launching anything (the checks with fake device addresses
run in a child process that sees no GPU; see fake_address_abi.py).  No
compute call is made here."""
import ctypes
import glob
import os
import re

import pytest

from gated_delta_rule_156_b200 import build as kbuild
from gated_delta_rule_156_b200 import kda as K

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    kbuild.build()
    return K.library()


def declared_entry_points():
    names = []
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        src = open(h).read()
        names += re.findall(r"KDA_API\s+[\w\s\*]+?\b(kda_\w+)\s*\(", src)
    return sorted(set(names))


def test_every_declared_symbol_is_exported(lib):
    names = declared_entry_points()
    assert "kda_chunk_fwd" in names and "kda_recurrent_step" in names
    for n in names:
        assert hasattr(lib, n), n
    assert set(K.EXPORTS) <= set(names)


def test_status_strings(lib):
    for code, name in K.STATUS_NAMES.items():
        assert lib.kda_status_string(code).decode().startswith(name)
    assert lib.kda_version() >= 100
    assert lib.kda_last_cuda_error() == 0


def test_fake_address_validation_in_a_process_without_gpus():
    # tests/fake_address_abi.py passes fake device addresses to every entry
    # point and expects host-side rejection; it runs in a child process that
    # sees no GPU, so a validation regression can never launch a kernel
    import subprocess
    import sys
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    r = subprocess.run(
        [sys.executable, "-m", "pytest", "-q", "-p", "no:cacheprovider",
         os.path.join(ROOT, "tests", "fake_address_abi.py")],
        cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout[-4000:] + r.stderr[-2000:]
    assert " passed" in r.stdout and "skipped" not in r.stdout, r.stdout[-2000:]


def test_backward_plan(lib):
    import torch
    kern, ws = K.chunk_bwd_plan(2, 8192, 32, 128, 128, 64, torch.bfloat16)
    # cumsum, prep, the state pass, 2 + 9 products, the chain, final (the
    # tensor-core kernels replace the SIMT ones one for one)
    assert kern == 16 and ws > 0
    kern_f, ws_f = K.chunk_bwd_plan(2, 8192, 32, 128, 128, 64, torch.float32)
    assert kern_f == 16
    # the tensor-core path keeps W^T and the transposed per-chunk copies too,
    # but its arrays share memory where their lifetimes do not overlap: less
    # than the fp32 path, which keeps every array apart, and at least what
    # the reverse chain alone reads and writes (Kb, W^T, Qt^T dO, P^T dO,
    # the chunk-start states, G, dDelta, its transposed copy)
    assert ws < ws_f
    tok, st = 4 * 2 * 8192 * 32 * 128, 4 * 2 * 128 * 32 * 128 * 128
    assert ws >= 5 * tok + 3 * st
    kern_p, _ = K.chunk_bwd_plan(1, 300, 2, 64, 64, 32, torch.float32,
                                 packed=True, n_seqs=3)
    assert kern_p == 17


@pytest.mark.parametrize("B,T,H,dk,dv,packed,n_seqs", [
    (2, 8192, 32, 128, 128, False, 0),   # the prefill workload
    (1, 2048, 4, 64, 64, False, 0),
    (2, 200, 3, 64, 128, False, 0),      # ragged last chunk, d_k != d_v
    (1, 300, 2, 128, 64, True, 3),       # packed layout
])
def test_backward_workspace_layout(lib, B, T, H, dk, dv, packed, n_seqs):
    import torch
    arrays = K.chunk_bwd_layout(B, T, H, dk, dv, 64, torch.bfloat16,
                                packed=packed, n_seqs=n_seqs)
    _, ws = K.chunk_bwd_plan(B, T, H, dk, dv, 64, torch.bfloat16,
                             packed=packed, n_seqs=n_seqs)
    assert len(arrays) > 20
    assert max(o + b for o, b, _, _ in arrays) <= ws
    for o, b, f, l in arrays:
        assert o % 256 == 0 and b > 0 and 0 <= f <= l
    # arrays whose launch ranges overlap never share a byte
    for i, (oi, bi, fi, li) in enumerate(arrays):
        for oj, bj, fj, lj in arrays[i + 1:]:
            if fi <= lj and fj <= li:
                assert oi + bi <= oj or oj + bj <= oi, (i, oi, bi, oj, bj)
    # and the packing does share memory: the arrays' sum exceeds the workspace
    assert sum(b for _, b, _, _ in arrays) > ws
    # the fp32 path keeps every array apart and reports none
    assert K.chunk_bwd_layout(B, T, H, dk, dv, 64, torch.float32,
                              packed=packed, n_seqs=n_seqs) == []


def test_split_plan(lib):
    import torch
    # plan: segments of ceil(chunks / n) chunks; the kernels are the setup,
    # the value run (order, chunk offsets, factorisation, chain on the
    # two-pass packed path), the transition run (order, chunk offsets and a
    # chain over the value run's packages), scan and fix
    seg, kern, ws = K.chunk_fwd_split_plan(131072, 8, 128, 128, 64,
                                           torch.bfloat16, 4)
    assert seg == 4 and kern == 1 + 4 + 3 + 2 and ws > 0
    # the fp32 path runs both four-stage pipelines in full
    seg32, kern32, _ = K.chunk_fwd_split_plan(131072, 8, 128, 128, 64,
                                              torch.float32, 4)
    assert seg32 == 4 and kern32 > kern
    seg, kern, ws = K.chunk_fwd_split_plan(1000, 2, 64, 64, 64,
                                           torch.float32, 7)
    assert seg == 6  # 16 chunks in segments of 3
    # bf16 with d in {64, 128}: segments rounded up to 128-token tiles
    # (3 chunks = 192 tokens -> 256), so 4 segments
    seg, kern, ws = K.chunk_fwd_split_plan(1000, 2, 64, 64, 64,
                                           torch.bfloat16, 7)
    assert seg == 4
    seg, kern, ws = K.chunk_fwd_split_plan(100, 2, 64, 64, 64,
                                           torch.bfloat16, 1)
    assert seg == 1 and kern == 2 and ws > 0  # the two-pass path itself
    # n_segments = 0 picks the largest k with (2k - 1) chains of H x (width
    # / 64) CTAs within the SMs: H = 8, d = 128 -> 16 CTAs a chain -> k = 5;
    # H = 32 -> 64 a chain -> 1 (not split)
    assert K.chunk_fwd_split_plan(131072, 8, 128, 128, 64, torch.bfloat16, 0,
                                  num_sms=148)[0] == 5
    assert K.chunk_fwd_split_plan(131072, 32, 128, 128, 64, torch.bfloat16, 0,
                                  num_sms=148)[0] == 1
    assert K.chunk_fwd_split_plan(131072, 4, 64, 64, 64, torch.bfloat16, 0,
                                  num_sms=148)[0] == 19


C_CALLER = r"""
#include <stdio.h>
#include "kda.h"
int main(void) {
  kda_shape s = {1, 64, 2, 48, 64, 64, 0, KDA_BF16};  /* d_k = 48 */
  int kern = 0, path = 0, seg = 0;
  size_t ws = 0;
  if (kda_version() < 100) return 1;
  if (kda_chunk_fwd_plan(&s, 0, 0, &path, &kern, &ws) != KDA_ERR_UNSUPPORTED)
    return 2;
  s.dk = 128;
  s.dv = 128;
  s.T = 131072;
  s.H = 8;
  if (kda_chunk_fwd_split_plan(&s, KDA_GATE_CHANNEL, 0, 148, &seg, &kern, &ws)
      != KDA_OK || seg != 5)
    return 3;
  printf("%s\n", kda_status_string(KDA_OK));
  return 0;
}
"""


@pytest.mark.skipif(__import__("shutil").which("gcc") is None, reason="needs gcc")
def test_plain_c_caller_links_and_runs(lib, tmp_path):
    # the boundary is a C ABI: a C99 program includes include/kda.h, links
    # libkda.so and calls its host-side entry points (no GPU needed)
    import subprocess
    from torch.utils.cpp_extension import CUDA_HOME
    cuda_inc = os.path.join(CUDA_HOME or "/usr/local/cuda", "include")
    src = tmp_path / "caller.c"
    src.write_text(C_CALLER)
    libdir = os.path.join(ROOT, "gated_delta_rule_156_b200")
    exe = tmp_path / "caller"
    subprocess.check_call(
        ["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
         "-I", cuda_inc, str(src), "-L", libdir, "-lkda",
         "-Wl,-rpath," + libdir, "-o", str(exe)])
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert out.returncode == 0, (out.returncode, out.stdout, out.stderr)
    assert out.stdout.startswith("KDA_OK")
