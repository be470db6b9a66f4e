"""The C-ABI library on the host: it loads without a GPU, exports every entry
point include/*.h declares, and rejects bad arguments before launching
anything (no compute call is made here)."""
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


# Fake device addresses: validation rejects before any CUDA call is made.
A = 0x7000_0000_0000


def _p(i):
    return ctypes.c_void_p(A + i * 0x1000_0000)


def shape(**kw):
    d = dict(B=1, T=64, H=2, dk=64, dv=64, chunk=64, n_seqs=0, io_dtype=0)
    d.update(kw)
    return K.KdaShape(**d)


def chunk_call(lib, s, q=1, k=2, v=3, la=4, b=5, s0=6, cu=None, out=7, sf=8,
               fn="kda_chunk_fwd"):
    P = lambda i: None if i is None else (ctypes.c_void_p(i) if isinstance(i, int) and i > 1000 else _p(i))  # noqa: E731
    return getattr(lib, fn)(None if s is None else ctypes.byref(s), P(q), P(k),
                            P(v), P(la), P(b), P(s0), P(cu), P(out), P(sf), None)


@pytest.mark.parametrize("fn", ["kda_chunk_fwd", "kda_chunk_fwd_staged"])
def test_chunk_validation(lib, fn):
    INV, UNS, MIS = 1, 2, 3
    assert chunk_call(lib, None, fn=fn) == INV
    assert chunk_call(lib, shape(H=0), fn=fn) == INV
    assert chunk_call(lib, shape(T=-1), fn=fn) == INV
    assert chunk_call(lib, shape(io_dtype=7), fn=fn) == INV
    assert chunk_call(lib, shape(dk=96), fn=fn) == UNS
    assert chunk_call(lib, shape(dv=256), fn=fn) == UNS
    assert chunk_call(lib, shape(chunk=128), fn=fn) == UNS
    assert chunk_call(lib, shape(), q=None, fn=fn) == INV
    assert chunk_call(lib, shape(), sf=None, fn=fn) == INV
    assert chunk_call(lib, shape(), out=A + 3 * 0x1000_0000 + 2, fn=fn) == MIS
    assert chunk_call(lib, shape(), la=A + 4 * 0x1000_0000 + 8, fn=fn) == MIS
    assert chunk_call(lib, shape(), b=A + 5 * 0x1000_0000 + 2, fn=fn) == MIS
    # out aliasing an input
    assert chunk_call(lib, shape(), out=1, fn=fn) == INV
    # final state overlapping (but not equal to) the initial state
    assert chunk_call(lib, shape(), sf=A + 6 * 0x1000_0000 + 16, fn=fn) == INV
    # packed layout needs B == 1 and n_seqs >= 1
    assert chunk_call(lib, shape(B=2, n_seqs=2), cu=9, fn=fn) == INV
    assert chunk_call(lib, shape(n_seqs=0), cu=9, fn=fn) == INV


def test_recurrent_validation(lib):
    INV, UNS, MIS = 1, 2, 3

    def call(s, q=1, k=2, v=3, la=4, b=5, st=6, out=7):
        P = lambda i: None if i is None else (ctypes.c_void_p(i) if i > 1000 else _p(i))  # noqa: E731
        return lib.kda_recurrent_step(None if s is None else ctypes.byref(s),
                                      P(q), P(k), P(v), P(la), P(b), P(st),
                                      P(out), None)

    assert call(None) == INV
    assert call(shape(H=0)) == INV
    assert call(shape(dk=48)) == UNS
    assert call(shape(), st=None) == INV
    assert call(shape(), v=None) == INV
    assert call(shape(), q=A + 0x1000_0000 + 4) == MIS
    assert call(shape(), out=6) == INV          # out aliases the state
    assert call(shape(), st=2) == INV           # state aliases k


def test_gated_validation(lib):
    INV, MIS = 1, 3

    def call(s, gate, la=4, **kw):
        P = lambda i: None if i is None else (ctypes.c_void_p(i) if i > 1000 else _p(i))  # noqa: E731
        args = dict(q=1, k=2, v=3, b=5, s0=6, cu=None, out=7, sf=8)
        args.update(kw)
        return lib.kda_chunk_fwd_gated(
            ctypes.byref(s), gate, P(args["q"]), P(args["k"]), P(args["v"]),
            P(la), P(args["b"]), P(args["s0"]), P(args["cu"]), P(args["out"]),
            P(args["sf"]), 0, None)

    assert call(shape(), 3) == INV                 # unknown gate layout
    assert call(shape(), -1) == INV
    assert call(shape(), 0, la=None) == INV        # channel gate needs a tensor
    assert call(shape(), 1, la=None) == INV        # head gate needs a tensor
    # a per-head gate needs only 4-byte alignment, a per-channel one 16
    assert call(shape(), 0, la=A + 4 * 0x1000_0000 + 4) == MIS
    assert call(shape(), 1, la=A + 4 * 0x1000_0000 + 2) == MIS
    # the out buffer may not overlap a per-head gate either
    assert call(shape(), 1, la=A + 7 * 0x1000_0000 + 64) == INV

    def step(s, gate, la=4):
        P = lambda i: None if i is None else (ctypes.c_void_p(i) if i > 1000 else _p(i))  # noqa: E731
        return lib.kda_recurrent_step_gated(
            ctypes.byref(s), gate, P(1), P(2), P(3), P(la), P(5), P(6), P(7),
            None)

    assert step(shape(), 5) == INV
    assert step(shape(), 1, la=None) == INV
    assert step(shape(), 0, la=A + 4 * 0x1000_0000 + 8) == MIS


def test_prologue_validation(lib):
    pro = K.KdaPrologue(1, float("nan"), 1, 1.0)
    s = shape()
    P = lambda i: None if i is None else _p(i)  # noqa: E731
    st = lib.kda_chunk_fwd_ex(ctypes.byref(s), 0, ctypes.byref(pro), P(1), P(2),
                              P(3), P(4), P(5), P(6), None, P(7), P(8), 0, None)
    assert st == 1  # NaN scale rejected before any launch
    st = lib.kda_recurrent_step_ex(ctypes.byref(s), 0, ctypes.byref(pro), P(1),
                                   P(2), P(3), P(4), P(5), P(6), P(7), None)
    assert st == 1


def bwd_call(lib, s, **kw):
    """kda_chunk_bwd with fake, disjoint addresses; keyword overrides take a
    slot index (an address) or None."""
    names = ["q", "k", "v", "la", "b", "s0", "cu", "do", "dsT", "dq", "dk",
             "dv", "dla", "db", "ds0"]
    slots = {n: i + 1 for i, n in enumerate(names)}
    slots["cu"] = None
    slots.update(kw)
    args = [_p(slots[n]) if isinstance(slots[n], int) else slots[n]
            for n in names]
    return lib.kda_chunk_bwd(ctypes.byref(s), *args, None)


INVALID, UNSUPPORTED, MISALIGNED = 1, 2, 3


def test_backward_validation(lib):
    # unsupported sizes, missing tensors, misalignment and overlapping
    # outputs are all rejected before any launch
    assert bwd_call(lib, shape(dk=48)) == UNSUPPORTED
    assert bwd_call(lib, shape(chunk=128)) == UNSUPPORTED
    assert bwd_call(lib, shape(), dq=None) == INVALID
    assert bwd_call(lib, shape(), la=None) == INVALID
    assert bwd_call(lib, shape(), do=None) == INVALID
    bad = ctypes.c_void_p(A + 0x1000_0000 + 8)
    assert bwd_call(lib, shape(), dk=bad) == MISALIGNED
    odd = ctypes.c_void_p(A + 3 * 0x1000_0000 + 2)
    assert bwd_call(lib, shape(), db=odd) == MISALIGNED
    # an output over an input, or over another output
    assert bwd_call(lib, shape(), dq=1) == INVALID
    assert bwd_call(lib, shape(), dv=10) == INVALID
    # the packed layout needs B == 1 and n_seqs >= 1
    assert bwd_call(lib, shape(B=2, n_seqs=2), cu=7) == INVALID


def test_backward_plan(lib):
    import torch
    kern, ws = K.chunk_bwd_plan(2, 8192, 32, 128, 128, 64, torch.bfloat16)
    # cumsum, prep, the state pass, 2 + 9 products, the chain, final
    assert kern == 16 and ws > 0
    kern_p, _ = K.chunk_bwd_plan(1, 300, 2, 64, 64, 32, torch.float32,
                                 packed=True, n_seqs=3)
    assert kern_p == 17


def split_call(lib, s, gate=0, n=2, **kw):
    """kda_chunk_fwd_split with fake, disjoint addresses."""
    names = ["q", "k", "v", "la", "b", "s0", "out", "sf"]
    slots = {nm: i + 1 for i, nm in enumerate(names)}
    slots.update(kw)
    args = [_p(slots[nm]) if isinstance(slots[nm], int) else slots[nm]
            for nm in names]
    return lib.kda_chunk_fwd_split(ctypes.byref(s), gate, *args, n, None)


def test_split_validation_and_plan(lib):
    import torch
    # one dense sequence only, and 1 .. 64 segments
    assert split_call(lib, shape(B=2)) == INVALID
    assert split_call(lib, shape(), n=-1) == INVALID
    assert split_call(lib, shape(), n=65) == INVALID
    assert split_call(lib, shape(dk=48)) == UNSUPPORTED
    assert split_call(lib, shape(), out=None) == INVALID
    assert split_call(lib, shape(), out=1) == INVALID       # out over q
    bad = ctypes.c_void_p(A + 0x1000_0000 + 8)
    assert split_call(lib, shape(), q=bad) == MISALIGNED
    assert split_call(lib, shape(), gate=7) == INVALID
    # plan: segments of ceil(chunks / n) chunks; the kernels are the setup,
    # both runs (two launches each on the fused packed path), scan and fix
    seg, kern, ws = K.chunk_fwd_split_plan(131072, 8, 128, 128, 64,
                                           torch.bfloat16, 4)
    assert seg == 4 and kern == 1 + 2 + 2 + 2 and ws > 0
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
    assert (seg, kern, ws) == (1, 1, 0)
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
