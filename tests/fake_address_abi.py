"""Host-side argument validation of the C ABI, exercised with fake device
addresses that are never dereferenced: every call here must be rejected on
the host before anything is launched.

A regression in that validation must not be able to launch a kernel on these
addresses, so this file only runs in a process that sees no GPU
(CUDA_VISIBLE_DEVICES set to the empty string): test_abi_cpu.py starts it
that way in a child process, and anywhere else it skips itself.  Were a check
ever to let a call through, the call would then fail with a CUDA error (no
device) instead of touching memory."""
import ctypes
import os

import pytest

if os.environ.get("CUDA_VISIBLE_DEVICES", None) != "":
    pytest.skip("runs only in a process with no visible GPU",
                allow_module_level=True)

from gated_delta_rule_156_b200 import build as kbuild  # noqa: E402
from gated_delta_rule_156_b200 import kda as K  # noqa: E402


@pytest.fixture(scope="module")
def lib():
    kbuild.build()
    return K.library()


def shape(**kw):
    d = dict(B=1, T=64, H=2, dk=64, dv=64, chunk=64, n_seqs=0, io_dtype=0)
    d.update(kw)
    return K.KdaShape(**d)


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


@pytest.mark.parametrize("fn", ["kda_chunk_fwd", "kda_chunk_fwd_staged",
                                "kda_chunk_fwd_staged_noalloc"])
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


def split_call(lib, s, gate=0, n=2, **kw):
    """kda_chunk_fwd_split with fake, disjoint addresses."""
    names = ["q", "k", "v", "la", "b", "s0", "out", "sf"]
    slots = {nm: i + 1 for i, nm in enumerate(names)}
    slots.update(kw)
    args = [_p(slots[nm]) if isinstance(slots[nm], int) else slots[nm]
            for nm in names]
    return lib.kda_chunk_fwd_split(ctypes.byref(s), gate, *args, n, None)


def test_split_validation(lib):
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


def test_noalloc_rejects_requests_beyond_the_scratch_size(lib):
    # one sequence of 2^20 tokens, H = 32, d = 128: the staged workspace is
    # four fp32 [tokens, H, 128] arrays (16 GiB each) plus the chunk-start
    # states, far beyond the fixed scratch array; the size check refuses it
    # before any CUDA call
    s = shape(T=1 << 20, H=32, dk=128, dv=128)
    size = ctypes.c_size_t(0)
    assert lib.kda_chunk_fwd_plan(ctypes.byref(s), 0, 1, None, None,
                                  ctypes.byref(size)) == 0
    assert size.value > 4 * (16 << 30) > K.NOALLOC_SCRATCH_BYTES
    base = 0x7000_0000_0000
    ptrs = [ctypes.c_void_p(base + i * (1 << 36)) for i in range(9)]
    st = lib.kda_chunk_fwd_staged_noalloc(ctypes.byref(s), *ptrs[:5],
                                          None, None, ptrs[5], ptrs[6], None)
    assert st == 2  # KDA_ERR_UNSUPPORTED
