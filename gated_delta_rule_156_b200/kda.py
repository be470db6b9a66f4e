"""Thin Python binding of libkda.so (argument marshalling only).

Every step of the forward pass runs in the library's CUDA kernels; torch only
provides device memory and the current CUDA stream.  There is no fallback: if
the library is missing or the tensors are not on a CUDA device the calls
raise.
"""
import ctypes
import os

import torch

from . import build as _build

KDA_OK = 0
KDA_BF16, KDA_F32 = 0, 1
STATUS_NAMES = {0: "KDA_OK", 1: "KDA_ERR_INVALID_ARG", 2: "KDA_ERR_UNSUPPORTED",
                3: "KDA_ERR_MISALIGNED", 4: "KDA_ERR_CUDA", 5: "KDA_ERR_TIMEOUT",
                6: "KDA_ERR_RANGE"}

# Entry points declared in include/kda.h (kept in sync by tests).
EXPORTS = ("kda_chunk_fwd", "kda_chunk_fwd_staged", "kda_recurrent_step",
           "kda_chunk_fwd_plan", "kda_selftest_umma", "kda_device_status",
           "kda_status_string", "kda_last_cuda_error", "kda_version",
           "kda_chunk_fwd_staged_noalloc", "kda_chunk_fwd_gated",
           "kda_recurrent_step_gated", "kda_chunk_fwd_ex",
           "kda_recurrent_step_ex", "kda_selftest_timeout", "kda_chunk_bwd",
           "kda_chunk_bwd_plan", "kda_chunk_fwd_split", "kda_workspace_pool",
           "kda_chunk_fwd_twopass", "kda_chunk_fwd_paired",
           "kda_chunk_fwd_split_plan", "kda_profile_pass_event",
           "kda_chunk_bwd_layout")
GATES = {"channel": 0, "head": 1, "none": 2}


class KdaShape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("T", ctypes.c_int), ("H", ctypes.c_int),
                ("dk", ctypes.c_int), ("dv", ctypes.c_int),
                ("chunk", ctypes.c_int), ("n_seqs", ctypes.c_int),
                ("io_dtype", ctypes.c_int)]


class KdaPrologue(ctypes.Structure):
    _fields_ = [("normalize_qk", ctypes.c_int), ("q_scale", ctypes.c_float),
                ("gate_logits", ctypes.c_int), ("gate_scale", ctypes.c_float)]


def _prologue(pro):
    """dict(normalize_qk=bool, q_scale=float, gate_logits=bool,
    gate_scale=float) -> KdaPrologue (missing keys: no-op defaults)."""
    pro = dict(pro or {})
    return KdaPrologue(int(bool(pro.get("normalize_qk", False))),
                       float(pro.get("q_scale", 1.0)),
                       int(bool(pro.get("gate_logits", False))),
                       float(pro.get("gate_scale", 1.0)))


class KdaError(RuntimeError):
    def __init__(self, status, where):
        self.status = status
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)} "
                         f"({library().kda_status_string(status).decode()})"
                         + (f" cuda error {library().kda_last_cuda_error()}"
                            if status == 4 else ""))


_lib = None


def library_path():
    return _build.LIB


def library():
    """The loaded libkda.so.  Raises if it has not been built."""
    global _lib
    if _lib is None:
        path = library_path()
        if not os.path.exists(path):
            raise RuntimeError(
                f"libkda.so not found at {path}; build it with "
                "`python -m gated_delta_rule_156_b200.build`")
        lib = ctypes.CDLL(path)
        vp, fp = ctypes.c_void_p, ctypes.c_void_p
        chunk_args = [ctypes.POINTER(KdaShape), vp, vp, vp, fp, fp, fp, vp, vp,
                      fp, vp]
        for name in ("kda_chunk_fwd", "kda_chunk_fwd_staged",
                     "kda_chunk_fwd_staged_noalloc"):
            fn = getattr(lib, name)
            fn.restype = ctypes.c_int
            fn.argtypes = chunk_args
        lib.kda_chunk_fwd_gated.restype = ctypes.c_int
        lib.kda_chunk_fwd_gated.argtypes = [
            ctypes.POINTER(KdaShape), ctypes.c_int, vp, vp, vp, fp, fp, fp, vp,
            vp, fp, ctypes.c_int, vp]
        lib.kda_recurrent_step_gated.restype = ctypes.c_int
        lib.kda_recurrent_step_gated.argtypes = [
            ctypes.POINTER(KdaShape), ctypes.c_int, vp, vp, vp, fp, fp, fp, vp,
            vp]
        lib.kda_chunk_fwd_ex.restype = ctypes.c_int
        lib.kda_chunk_fwd_ex.argtypes = [
            ctypes.POINTER(KdaShape), ctypes.c_int, ctypes.POINTER(KdaPrologue),
            vp, vp, vp, fp, fp, fp, vp, vp, fp, ctypes.c_int, vp]
        for name in ("kda_chunk_fwd_twopass", "kda_chunk_fwd_paired"):
            fn = getattr(lib, name)
            fn.restype = ctypes.c_int
            fn.argtypes = [
                ctypes.POINTER(KdaShape), ctypes.c_int,
                ctypes.POINTER(KdaPrologue), vp, vp, vp, fp, fp, fp, vp, vp,
                fp, vp]
        lib.kda_recurrent_step_ex.restype = ctypes.c_int
        lib.kda_recurrent_step_ex.argtypes = [
            ctypes.POINTER(KdaShape), ctypes.c_int, ctypes.POINTER(KdaPrologue),
            vp, vp, vp, fp, fp, fp, vp, vp]
        lib.kda_recurrent_step.restype = ctypes.c_int
        lib.kda_recurrent_step.argtypes = [ctypes.POINTER(KdaShape), vp, vp, vp,
                                           fp, fp, fp, vp, vp]
        lib.kda_chunk_fwd_plan.restype = ctypes.c_int
        lib.kda_chunk_fwd_plan.argtypes = [
            ctypes.POINTER(KdaShape), ctypes.c_int, ctypes.c_int,
            ctypes.POINTER(ctypes.c_int), ctypes.POINTER(ctypes.c_int),
            ctypes.POINTER(ctypes.c_size_t)]
        lib.kda_chunk_fwd_split.restype = ctypes.c_int
        lib.kda_chunk_fwd_split.argtypes = [
            ctypes.POINTER(KdaShape), ctypes.c_int, vp, vp, vp, fp, fp, fp, vp,
            fp, ctypes.c_int, vp]
        lib.kda_chunk_fwd_split_plan.restype = ctypes.c_int
        lib.kda_chunk_fwd_split_plan.argtypes = [
            ctypes.POINTER(KdaShape), ctypes.c_int, ctypes.c_int, ctypes.c_int,
            ctypes.POINTER(ctypes.c_int), ctypes.POINTER(ctypes.c_int),
            ctypes.POINTER(ctypes.c_size_t)]
        lib.kda_chunk_bwd.restype = ctypes.c_int
        lib.kda_chunk_bwd.argtypes = [ctypes.POINTER(KdaShape)] + [vp] * 16
        lib.kda_chunk_bwd_plan.restype = ctypes.c_int
        lib.kda_chunk_bwd_plan.argtypes = [
            ctypes.POINTER(KdaShape), ctypes.c_int, ctypes.POINTER(ctypes.c_int),
            ctypes.POINTER(ctypes.c_size_t)]
        lib.kda_chunk_bwd_layout.restype = ctypes.c_int
        lib.kda_chunk_bwd_layout.argtypes = [
            ctypes.POINTER(KdaShape), ctypes.c_int, ctypes.c_int,
            ctypes.POINTER(ctypes.c_size_t), ctypes.POINTER(ctypes.c_size_t),
            ctypes.POINTER(ctypes.c_int), ctypes.POINTER(ctypes.c_int),
            ctypes.POINTER(ctypes.c_int)]
        lib.kda_selftest_umma.restype = ctypes.c_int
        lib.kda_selftest_umma.argtypes = [ctypes.c_int] * 5 + [vp, vp, vp, vp]
        lib.kda_selftest_timeout.restype = ctypes.c_int
        lib.kda_selftest_timeout.argtypes = [ctypes.c_int, vp]
        lib.kda_device_status.restype = ctypes.c_int
        lib.kda_device_status.argtypes = [vp]
        lib.kda_status_string.restype = ctypes.c_char_p
        lib.kda_status_string.argtypes = [ctypes.c_int]
        lib.kda_workspace_pool.restype = ctypes.c_int
        lib.kda_workspace_pool.argtypes = [ctypes.POINTER(ctypes.c_size_t),
                                           ctypes.POINTER(ctypes.c_size_t)]
        lib.kda_profile_pass_event.restype = ctypes.c_int
        lib.kda_profile_pass_event.argtypes = [ctypes.c_void_p]
        lib.kda_last_cuda_error.restype = ctypes.c_int
        lib.kda_last_cuda_error.argtypes = []
        lib.kda_version.restype = ctypes.c_int
        lib.kda_version.argtypes = []
        _lib = lib
    return _lib


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _check_dev(name, t, dtype=None):
    if t is None:
        return
    if not isinstance(t, torch.Tensor) or t.device.type != "cuda":
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")


def _io(q):
    if q.dtype == torch.bfloat16:
        return KDA_BF16
    if q.dtype == torch.float32:
        return KDA_F32
    raise ValueError(f"unsupported io dtype {q.dtype}")


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def chunk_fwd(q, k, v, log_alpha, beta, initial_state=None, cu_seqlens=None,
              chunk=64, out=None, final_state=None, staged=False, stream=None,
              gate="channel", prologue=None, twopass=False, paired=False):
    """Chunkwise KDA forward (kda_chunk_fwd / kda_chunk_fwd_staged, or
    kda_chunk_fwd_gated when ``gate`` is not "channel").

    q, k [B, T, H, d_k]; v [B, T, H, d_v] (bf16 or fp32, same dtype);
    log_alpha fp32 [B, T, H, d_k] (gate="channel"), [B, T, H] (gate="head")
    or None (gate="none"); beta [B, T, H] fp32; initial_state
    [N, H, d_k, d_v] fp32 or None; cu_seqlens int32 [N + 1] or None (then
    B == 1 and T is the packed total).  ``prologue`` (dict, see
    kda_prologue) normalises q and k and/or maps gate logits in-kernel
    (kda_chunk_fwd_ex).  ``twopass`` forces the factorisation pass + chain
    kernel (kda_chunk_fwd_twopass, the default for bf16 d in {64, 128},
    chunk 64); ``paired`` the one-kernel cluster-pair path
    (kda_chunk_fwd_paired).  Returns (out, final_state).
    """
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    n = B if cu_seqlens is None else cu_seqlens.numel() - 1
    if out is None:
        out = torch.empty((B, T, H, dv), dtype=q.dtype, device=q.device)
    if final_state is None:
        final_state = torch.empty((n, H, dk, dv), dtype=torch.float32,
                                  device=q.device)
    for name, t, dt in (("q", q, None), ("k", k, q.dtype), ("v", v, q.dtype),
                        ("log_alpha", log_alpha, torch.float32),
                        ("beta", beta, torch.float32),
                        ("initial_state", initial_state, torch.float32),
                        ("cu_seqlens", cu_seqlens, torch.int32),
                        ("out", out, q.dtype),
                        ("final_state", final_state, torch.float32)):
        _check_dev(name, t, dt)
    shape = KdaShape(B, T, H, dk, dv, chunk, n if cu_seqlens is not None else 0,
                     _io(q))
    if twopass or paired:  # an explicit tensor-core evaluation
        name = "kda_chunk_fwd_twopass" if twopass else "kda_chunk_fwd_paired"
        pro = None if prologue is None else _prologue(prologue)
        st = getattr(library(), name)(
            ctypes.byref(shape), GATES[gate],
            None if pro is None else ctypes.byref(pro), _ptr(q), _ptr(k),
            _ptr(v), _ptr(log_alpha), _ptr(beta), _ptr(initial_state),
            _ptr(cu_seqlens), _ptr(out), _ptr(final_state), _stream(stream))
        if st != KDA_OK:
            raise KdaError(st, name)
        return out, final_state
    if prologue is not None:
        pro = _prologue(prologue)
        st = library().kda_chunk_fwd_ex(
            ctypes.byref(shape), GATES[gate], ctypes.byref(pro), _ptr(q),
            _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), _ptr(initial_state),
            _ptr(cu_seqlens), _ptr(out), _ptr(final_state), int(staged),
            _stream(stream))
        if st != KDA_OK:
            raise KdaError(st, "kda_chunk_fwd_ex")
        return out, final_state
    if gate != "channel":
        st = library().kda_chunk_fwd_gated(
            ctypes.byref(shape), GATES[gate], _ptr(q), _ptr(k), _ptr(v),
            _ptr(log_alpha), _ptr(beta), _ptr(initial_state), _ptr(cu_seqlens),
            _ptr(out), _ptr(final_state), int(staged), _stream(stream))
        if st != KDA_OK:
            raise KdaError(st, "kda_chunk_fwd_gated")
        return out, final_state
    fn = library().kda_chunk_fwd_staged if staged else library().kda_chunk_fwd
    st = fn(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha),
            _ptr(beta), _ptr(initial_state), _ptr(cu_seqlens), _ptr(out),
            _ptr(final_state), _stream(stream))
    if st != KDA_OK:
        raise KdaError(st, "kda_chunk_fwd_staged" if staged else "kda_chunk_fwd")
    return out, final_state


def chunk_fwd_split(q, k, v, log_alpha, beta, initial_state=None,
                    n_segments=2, chunk=64, out=None, final_state=None,
                    gate="channel", stream=None):
    """Prefill of one long sequence as ``n_segments`` segments evaluated side
    by side and joined by a scan of their state transitions
    (kda_chunk_fwd_split; ``n_segments=0`` lets the library pick the count
    from the SM count).  Shapes as chunk_fwd with B == 1 and no cu_seqlens.
    Returns (out, final_state)."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    if out is None:
        out = torch.empty((B, T, H, dv), dtype=q.dtype, device=q.device)
    if final_state is None:
        final_state = torch.empty((B, H, dk, dv), dtype=torch.float32,
                                  device=q.device)
    for name, t, dt in (("q", q, None), ("k", k, q.dtype), ("v", v, q.dtype),
                        ("log_alpha", log_alpha, torch.float32),
                        ("beta", beta, torch.float32),
                        ("initial_state", initial_state, torch.float32),
                        ("out", out, q.dtype),
                        ("final_state", final_state, torch.float32)):
        _check_dev(name, t, dt)
    shape = KdaShape(B, T, H, dk, dv, chunk, 0, _io(q))
    st = library().kda_chunk_fwd_split(
        ctypes.byref(shape), GATES[gate], _ptr(q), _ptr(k), _ptr(v),
        _ptr(log_alpha), _ptr(beta), _ptr(initial_state), _ptr(out),
        _ptr(final_state), int(n_segments), _stream(stream))
    if st != KDA_OK:
        raise KdaError(st, "kda_chunk_fwd_split")
    return out, final_state


def chunk_fwd_split_plan(T, H, dk, dv, chunk, dtype, n_segments,
                         gate="channel", num_sms=148):
    """(segments, kernels, workspace_bytes) of a chunk_fwd_split call
    (``num_sms`` matters only for ``n_segments=0``)."""
    io = KDA_BF16 if dtype == torch.bfloat16 else KDA_F32
    shape = KdaShape(1, T, H, dk, dv, chunk, 0, io)
    seg, kern, ws = ctypes.c_int(), ctypes.c_int(), ctypes.c_size_t()
    st = library().kda_chunk_fwd_split_plan(
        ctypes.byref(shape), GATES[gate], int(n_segments), int(num_sms),
        ctypes.byref(seg), ctypes.byref(kern), ctypes.byref(ws))
    if st != KDA_OK:
        raise KdaError(st, "kda_chunk_fwd_split_plan")
    return seg.value, kern.value, ws.value


def chunk_bwd(q, k, v, log_alpha, beta, initial_state, cu_seqlens, d_out,
              d_final_state=None, chunk=64, want_initial_state=True,
              stream=None):
    """Backward pass of chunk_fwd (kda_chunk_bwd; per-channel gate, no input
    prologue): the gradients of sum(d_out * out) + sum(d_final_state *
    final_state).  Shapes as chunk_fwd; d_out like out; d_final_state fp32
    [N, H, d_k, d_v] or None.  Returns (dq, dk, dv, dlog_alpha, dbeta,
    d_initial_state) with d_initial_state None unless want_initial_state.
    """
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    n = B if cu_seqlens is None else cu_seqlens.numel() - 1
    for name, t, dt in (("q", q, None), ("k", k, q.dtype), ("v", v, q.dtype),
                        ("log_alpha", log_alpha, torch.float32),
                        ("beta", beta, torch.float32),
                        ("initial_state", initial_state, torch.float32),
                        ("cu_seqlens", cu_seqlens, torch.int32),
                        ("d_out", d_out, q.dtype),
                        ("d_final_state", d_final_state, torch.float32)):
        _check_dev(name, t, dt)
    dq = torch.empty_like(q)
    dkk = torch.empty_like(k)
    dvv = torch.empty_like(v)
    dla = torch.empty((B, T, H, dk), dtype=torch.float32, device=q.device)
    dbeta = torch.empty((B, T, H), dtype=torch.float32, device=q.device)
    ds0 = (torch.empty((n, H, dk, dv), dtype=torch.float32, device=q.device)
           if want_initial_state else None)
    shape = KdaShape(B, T, H, dk, dv, chunk, n if cu_seqlens is not None else 0,
                     _io(q))
    st = library().kda_chunk_bwd(
        ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha),
        _ptr(beta), _ptr(initial_state), _ptr(cu_seqlens), _ptr(d_out),
        _ptr(d_final_state), _ptr(dq), _ptr(dkk), _ptr(dvv), _ptr(dla),
        _ptr(dbeta), _ptr(ds0), _stream(stream))
    if st != KDA_OK:
        raise KdaError(st, "kda_chunk_bwd")
    return dq, dkk, dvv, dla, dbeta, ds0


def chunk_bwd_plan(B, T, H, dk, dv, chunk, dtype, packed=False, n_seqs=0):
    """(kernels, workspace_bytes) of a chunk_bwd call of this shape."""
    io = KDA_BF16 if dtype == torch.bfloat16 else KDA_F32
    shape = KdaShape(B, T, H, dk, dv, chunk, n_seqs if packed else 0, io)
    kern, ws = ctypes.c_int(), ctypes.c_size_t()
    st = library().kda_chunk_bwd_plan(ctypes.byref(shape), int(packed),
                                      ctypes.byref(kern), ctypes.byref(ws))
    if st != KDA_OK:
        raise KdaError(st, "kda_chunk_bwd_plan")
    return kern.value, ws.value


def chunk_bwd_layout(B, T, H, dk, dv, chunk, dtype, packed=False, n_seqs=0):
    """The workspace arrays of a chunk_bwd call of this shape, as (offset,
    bytes, first launch, last launch) tuples (kda_chunk_bwd_layout); empty on
    the fp32 path, whose arrays are all apart."""
    io = KDA_BF16 if dtype == torch.bfloat16 else KDA_F32
    shape = KdaShape(B, T, H, dk, dv, chunk, n_seqs if packed else 0, io)
    cap = 64
    offs, sizes = (ctypes.c_size_t * cap)(), (ctypes.c_size_t * cap)()
    first, last, count = (ctypes.c_int * cap)(), (ctypes.c_int * cap)(), \
        ctypes.c_int()
    st = library().kda_chunk_bwd_layout(ctypes.byref(shape), int(packed), cap,
                                        offs, sizes, first, last,
                                        ctypes.byref(count))
    if st != KDA_OK:
        raise KdaError(st, "kda_chunk_bwd_layout")
    return [(offs[i], sizes[i], first[i], last[i])
            for i in range(min(count.value, cap))]


def recurrent_step(q, k, v, log_alpha, beta, state, out=None, stream=None,
                   gate="channel", prologue=None):
    """Token-by-token KDA (kda_recurrent_step, or kda_recurrent_step_gated
    when ``gate`` is "head" or "none"); ``state`` [B, H, d_k, d_v] fp32 is
    updated in place.  q, k [B, T, H, d_k] (T >= 1 tokens per sequence).
    Returns out [B, T, H, d_v]."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    if out is None:
        out = torch.empty((B, T, H, dv), dtype=q.dtype, device=q.device)
    for name, t, dt in (("q", q, None), ("k", k, q.dtype), ("v", v, q.dtype),
                        ("log_alpha", log_alpha, torch.float32),
                        ("beta", beta, torch.float32),
                        ("state", state, torch.float32), ("out", out, q.dtype)):
        _check_dev(name, t, dt)
    shape = KdaShape(B, T, H, dk, dv, 0, 0, _io(q))
    if prologue is not None:
        pro = _prologue(prologue)
        st = library().kda_recurrent_step_ex(
            ctypes.byref(shape), GATES[gate], ctypes.byref(pro), _ptr(q),
            _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), _ptr(state),
            _ptr(out), _stream(stream))
        if st != KDA_OK:
            raise KdaError(st, "kda_recurrent_step_ex")
        return out
    st = library().kda_recurrent_step_gated(
        ctypes.byref(shape), GATES[gate], _ptr(q), _ptr(k), _ptr(v),
        _ptr(log_alpha), _ptr(beta), _ptr(state), _ptr(out), _stream(stream)) \
        if gate != "channel" else library().kda_recurrent_step(
            ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha),
            _ptr(beta), _ptr(state), _ptr(out), _stream(stream))
    if st != KDA_OK:
        raise KdaError(st, "kda_recurrent_step")
    return out


def chunk_fwd_plan(B, T, H, dk, dv, chunk, dtype, packed=False, n_seqs=0,
                   staged=False):
    """(path, kernels, workspace_bytes) of a chunk_fwd call of this shape:
    path is "twopass" or "staged"; no device work is done."""
    io = KDA_BF16 if dtype == torch.bfloat16 else KDA_F32
    shape = KdaShape(B, T, H, dk, dv, chunk, n_seqs if packed else 0, io)
    path, kern, ws = ctypes.c_int(), ctypes.c_int(), ctypes.c_size_t()
    st = library().kda_chunk_fwd_plan(ctypes.byref(shape), int(packed),
                                      int(staged), ctypes.byref(path),
                                      ctypes.byref(kern), ctypes.byref(ws))
    if st != KDA_OK:
        raise KdaError(st, "kda_chunk_fwd_plan")
    return ({2: "twopass", 1: "fused"}.get(path.value, "staged"), kern.value,
            ws.value)


def chunk_fwd_kernel_count(B, T, H, dk, dv, chunk, dtype, packed=False):
    return chunk_fwd_plan(B, T, H, dk, dv, chunk, dtype, packed, 1)[1]


def chunk_fwd_path(B, T, H, dk, dv, chunk, dtype, packed=False):
    return chunk_fwd_plan(B, T, H, dk, dv, chunk, dtype, packed, 1)[0]


def selftest_umma(A, B, a_mn, b_mn, panel_rows=None, stream=None):
    """Diagnostic tensor-core product through the fused kernel's operand
    layouts (kda_selftest_umma).  A is [128, K] (a_mn=False) or [K, 128]
    (a_mn=True); B is [N, K] (b_mn=False) or [K, N] (b_mn=True); bf16.
    Returns D = A_logical @ B_logical as [128, N] fp32."""
    K = A.shape[1] if not a_mn else A.shape[0]
    N = B.shape[0] if not b_mn else B.shape[1]
    D = torch.empty((128, N), dtype=torch.float32, device=A.device)
    for name, t in (("A", A), ("B", B)):
        _check_dev(name, t, torch.bfloat16)
    st = library().kda_selftest_umma(int(a_mn), int(b_mn), N, K,
                                     panel_rows or K, _ptr(A), _ptr(B),
                                     _ptr(D), _stream(stream))
    if st != KDA_OK:
        raise KdaError(st, "kda_selftest_umma")
    return D


def profile_pass_event(event):
    """Set (a torch.cuda.Event, already recorded once so that it exists) or
    clear (None) the event that two-pass calls on this thread record between
    their factorisation pass and their chain kernel
    (kda_profile_pass_event)."""
    h = None if event is None else ctypes.c_void_p(event.cuda_event)
    if event is not None and not event.cuda_event:
        raise ValueError("record the event once before passing it")
    st = library().kda_profile_pass_event(h)
    if st != 0:
        raise KdaError(st, "kda_profile_pass_event")


def workspace_pool():
    """(reserved, used) bytes of the device memory pool the library's
    stream-ordered workspace comes from (kda_workspace_pool)."""
    r, u = ctypes.c_size_t(), ctypes.c_size_t()
    st = library().kda_workspace_pool(ctypes.byref(r), ctypes.byref(u))
    if st != KDA_OK:
        raise KdaError(st, "kda_workspace_pool")
    return r.value, u.value


def device_status(stream=None):
    """Synchronise the stream and return the library's device-side status
    code (0 = no bounded wait ran out since the last call)."""
    return library().kda_device_status(_stream(stream))


NOALLOC_SCRATCH_BYTES = 16 << 20  # KDA_NOALLOC_SCRATCH_BYTES in include/kda.h


def chunk_fwd_noalloc(q, k, v, log_alpha, beta, initial_state=None,
                      cu_seqlens=None, chunk=64, out=None, final_state=None,
                      stream=None):
    """kda_chunk_fwd_staged_noalloc: the four-stage fp32 pipeline with its
    workspace in the library's fixed device array, for callers that must not
    allocate device memory during the call.  ``out`` and ``final_state``
    should be passed in by such callers (they are allocated here only when
    omitted).  Calls that overlap on the GPU race on the shared array."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    n = B if cu_seqlens is None else cu_seqlens.numel() - 1
    if out is None:
        out = torch.empty((B, T, H, dv), dtype=q.dtype, device=q.device)
    if final_state is None:
        final_state = torch.empty((n, H, dk, dv), dtype=torch.float32,
                                  device=q.device)
    for name, t, dt in (("q", q, None), ("k", k, q.dtype), ("v", v, q.dtype),
                        ("log_alpha", log_alpha, torch.float32),
                        ("beta", beta, torch.float32),
                        ("initial_state", initial_state, torch.float32),
                        ("cu_seqlens", cu_seqlens, torch.int32),
                        ("out", out, q.dtype),
                        ("final_state", final_state, torch.float32)):
        _check_dev(name, t, dt)
    shape = KdaShape(B, T, H, dk, dv, chunk, n if cu_seqlens is not None else 0,
                     _io(q))
    st = library().kda_chunk_fwd_staged_noalloc(
        ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha),
        _ptr(beta), _ptr(initial_state), _ptr(cu_seqlens), _ptr(out),
        _ptr(final_state), _stream(stream))
    if st != KDA_OK:
        raise KdaError(st, "kda_chunk_fwd_staged_noalloc")
    return out, final_state


def selftest_timeout(limit_us=1000, stream=None):
    """Diagnostic (kda_selftest_timeout): a kernel whose bounded wait runs out
    after limit_us; the next device_status() then reports KDA_ERR_TIMEOUT."""
    st = library().kda_selftest_timeout(int(limit_us), _stream(stream))
    if st != KDA_OK:
        raise KdaError(st, "kda_selftest_timeout")
