"""fp64 CPU oracle of the Kimi Delta Attention forward pass.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this module.  It shares no code with
the CUDA path and imports nothing from it.

Three independent CPU computations of the same forward quantity, and its
gradients:

``recurrent``     the plain definition, token by token, in C (kda_recurrence.c,
                  fp64, OpenMP over (sequence, head)).  This is the oracle.
``brute_force``   the unrolled product form of the same recurrence for one
                  (sequence, head) and T <= 8, written with explicit
                  d_k x d_k transition matrices M_t = (I - b_t k_t k_t^T) Diag(a_t):
                  S_t = M_t ... M_1 S_0 + sum_i (M_t ... M_{i+1}) b_i k_i v_i^T.
                  Each prefix t is recomputed from scratch, so it is not the
                  recurrence evaluated a second time.
``recurrent_bwd`` the reverse-mode gradients of ``recurrent`` (the chain rule
                  applied line by line to the token step, in C, fp64), pinned
                  by central finite differences of ``recurrent``.
``chunked_debug`` an fp64 model of the chunkwise rewrite that the GPU prefill
                  kernels use (decay prefix sums, the strictly-lower factor
                  matrix A, T = (I + A)^-1 by forward substitution, W, U, the
                  per-chunk state pass and the output).  Used to localise GPU
                  stage errors; pinned to ``recurrent`` by the tests.

Sources (paraphrased): the delta-rule read/error/write ("Kimi Delta Attention",
akshathtiwari.co.in, delta-rule passage; "Attention? More like notation
warfare", Key Points); the per-key-channel forget vector applied as
Diag(alpha_t) ("Kimi Delta Attention", akshathtiwari.co.in, channel-wise gating
passage; "Teacher guide - Kimi Delta Attention", Misconceptions table row 2;
"The fourth layer remembers", forget-gate paragraph); the chunkwise
reorganisation of the recurrence into matrix products ("You Could Have Come Up
with Kimi Delta Attention", daily.dev, Summary; the explainer's remark on the
Diagonal-Plus-Low-Rank chunkwise algorithm).
"""
import ctypes
import os

import numpy as np

from . import build_oracle

_libs = {}


def _load(path=None):
    """Load (building if needed) the oracle library, or another build of the
    same source at ``path`` (the tests load deliberately broken copies)."""
    if path is None:
        path = build_oracle.build()
    if path not in _libs:
        lib = ctypes.CDLL(path)
        P = ctypes.POINTER(ctypes.c_double)
        I64 = ctypes.c_int64
        lib.kda_oracle_recurrent.restype = ctypes.c_int
        lib.kda_oracle_recurrent.argtypes = [
            I64, ctypes.POINTER(I64), I64, I64, I64, P, P, P, P, P, P, P, P]
        lib.kda_oracle_recurrent_bwd.restype = ctypes.c_int
        lib.kda_oracle_recurrent_bwd.argtypes = [
            I64, ctypes.POINTER(I64), I64, I64, I64] + [P] * 14
        lib.kda_oracle_num_threads.restype = ctypes.c_int
        lib.kda_oracle_num_threads.argtypes = []
        _libs[path] = lib
    return _libs[path]


def num_threads() -> int:
    """Threads the oracle's OpenMP region uses (OMP_NUM_THREADS or all cores)."""
    return int(_load().kda_oracle_num_threads())


def _f64(x):
    if x is None:
        return None
    if hasattr(x, "detach"):  # a torch tensor on the host
        x = x.detach().cpu().double().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def recurrent(q, k, v, log_alpha, beta, initial_state=None, seq_offsets=None,
              library=None):
    """Token-by-token fp64 recurrence (the oracle).

    Shapes: q, k, log_alpha [B, T, H, d_k] (or [T_total, H, d_k] with
    ``seq_offsets``); v [.., H, d_v]; beta [.., H]; initial_state
    [n_seqs, H, d_k, d_v] or None (zeros).  ``seq_offsets`` (n_seqs + 1 token
    offsets into the packed token axis) selects the variable-length layout.
    Returns (out [same leading shape, H, d_v], final_state [n_seqs, H, d_k, d_v]),
    both float64.  ``library`` selects another build of the C source.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    la, b = _f64(log_alpha), _f64(beta)
    s0 = _f64(initial_state)
    lead = q.shape[:-2]
    H, dk = q.shape[-2], q.shape[-1]
    dv = v.shape[-1]
    if seq_offsets is None:
        if q.ndim != 4:
            raise ValueError("without seq_offsets q must be [B, T, H, d_k]")
        B, T = q.shape[0], q.shape[1]
        offs = np.arange(B + 1, dtype=np.int64) * T
    else:
        if q.ndim == 4:
            if q.shape[0] != 1:
                raise ValueError("packed layout needs B == 1")
        offs = np.ascontiguousarray(np.asarray(seq_offsets, dtype=np.int64))
    n_seqs = len(offs) - 1
    T_total = int(np.prod(lead))
    if offs[0] != 0 or offs[-1] != T_total:
        raise ValueError("seq_offsets must start at 0 and end at the token count")
    if s0 is not None and s0.shape != (n_seqs, H, dk, dv):
        raise ValueError(f"initial_state shape {s0.shape} != {(n_seqs, H, dk, dv)}")
    out = np.zeros(lead + (H, dv), dtype=np.float64)
    fin = np.zeros((n_seqs, H, dk, dv), dtype=np.float64)
    rc = _load(library).kda_oracle_recurrent(
        n_seqs, offs.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), H, dk, dv,
        _ptr(q), _ptr(k), _ptr(v), _ptr(la), _ptr(b), _ptr(s0), _ptr(out),
        _ptr(fin))
    if rc != 0:
        raise RuntimeError(f"kda_oracle_recurrent failed ({rc})")
    return out, fin


def recurrent_bwd(q, k, v, log_alpha, beta, initial_state, d_out,
                  d_final_state=None, seq_offsets=None, library=None):
    """Gradients of the token-by-token recurrence (reverse mode, fp64) for
    L = sum(d_out * out) + sum(d_final_state * final_state), in C
    (kda_recurrence.c, ``kda_oracle_recurrent_bwd``).

    Shapes as ``recurrent``; d_out like the output, d_final_state like the
    final state (None = zero).  Returns (dq, dk, dv, dlog_alpha, dbeta,
    d_initial_state), float64, in the shapes of the corresponding inputs
    (d_initial_state [n_seqs, H, d_k, d_v] whether or not a state was given).
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    la, b = _f64(log_alpha), _f64(beta)
    s0, do, dsT = _f64(initial_state), _f64(d_out), _f64(d_final_state)
    lead = q.shape[:-2]
    H, dk = q.shape[-2], q.shape[-1]
    dv = v.shape[-1]
    if seq_offsets is None:
        if q.ndim != 4:
            raise ValueError("without seq_offsets q must be [B, T, H, d_k]")
        B, T = q.shape[0], q.shape[1]
        offs = np.arange(B + 1, dtype=np.int64) * T
    else:
        if q.ndim == 4 and q.shape[0] != 1:
            raise ValueError("packed layout needs B == 1")
        offs = np.ascontiguousarray(np.asarray(seq_offsets, dtype=np.int64))
    n_seqs = len(offs) - 1
    if offs[0] != 0 or offs[-1] != int(np.prod(lead)):
        raise ValueError("seq_offsets must start at 0 and end at the token count")
    if do.shape != lead + (H, dv):
        raise ValueError(f"d_out shape {do.shape} != {lead + (H, dv)}")
    for name, st in (("initial_state", s0), ("d_final_state", dsT)):
        if st is not None and st.shape != (n_seqs, H, dk, dv):
            raise ValueError(f"{name} shape {st.shape} != {(n_seqs, H, dk, dv)}")
    dq, dkk, dla = (np.zeros(lead + (H, dk)) for _ in range(3))
    dvv = np.zeros(lead + (H, dv))
    dbeta = np.zeros(lead + (H,))
    ds0 = np.zeros((n_seqs, H, dk, dv))
    rc = _load(library).kda_oracle_recurrent_bwd(
        n_seqs, offs.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), H, dk, dv,
        _ptr(q), _ptr(k), _ptr(v), _ptr(la), _ptr(b), _ptr(s0), _ptr(do),
        _ptr(dsT), _ptr(dq), _ptr(dkk), _ptr(dvv), _ptr(dla), _ptr(dbeta),
        _ptr(ds0))
    if rc != 0:
        raise RuntimeError(f"kda_oracle_recurrent_bwd failed ({rc})")
    return dq, dkk, dvv, dla, dbeta, ds0


def brute_force(q, k, v, log_alpha, beta, initial_state=None):
    """Unrolled-product evaluation for ONE (sequence, head), T <= 8.

    q, k, log_alpha [T, d_k]; v [T, d_v]; beta [T]; initial_state [d_k, d_v].
    Returns (out [T, d_v], final_state [d_k, d_v]).
    """
    q, k, v, la, b = map(_f64, (q, k, v, log_alpha, beta))
    T, dk = k.shape
    dv = v.shape[1]
    if T > 8:
        raise ValueError("brute force is for T <= 8")
    S0 = np.zeros((dk, dv)) if initial_state is None else _f64(initial_state)
    eye = np.eye(dk)
    M = [(eye - b[t] * np.outer(k[t], k[t])) @ np.diag(np.exp(la[t]))
         for t in range(T)]

    def prod(lo, hi):  # M_hi-1 @ ... @ M_lo  (identity when empty)
        P = eye.copy()
        for t in range(lo, hi):
            P = M[t] @ P
        return P

    out = np.zeros((T, dv))
    S_t = S0
    for t in range(1, T + 1):
        S_t = prod(0, t) @ S0
        for i in range(t):
            S_t = S_t + prod(i + 1, t) @ (b[i] * np.outer(k[i], v[i]))
        out[t - 1] = S_t.T @ q[t - 1]
    return out, S_t


def _forward_substitution_inverse(A):
    """(I + A)^-1 for strictly-lower A, one row at a time:
    row r of X = e_r - sum_{i<r} A[r, i] * row i of X."""
    n = A.shape[0]
    X = np.zeros_like(A)
    for r in range(n):
        X[r, r] = 1.0
        for i in range(r):
            X[r, :] -= A[r, i] * X[i, :]
    return X


def chunked_debug(q, k, v, log_alpha, beta, initial_state=None, chunk=64):
    """fp64 model of the chunkwise rewrite for ONE (sequence, head).

    Per chunk of C tokens (positions r = 1..C), with chunk-start state S_0:
      g_r   = sum_{i<=r} l_i                   (per key channel)
      Kt    = k * exp(g)      Kb = k * exp(-g)      Qt = q * exp(g)
      Kh    = k * exp(g_C - g)
      A     = strictly_lower(Diag(beta) Kt Kb^T)
      Tm    = (I + A)^-1      (forward substitution)
      W     = Tm Diag(beta) Kt          U = Tm Diag(beta) V
      Delta = U - W S_0
      O     = Qt S_0 + lower_incl(Qt Kb^T) Delta
      S_C   = Diag(exp(g_C)) S_0 + Kh^T Delta
    The last chunk may be shorter than C.  Returns a dict with 'out', 'final'
    and per-chunk lists 'g', 'A', 'Tm', 'W', 'U', 'S_start'.
    """
    q, k, v, la, b = map(_f64, (q, k, v, log_alpha, beta))
    T, dk = k.shape
    dv = v.shape[1]
    S = np.zeros((dk, dv)) if initial_state is None else _f64(initial_state).copy()
    out = np.zeros((T, dv))
    rec = {k_: [] for k_ in ("g", "A", "Tm", "W", "U", "S_start")}
    for c0 in range(0, T, chunk):
        c1 = min(T, c0 + chunk)
        kc, qc, vc, lc, bc = k[c0:c1], q[c0:c1], v[c0:c1], la[c0:c1], b[c0:c1]
        g = np.cumsum(lc, axis=0)
        Kt, Kb, Qt = kc * np.exp(g), kc * np.exp(-g), qc * np.exp(g)
        Kh = kc * np.exp(g[-1][None, :] - g)
        A = np.tril(bc[:, None] * (Kt @ Kb.T), -1)
        Tm = _forward_substitution_inverse(A)
        W = Tm @ (bc[:, None] * Kt)
        U = Tm @ (bc[:, None] * vc)
        Delta = U - W @ S
        out[c0:c1] = Qt @ S + np.tril(Qt @ Kb.T, 0) @ Delta
        for name, val in (("g", g), ("A", A), ("Tm", Tm), ("W", W), ("U", U),
                          ("S_start", S.copy())):
            rec[name].append(val)
        S = np.exp(g[-1])[:, None] * S + Kh.T @ Delta
    rec["out"] = out
    rec["final"] = S
    return rec


def chunked_bwd_debug(q, k, v, log_alpha, beta, initial_state, d_out,
                      d_final_state=None, chunk=64):
    """fp64 model of the chunkwise backward for ONE (sequence, head): the chain
    rule applied to each line of ``chunked_debug``, chunk by chunk in reverse.

    Per chunk, with G = Diag(exp(g_C)) dS_C (dS_C the gradient of the state
    leaving the chunk):
      S_C = Diag(exp(g_C)) (S_0 + Kb^T Delta):
          dS_0 = G, dDelta = Kb G, dKb = Delta G^T,
          d exp(g_C) = rowsum((S_0 + Kb^T Delta) * dS_C)
      O = Qt S_0 + P Delta, P = lower_incl(Qt Kb^T):
          dQt = dO S_0^T + dP Kb, dS_0 += Qt^T dO, dDelta += P^T dO,
          dP = lower_incl(dO Delta^T), dKb += dP^T Qt
      Delta = U - W S_0:  dU = dDelta, dW = -dDelta S_0^T, dS_0 -= W^T dDelta
      W = Tm Diag(b) Kt, U = Tm Diag(b) V:
          dTm = dW (b Kt)^T + dU (b V)^T, dKt = b Tm^T dW, dV = b Tm^T dU,
          db = rowsum(Tm^T dW * Kt) + rowsum(Tm^T dU * V)
      Tm = (I + A)^-1:  dA = strictly_lower(-Tm^T dTm Tm^T)
      A = strictly_lower(Diag(b) Kt Kb^T):
          db += rowsum(dA * Kt Kb^T), dKt += (b dA) Kb, dKb += (b dA)^T Kt
      Kt = k e^g, Kb = k e^-g, Qt = q e^g:
          dk = dKt e^g + dKb e^-g, dq = dQt e^g,
          dg = dKt * Kt + dQt * Qt - dKb * Kb  (+ exp(g_C) d exp(g_C) on row C)
      g = cumsum(l):  dl = reverse cumsum of dg within the chunk
    and dS_0 becomes the previous chunk's dS_C.  Returns (dq, dk, dv,
    dlog_alpha, dbeta, d_initial_state) in float64.  Used to check the
    chunkwise algebra the GPU backward follows; pinned to ``recurrent_bwd``.
    """
    q, k, v, la, b, do = map(_f64, (q, k, v, log_alpha, beta, d_out))
    T, dk = k.shape
    dv = v.shape[1]
    fwd = chunked_debug(q, k, v, la, b, initial_state, chunk)
    dq, dkk, dla = np.zeros((T, dk)), np.zeros((T, dk)), np.zeros((T, dk))
    dvv, db = np.zeros((T, dv)), np.zeros(T)
    dS = np.zeros((dk, dv)) if d_final_state is None else _f64(d_final_state).copy()
    for ci in reversed(range(len(fwd["g"]))):
        c0 = ci * chunk
        c1 = min(T, c0 + chunk)
        kc, qc, vc, bc, doc = k[c0:c1], q[c0:c1], v[c0:c1], b[c0:c1], do[c0:c1]
        g, Tm, W, U, S0 = (fwd[n][ci] for n in ("g", "Tm", "W", "U", "S_start"))
        eg, emg = np.exp(g), np.exp(-g)
        Kt, Kb, Qt = kc * eg, kc * emg, qc * eg
        gam = eg[-1]
        Delta = U - W @ S0
        P = np.tril(Qt @ Kb.T, 0)
        # S_C = Diag(gam) (S_0 + Kb^T Delta)
        G = gam[:, None] * dS
        dS0 = G.copy()
        dDelta = Kb @ G
        dKb = Delta @ G.T
        dgam = ((S0 + Kb.T @ Delta) * dS).sum(axis=1)
        # O = Qt S_0 + P Delta
        dQt = doc @ S0.T
        dS0 += Qt.T @ doc
        dP = np.tril(doc @ Delta.T, 0)
        dDelta += P.T @ doc
        dQt += dP @ Kb
        dKb += dP.T @ Qt
        # Delta = U - W S_0
        dW = -dDelta @ S0.T
        dS0 -= W.T @ dDelta
        # W = Tm (b Kt), U = Tm (b V)
        BK, BV = bc[:, None] * Kt, bc[:, None] * vc
        dTm = dW @ BK.T + dDelta @ BV.T
        dBK, dBV = Tm.T @ dW, Tm.T @ dDelta
        dKt = bc[:, None] * dBK
        dvv[c0:c1] = bc[:, None] * dBV
        db[c0:c1] = (dBK * Kt).sum(axis=1) + (dBV * vc).sum(axis=1)
        # Tm = (I + A)^-1, A = strictly_lower(b Kt Kb^T)
        dA = np.tril(-Tm.T @ dTm @ Tm.T, -1)
        db[c0:c1] += (dA * (Kt @ Kb.T)).sum(axis=1)
        dM = bc[:, None] * dA
        dKt += dM @ Kb
        dKb += dM.T @ Kt
        # Kt = k e^g, Kb = k e^-g, Qt = q e^g, g = cumsum(l)
        dkk[c0:c1] = dKt * eg + dKb * emg
        dq[c0:c1] = dQt * eg
        dg = dKt * Kt + dQt * Qt - dKb * Kb
        dg[-1] += dgam * gam
        dla[c0:c1] = np.cumsum(dg[::-1], axis=0)[::-1]
        dS = dS0
    return dq, dkk, dvv, dla, db, dS


def prologue(q, k, gate, normalize_qk=True, q_scale=1.0, gate_logits=True,
             gate_scale=1.0):
    """The optional input prologue, in fp64, as its plain definition:
      q <- q_scale * q / ||q||,  k <- k / ||k||   (L2 norm over d_k, per token
                                                 and head; only if normalize_qk)
      log(alpha) <- gate_scale * logsigmoid(gate) (only if gate_logits), with
      logsigmoid(x) = log(1 / (1 + exp(-x))).
    ``gate`` may be a per-channel [.., d_k], per-head [..] tensor, or None.
    Returns (q, k, log_alpha) as float64 arrays (log_alpha None if gate is).
    """
    q, k = _f64(q), _f64(k)
    if normalize_qk:
        q = q_scale * q / np.sqrt(np.sum(q * q, axis=-1, keepdims=True))
        k = k / np.sqrt(np.sum(k * k, axis=-1, keepdims=True))
    elif q_scale != 1.0:
        q = q_scale * q
    la = None if gate is None else _f64(gate)
    if la is not None and gate_logits:
        la = gate_scale * -np.logaddexp(0.0, -la)
    return q, k, la
