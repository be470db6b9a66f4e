"""Helpers shared by the GPU parity tests: error metrics and oracle runs on
selected (sequence, head) units."""
import numpy as np
import torch

from oracle import kda_oracle

# Tolerances on the relative L2 error over a whole tensor (and per sampled
# unit): bf16 inputs/outputs with an fp32 state, and the all-fp32 mode.
TOL_BF16 = 1e-2
TOL_F32 = 1e-4


def rel_l2(x, ref):
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    den = np.linalg.norm(ref)
    num = np.linalg.norm(x - ref)
    return float(num / den) if den > 0 else float(num)


def max_abs(x, ref):
    return float(np.max(np.abs(np.asarray(x, np.float64) - np.asarray(ref, np.float64))))


def host64(t):
    return t.detach().float().cpu().double().numpy()


def check(name, got, ref, tol):
    e = rel_l2(got, ref)
    m = max_abs(got, ref)
    assert np.all(np.isfinite(np.asarray(got, np.float64))), f"{name}: non-finite"
    assert e <= tol, f"{name}: rel-L2 {e:.3e} > {tol:.0e} (max-abs {m:.3e})"
    return e, m


def oracle_dense(d):
    """Oracle over a whole dense-layout input dict (small configs)."""
    return kda_oracle.recurrent(host64(d["q"]), host64(d["k"]), host64(d["v"]),
                                host64(d["log_alpha"]), host64(d["beta"]),
                                None if d["initial_state"] is None
                                else host64(d["initial_state"]))


def oracle_units(q, k, v, la, beta, s0, units, offsets=None):
    """Oracle for selected (sequence, head) units of a dense [B, T, H, d] or
    packed [1, T_total, H, d] input (``offsets``: token offsets per sequence,
    host list).  The units are packed into one oracle call (one head each) so
    they run in parallel.  Returns {(s, h): (out [T_s, d_v], final [d_k, d_v])}."""
    parts = {n: [] for n in ("q", "k", "v", "la", "b", "s0")}
    offs = [0]
    for s, h in units:
        if offsets is None:
            sl = (s, slice(None), h)
        else:
            sl = (0, slice(offsets[s], offsets[s + 1]), h)
        for n, x in (("q", q), ("k", k), ("v", v), ("la", la)):
            parts[n].append(host64(x[sl]))
        parts["b"].append(host64(beta[sl]))
        parts["s0"].append(None if s0 is None else host64(s0[s, h]))
        offs.append(offs[-1] + parts["q"][-1].shape[0])
    cat = {n: np.concatenate(parts[n], 0) for n in ("q", "k", "v", "la", "b")}
    st = None if s0 is None else np.stack(parts["s0"])[:, None]
    o, f = kda_oracle.recurrent(cat["q"][:, None], cat["k"][:, None],
                                cat["v"][:, None], cat["la"][:, None],
                                cat["b"][:, None], st, seq_offsets=offs)
    return {u: (o[offs[i]:offs[i + 1], 0], f[i, 0]) for i, u in enumerate(units)}


def sample_units(n_seqs, H, count, seed=0, must=()):
    rng = np.random.default_rng(seed)
    units = set(must)
    while len(units) < min(count, n_seqs * H):
        units.add((int(rng.integers(n_seqs)), int(rng.integers(H))))
    return sorted(units)


def nan_like(t):
    return torch.full_like(t, float("nan"))


def check_units(name, got, ref, tol, unit_axes):
    """Whole-tensor comparison that also bounds every unit: rel-L2 over the
    whole tensor and over each slice that fixes the ``unit_axes`` (e.g. each
    (sequence, head)), max-abs over everything.  Returns (whole rel-L2,
    worst unit rel-L2, max-abs)."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, (name, got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{name}: non-finite"
    whole = rel_l2(got, ref)
    red = tuple(i for i in range(got.ndim) if i not in unit_axes)
    num = np.sqrt(np.sum((got - ref) ** 2, axis=red))
    den = np.sqrt(np.sum(ref ** 2, axis=red))
    per = np.where(den > 0, num / np.where(den > 0, den, 1.0), num)
    worst = float(np.max(per)) if per.size else 0.0
    m = max_abs(got, ref) if got.size else 0.0
    assert whole <= tol, f"{name}: rel-L2 {whole:.3e} > {tol:.0e} (max-abs {m:.3e})"
    assert worst <= tol, (f"{name}: worst unit rel-L2 {worst:.3e} > {tol:.0e} "
                          f"at {np.unravel_index(np.argmax(per), per.shape)}")
    return whole, worst, m
