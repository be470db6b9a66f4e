"""Seeded synthetic workloads for the KDA forward pass.

This module only draws random inputs; it holds none of the method's arithmetic.
Both the CUDA path's tests/bench and the CPU oracle take their inputs from it.

Recipe (every config uses seed 1000 + config id unless told otherwise):
  q, k       ~ N(0, 1), then L2-normalised per token and head (over d_k);
               configs 2 and 3 then scale q by 1/sqrt(d_k).
  v          ~ N(0, 1)
  beta       = sigmoid(N(0, 1))                     one per token and head
  log_alpha  = logsigmoid(N(0, 1)) / 16             one per token, head, key channel
               (the divisor is a parameter of draw(); strong-gate tests use 1)
  state      ~ N(0, 0.1) (standard deviation 0.1) where the config has one
Draw order from one torch.Generator: q, k, v, beta, log_alpha, state.  The
lengths of the packed config are drawn first from a separate CPU generator,
so they are the same on every device.
"""
import math

import torch

CONFIGS = {
    0: dict(name="tiny-fp32", kind="chunk", B=1, H=1, T=128, dk=32, dv=32,
            chunk=16, io="f32", scale_q=False, init_state=False),
    1: dict(name="small-bf16", kind="chunk", B=1, H=4, T=2048, dk=64, dv=64,
            chunk=64, io="bf16", scale_q=False, init_state=True),
    2: dict(name="kimi-linear-layer", kind="chunk", B=2, H=32, T=8192, dk=128,
            dv=128, chunk=64, io="bf16", scale_q=True, init_state=False),
    3: dict(name="packed-varlen-long", kind="varlen", n_short=16,
            len_lo=256, len_hi=16384, long_len=131072, H=32, dk=128, dv=128,
            chunk=64, io="bf16", scale_q=True, init_state=True),
    4: dict(name="decode", kind="decode", N=256, H=32, dk=128, dv=128,
            steps=64, io="bf16", scale_q=False, init_state=True),
}

DTYPES = {"f32": torch.float32, "bf16": torch.bfloat16}


def seed_of(cfg_id: int) -> int:
    return 1000 + int(cfg_id)


def varlen_lengths(n_short=16, lo=256, hi=16384, long_len=131072, seed=1003):
    """Sequence lengths of the packed workload: n_short ~ U{lo..hi}, then one
    sequence of long_len, in that order."""
    g = torch.Generator(device="cpu").manual_seed(seed)
    short = torch.randint(lo, hi + 1, (n_short,), generator=g).tolist()
    return short + ([long_len] if long_len else [])


def _unit(x):
    return x / x.norm(dim=-1, keepdim=True)


def draw(lead, H, dk, dv, *, io="bf16", scale_q=False, n_states=None,
         device="cpu", seed=0, state_std=0.1, gate_divisor=16.0):
    """Draw one set of KDA inputs with leading shape ``lead`` (e.g. (B, T)).

    Returns dict(q, k, v [lead, H, d] in the io dtype; log_alpha [lead, H, dk]
    and beta [lead, H] in fp32; initial_state [n_states, H, dk, dv] fp32 or
    None).  ``gate_divisor`` divides the logsigmoid gate (16 in every named
    config; 1 gives the undivided logsigmoid(N(0, 1)) gate, whose decay over
    a 64-token chunk is about 16 times stronger).
    """
    g = torch.Generator(device=device).manual_seed(int(seed))
    dt = DTYPES[io]
    shape_k = tuple(lead) + (H, dk)
    shape_v = tuple(lead) + (H, dv)
    opts = dict(generator=g, device=device, dtype=torch.float32)
    q = _unit(torch.randn(shape_k, **opts))
    if scale_q:
        q = q * (1.0 / math.sqrt(dk))
    k = _unit(torch.randn(shape_k, **opts))
    v = torch.randn(shape_v, **opts)
    beta = torch.sigmoid(torch.randn(tuple(lead) + (H,), **opts))
    log_alpha = (torch.nn.functional.logsigmoid(torch.randn(shape_k, **opts))
                 / gate_divisor)
    state = None
    if n_states:
        state = torch.randn((n_states, H, dk, dv), **opts) * state_std
    return dict(q=q.to(dt), k=k.to(dt), v=v.to(dt), log_alpha=log_alpha,
                beta=beta, initial_state=state)


def make(cfg_id, device="cpu", seed=None, **over):
    """Inputs of one named config (with optional overrides of its fields)."""
    cfg = dict(CONFIGS[cfg_id])
    cfg.update(over)
    seed = seed_of(cfg_id) if seed is None else seed
    H, dk, dv = cfg["H"], cfg["dk"], cfg["dv"]
    if cfg["kind"] == "chunk":
        B, T = cfg["B"], cfg["T"]
        d = draw((B, T), H, dk, dv, io=cfg["io"], scale_q=cfg["scale_q"],
                 n_states=B if cfg["init_state"] else None, device=device,
                 seed=seed)
        d.update(cu_seqlens=None, lengths=[T] * B)
    elif cfg["kind"] == "varlen":
        lengths = cfg.get("lengths") or varlen_lengths(
            cfg["n_short"], cfg["len_lo"], cfg["len_hi"], cfg["long_len"],
            seed=seed)
        T = int(sum(lengths))
        d = draw((1, T), H, dk, dv, io=cfg["io"], scale_q=cfg["scale_q"],
                 n_states=len(lengths) if cfg["init_state"] else None,
                 device=device, seed=seed)
        cu = [0]
        for n in lengths:
            cu.append(cu[-1] + n)
        d.update(cu_seqlens=torch.tensor(cu, dtype=torch.int32, device=device),
                 lengths=list(lengths))
    else:  # decode: one token per sequence per step, `steps` steps
        N, S = cfg["N"], cfg["steps"]
        d = draw((S, N), H, dk, dv, io=cfg["io"], scale_q=cfg["scale_q"],
                 n_states=N if cfg["init_state"] else None, device=device,
                 seed=seed)
        d.update(cu_seqlens=None, lengths=[S] * N)
    d["cfg"] = cfg
    return d
