"""The roofline numerators bench.py reports: the algorithmic bytes of a
prefill and of a decode step against the sizes of the tensors one call
actually reads and writes, and the per-launch flop count against the sum of
2 m n k over the chunk products the fused kernel issues."""
import sys
import os

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402
import kda_workloads as W  # noqa: E402


def nbytes(*ts):
    return sum(t.numel() * t.element_size() for t in ts if t is not None)


@pytest.mark.parametrize("B,T,H,dk,dv,io,state", [
    (2, 96, 3, 64, 64, "bf16", False), (1, 40, 2, 32, 128, "f32", True),
    (2, 8192, 32, 128, 128, "bf16", False)])
def test_prefill_bytes_are_the_tensors_touched(B, T, H, dk, dv, io, state):
    if T * H * dk > 10 ** 6:  # the headline shape: count from shapes alone
        esz = 2
        expect = (B * T * H * (2 * dk + 2 * dv) * esz + B * T * H * dk * 4 +
                  B * T * H * 4 + B * H * dk * dv * 4)
        assert expect == 811_597_824
    else:
        d = W.draw((B, T), H, dk, dv, io=io, n_states=B if state else None,
                   seed=1)
        out = torch.empty_like(d["v"])
        fin = torch.empty((B, H, dk, dv), dtype=torch.float32)
        expect = nbytes(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"],
                        d["initial_state"], out, fin)
    got = bench.prefill_bytes(B, T, H, dk, dv, io_bytes=2 if io == "bf16" else 4,
                              init_state=state)
    assert got == expect


def test_decode_bytes_are_the_tensors_touched():
    N, H, d = 5, 3, 64
    x = W.draw((N, 1), H, d, d, io="bf16", n_states=N, seed=2)
    out = torch.empty_like(x["v"])
    state = x["initial_state"]
    expect = nbytes(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], out) + \
        2 * nbytes(state)  # the state is read and written in place
    assert bench.decode_bytes(N, H, d, d) == expect
    assert bench.decode_bytes(256, 32, 128, 128) == 1_086_357_504


def test_prefill_flops_are_the_chunk_products():
    # per chunk of C tokens and head: [Kt; Qt] Kb^T (2C x C x dk), W = T' Kt
    # (C x dk x C), U = T' V (C x dv x C), [W; Qt] S (2C x dv x dk),
    # S += Kb^T Delta (dk x dv x C), P Delta (C x dv x C)
    B, T, H, dk, dv, C = 2, 8192, 32, 128, 128, 64
    products = [(2 * C, C, dk), (C, dk, C), (C, dv, C), (2 * C, dv, dk),
                (dk, dv, C), (C, dv, C)]
    per_chunk = sum(2 * m * n * k for m, n, k in products)
    expect = B * H * (T // C) * per_chunk
    assert bench.prefill_flops(B, T, H, dk, dv, C) == expect == 94_489_280_512


def test_twopass_design_bytes_count_the_package_round_trip():
    # package: [W; Q~] panels (64 tokens x 64 channels, bf16, both halves),
    # Kb (two 8 KiB panels), P and T' (64 x 64 bf16), and the vector of
    # exp(g_C - rho), exp(rho) per channel plus the rho flag and padding
    for dk in (64, 128):
        panels = (dk // 64) * 2 * 64 * 64 * 2
        expect = panels + 2 * 64 * 64 * 2 + 2 * (64 * 64 * 2) + (2 * dk + 4) * 4
        assert bench.twopass_package_bytes(dk) == expect
    assert bench.twopass_package_bytes(128) == 66_576
    B, T, H, dk, dv = 2, 8192, 32, 128, 128
    d = W.make(2, device="cpu")
    inputs = nbytes(d["q"], d["k"], d["log_alpha"], d["beta"])
    packages = B * (T // 64) * H * 66_576
    out = torch.empty(B, T, H, dv, dtype=torch.bfloat16)
    fin = torch.empty(B, H, dk, dv, dtype=torch.float32)
    f, c = bench.twopass_design_bytes(B, T, H, dk, dv)
    assert f == inputs + packages
    assert c == packages + nbytes(d["v"], out, fin)
    assert f + c == 1_902_379_008
