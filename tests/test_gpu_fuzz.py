"""Seeded random shapes and segment tables through the CUDA path, compared
with the oracle: ragged M/N/K, every segment mode, random widths (multiples of
32 over K; any widths over N with one group, multiples of 128 with one group
per output segment), with and without bias and SmoothQuant divisor."""
import numpy as np
import pytest
import torch

from w8a8_gemm_b200 import workloads as wl

from parity import (bf16_ulp_diff, gpu_run, oracle_acc, oracle_prep, oracle_y, rel_err_floor)

pytestmark = pytest.mark.gpu


def _random_layer(seed):
    rng = np.random.default_rng(1000 + seed)
    mode = int(rng.integers(0, 3))
    M = int(rng.integers(1, 320))
    if mode == wl.MODE_INPUT:
        widths = [32 * int(w) for w in rng.integers(1, 9, size=int(rng.integers(2, 7)))]
        K = sum(widths)
        offsets = [0] + list(np.cumsum(widths))
        N = int(rng.integers(1, 300))
        G = 1
    else:
        K = 16 * int(rng.integers(1, 40))
        if mode == wl.MODE_OUTPUT and rng.random() < 0.5:
            n_seg = int(rng.integers(2, 4))
            widths = [128 * int(w) for w in rng.integers(1, 3, size=n_seg)]
            G = n_seg
        else:
            n_seg = int(rng.integers(1, 4)) if mode == wl.MODE_OUTPUT else 1
            widths = [int(w) for w in rng.integers(1, 200, size=n_seg)]
            G = 1
        N = sum(widths)
        offsets = [0] + list(np.cumsum(widths)) if mode == wl.MODE_OUTPUT else [0, K]
    g = torch.Generator().manual_seed(seed)
    sigma = torch.exp(torch.rand(K, generator=g) * 3 - 1.5)
    x = (torch.randn(M, K, generator=g) * sigma).to(torch.bfloat16)
    x_cal = (torch.randn(32, K, generator=g) * sigma).to(torch.bfloat16)
    if rng.random() < 0.5:       # GELU-like skew on half of the cases
        x = torch.nn.functional.gelu(x.float()).to(torch.bfloat16)
        x_cal = torch.nn.functional.gelu(x_cal.float()).to(torch.bfloat16)
    w = (torch.randn(N, K, generator=g) * 0.05).to(torch.bfloat16)
    bias = (torch.randn(N, generator=g) * 0.1).to(torch.bfloat16) if rng.random() < 0.7 else None
    d = (torch.rand(G, K, generator=g) * 1.5 + 0.5) if rng.random() < 0.5 else None
    return wl.Layer(f"fuzz{seed}", x, x_cal, w, bias, d, mode, [int(v) for v in offsets], G)


@pytest.mark.parametrize("seed", range(24))
def test_random_shapes(seed):
    L = _random_layer(seed)
    prep = oracle_prep(L)
    g = gpu_run(L, out_dtype=torch.float32, s32=True)
    assert np.array_equal(g["s_act"].cpu().numpy(), prep["s_act"])
    assert np.array_equal(g["wq"].cpu().numpy(), prep["wq"])
    assert np.array_equal(g["s_w"].cpu().numpy(), prep["s_w"])
    assert np.array_equal(g["planes"].cpu().numpy(), prep["planes"])
    assert np.array_equal(g["acc"].cpu().numpy(), oracle_acc(L, prep))
    r = oracle_y(L, prep)
    y = g["y"].cpu().numpy()
    assert rel_err_floor(y, r) <= 1e-3
    assert np.array_equal(y, r)
    gb = gpu_run(L, out_dtype=torch.bfloat16)
    assert bf16_ulp_diff(gb["y"], r) == 0
