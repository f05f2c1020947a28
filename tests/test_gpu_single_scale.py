"""Single-scale path (SQ_FLAG_SINGLE_SCALE: DualScale only where activations are
strongly polarity-asymmetric, one merged plane elsewhere) against the oracle's
single-scale mode, and against the DualScale path run with s+ = s-."""
import numpy as np
import pytest
import torch

from w8a8_gemm_b200 import binding as B
from w8a8_gemm_b200 import workloads as wl

from parity import (bf16_ulp_diff, gpu_run, oracle_acc, oracle_prep, oracle_y, rel_err_floor, sample_rows, segments)

pytestmark = pytest.mark.gpu

LAYERS = {
    "none_tails": lambda: wl.gelu_layer("none", 300, 416, 520, seed=1, bias=True),
    "none_ragged": lambda: wl.gelu_layer("rag", 5, 48, 13, seed=3, bias=True),
    "input_heads": lambda: wl.outproj_layer("heads", 300, 448, 264, 64, seed=5),
    "input_odd_n": lambda: wl.outproj_layer("oddn", 150, 256, 261, 64, seed=15),
    "output_g3": lambda: wl.adanorm_layer("o3", 200, 256, 768, 3, seed=8, G=3),
    "output_g2_bn128": lambda: wl.adanorm_layer("o2", 130, 128, 256, 2, seed=9, G=2),
}


@pytest.mark.parametrize("name", sorted(LAYERS))
def test_single_scale_small(name):
    L = LAYERS[name]()
    prep = oracle_prep(L, single=True)
    g = gpu_run(L, out_dtype=torch.float32, s32=True, single=True)
    assert np.array_equal(g["s_act"].cpu().numpy(), prep["s_act"])
    assert np.array_equal(g["planes"].cpu().numpy(), prep["planes"])
    assert np.array_equal(g["acc"].cpu().numpy(), oracle_acc(L, prep))
    r = oracle_y(L, prep)
    y = g["y"].cpu().numpy()
    assert rel_err_floor(y, r) <= 1e-3
    assert np.array_equal(y, r)
    gb = gpu_run(L, out_dtype=torch.bfloat16, single=True)
    assert bf16_ulp_diff(gb["y"], r) == 0


def test_single_scale_equals_dualscale_with_equal_steps_on_gpu():
    """One merged plane and one product equal the DualScale planes and products
    run with s+ = s- (integer sums, bit for bit)."""
    L = wl.gelu_layer("eq", 260, 320, 300, seed=4, bias=True)
    g1 = gpu_run(L, out_dtype=torch.float32, s32=True, single=True)
    seg2 = segments(L)
    planes2 = torch.empty(1, 2, L.M, L.K, dtype=torch.int8, device="cuda")
    B.sq_quantize_act(L.x.cuda(), None, g1["s_act"], seg2, planes2)
    acc2 = torch.empty(1, 2, L.M, L.N, dtype=torch.int32, device="cuda")
    B.sq_debug_gemm_s32(planes2, g1["wq"], seg2, acc2)
    torch.cuda.synchronize()
    assert torch.equal(g1["planes"][:, 0].to(torch.int16),
                       planes2[:, 0].to(torch.int16) + planes2[:, 1])
    assert torch.equal(g1["acc"][:, 0].long(), acc2[:, 0].long() + acc2[:, 1])


def test_single_scale_full_size_ffn():
    for L in wl.config_layers("c4_sd35_ffn", seed=0):
        prep = oracle_prep(L, single=True)
        g = gpu_run(L, out_dtype=torch.bfloat16, single=True)
        assert np.array_equal(g["planes"].cpu().numpy(), prep["planes"])
        rows = sample_rows(L.M)
        r = oracle_y(L, prep, rows=rows)
        assert bf16_ulp_diff(g["y"][torch.from_numpy(rows).cuda()], r) == 0
