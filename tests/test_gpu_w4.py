"""W4A8 ("SegQuant-4") through the CUDA path against the oracle: packed 4-bit
weight codes and their scales bit-exact, the expanded GEMM operand equal to
16 x the codes, raw accumulators equal to 16 x the oracle's, and outputs held
to the same bar as W8A8 (fp32 bit-exact and bf16 = RNE of the oracle, for
every segment mode)."""
import numpy as np
import pytest
import torch

from w8a8_gemm_b200 import workloads as wl

from parity import (bf16_ulp_diff, gpu_run, oracle_acc, oracle_prep, oracle_y, rel_err_floor, sample_rows)

pytestmark = pytest.mark.gpu

LAYERS = {
    "none_tails": lambda: wl.gelu_layer("none", 300, 416, 520, seed=21, bias=True),
    "none_ragged": lambda: wl.gelu_layer("rag", 5, 48, 13, seed=22, bias=True),
    "input_heads": lambda: wl.outproj_layer("heads", 300, 448, 264, 64, seed=23),
    "input_odd_n": lambda: wl.outproj_layer("oddn", 150, 256, 261, 64, seed=26),
    "output_g1": lambda: wl.adanorm_layer("o1", 200, 256, 768, 3, seed=24, G=1),
    "output_groups": lambda: wl.adanorm_layer("og", 130, 256, 768, 3, seed=25, G=3),
}


@pytest.mark.parametrize("single", [False, True])
@pytest.mark.parametrize("name", sorted(LAYERS))
def test_w4_layers_against_oracle(name, single):
    L = LAYERS[name]()
    prep = oracle_prep(L, single, weight_bits=4)
    g = gpu_run(L, out_dtype=torch.float32, s32=True, single=single, weight_bits=4)
    assert np.array_equal(g["wq"].cpu().numpy(), prep["wq4"])
    assert np.array_equal(g["s_w"].cpu().numpy(), prep["s_w"])
    assert np.array_equal(g["wq16"].cpu().numpy(), 16 * prep["wq"].astype(np.int32))
    assert np.array_equal(g["planes"].cpu().numpy(), prep["planes"])
    assert np.array_equal(g["acc"].cpu().numpy(), 16 * oracle_acc(L, prep))
    r = oracle_y(L, prep)
    y = g["y"].cpu().numpy()
    assert rel_err_floor(y, r) <= 1e-3
    assert np.array_equal(y, r)
    gb = gpu_run(L, out_dtype=torch.bfloat16, single=single, weight_bits=4)
    assert bf16_ulp_diff(gb["y"], r) == 0


def test_w4_full_size_ffn_sampled_rows():
    """The SD3.5-medium FFN pair with W4A8 weights at full size."""
    for L in wl.config_layers("c4_sd35_ffn", seed=0):
        prep = oracle_prep(L, weight_bits=4)
        g = gpu_run(L, out_dtype=torch.bfloat16, weight_bits=4)
        assert np.array_equal(g["wq"].cpu().numpy(), prep["wq4"])
        assert np.array_equal(g["s_w"].cpu().numpy(), prep["s_w"])
        rows = sample_rows(L.M)
        r = oracle_y(L, prep, rows=rows)
        assert bf16_ulp_diff(g["y"][torch.from_numpy(rows).cuda()], r) == 0
        del g
        torch.cuda.empty_cache()
