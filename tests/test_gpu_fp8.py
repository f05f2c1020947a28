"""FP8 (E4M3) DualScale through the CUDA path against the oracle: calibrated
steps, E4M3 planes and weights bit-exact; the tensor core's fp32 sums of the
(exact) E4M3 products within 2^-20 of the sum of |products| of the exact sums
(any fp32 summation order is far inside this); outputs within the fp32 bar
(and bf16 within it widened by one bf16 ulp)."""
import numpy as np
import pytest
import torch

from w8a8_gemm_b200 import workloads as wl

from parity import (bf16_close, gpu_run, oracle_acc_fp8, oracle_prep, oracle_y, rel_err_floor,
                    sample_rows)

pytestmark = pytest.mark.gpu

LAYERS = {
    "none_tails": lambda: wl.gelu_layer("none", 300, 416, 520, seed=41, bias=True),
    "none_ragged": lambda: wl.gelu_layer("rag", 5, 48, 13, seed=42, bias=True),
    "input_heads": lambda: wl.outproj_layer("heads", 300, 448, 264, 64, seed=43),
    "input_odd_n": lambda: wl.outproj_layer("oddn", 150, 256, 261, 64, seed=45),
    "output_groups": lambda: wl.adanorm_layer("og", 130, 256, 768, 3, seed=44, G=3),
}


def _check_acc(L, prep, acc_bits):
    acc = acc_bits.cpu().numpy().view(np.float32)
    exact = oracle_acc_fp8(L, prep)
    bound = oracle_acc_fp8(L, prep, absolute=True).astype(np.float64) * 2.0 ** -20
    assert np.all(np.abs(acc.astype(np.float64) - exact) <= bound + 1e-30)


@pytest.mark.parametrize("single", [False, True])
@pytest.mark.parametrize("name", sorted(LAYERS))
def test_fp8_layers_against_oracle(name, single):
    L = LAYERS[name]()
    prep = oracle_prep(L, single, fp8=True)
    g = gpu_run(L, out_dtype=torch.float32, s32=True, single=single, fp8=True)
    assert np.array_equal(g["s_act"].cpu().numpy(), prep["s_act"])
    assert np.array_equal(g["s_w"].cpu().numpy(), prep["s_w"])
    assert np.array_equal(g["wq"].cpu().numpy().view(np.uint8), prep["wq"])
    assert np.array_equal(g["planes"].cpu().numpy().view(np.uint8), prep["planes"])
    _check_acc(L, prep, g["acc"])
    r = oracle_y(L, prep)
    assert rel_err_floor(g["y"].cpu().numpy(), r) <= 1e-3
    gb = gpu_run(L, out_dtype=torch.bfloat16, single=single, fp8=True)
    assert bf16_close(gb["y"], r)


def test_fp8_every_bf16_value_quantizes_like_oracle():
    """All 65536 bf16 patterns through the FP8 quantizer (one row of K = 65536
    channels) with steps that put the codes across the whole E4M3 range."""
    bits = torch.arange(65536, dtype=torch.int32).to(torch.int16).view(torch.bfloat16)
    x = bits.reshape(1, 65536)
    x_cal = torch.tensor([[300.0, -0.5] + [0.0] * 65534], dtype=torch.bfloat16)
    L = wl.Layer("allbf16", x, x_cal, torch.ones(16, 65536, dtype=torch.bfloat16), None, None,
                 wl.MODE_NONE, [0, 65536], 1)
    prep = oracle_prep(L, fp8=True)
    g = gpu_run(L, fp8=True)
    assert np.array_equal(g["s_act"].cpu().numpy(), prep["s_act"])
    assert np.array_equal(g["planes"].cpu().numpy().view(np.uint8), prep["planes"])


def test_fp8_full_size_ffn_sampled_rows():
    for L in wl.config_layers("c4_sd35_ffn", seed=0):
        prep = oracle_prep(L, fp8=True)
        g = gpu_run(L, out_dtype=torch.bfloat16, fp8=True)
        assert np.array_equal(g["planes"].cpu().numpy().view(np.uint8), prep["planes"])
        assert np.array_equal(g["wq"].cpu().numpy().view(np.uint8), prep["wq"])
        rows = sample_rows(L.M)
        r = oracle_y(L, prep, rows=rows)
        assert bf16_close(g["y"][torch.from_numpy(rows).cuda()], r)
        del g
        torch.cuda.empty_cache()
