"""The fused producer (sq_dualscale_seglinear_gemm_gelu_quant) against the
oracle: the next layer's planes must equal, bit for bit, the oracle's
DualScale quantization of bf16(gelu(bf16(y))), y being the oracle's fp32
output of this layer (the GPU's fp32 epilogue is bit-identical to it, and the
GELU and codes run the oracle's fp32 operations)."""
import numpy as np
import pytest
import torch

import oracle
from w8a8_gemm_b200 import binding as B
from w8a8_gemm_b200 import workloads as wl

from parity import gpu_run, oracle_prep, oracle_y, sample_rows

pytestmark = pytest.mark.gpu


def _steps_next(x2_bits):
    """Next layer's {s+, s-} from its input values (AMax, as calibration does)."""
    v = (x2_bits.astype(np.uint32) << 16).view(np.float32)
    hi, lo = float(v.max()), float(v.min())
    return np.array([np.float32(hi) / np.float32(127.0) if hi > 0 else 1.0,
                     np.float32(-lo) / np.float32(128.0) if lo < 0 else 1.0], np.float32)


def _run_fused(L, g, s_next, single_next, single):
    dev = torch.device("cuda")
    seg = B.Segments(flags=B.SQ_FLAG_SINGLE_SCALE) if single else B.Segments()
    pn = 1 if single_next else 2
    out = torch.full((1, pn, L.M, L.N), 77, dtype=torch.int8, device=dev)
    bias = None if L.bias is None else L.bias.to(dev)
    B.sq_dualscale_seglinear_gemm_gelu_quant(g["planes"], g["wq"], g["s_w"], g["s_act"], bias,
                                             seg, torch.from_numpy(s_next).to(dev), out,
                                             single_next=single_next)
    torch.cuda.synchronize()
    assert B.sq_get_device_status() == 0
    return out.cpu().numpy()


LAYERS = {
    "tails": lambda: wl.gelu_layer("fz", 300, 416, 528, seed=61, bias=True),
    "ragged_m": lambda: wl.gelu_layer("fr", 130, 256, 256, seed=62, bias=True),
    "no_bias": lambda: wl.gelu_layer("fn", 200, 160, 384, seed=63, bias=False),
}


@pytest.mark.parametrize("single_next", [False, True])
@pytest.mark.parametrize("single", [False, True])
@pytest.mark.parametrize("name", sorted(LAYERS))
def test_fused_planes_bitexact(name, single, single_next):
    L = LAYERS[name]()
    prep = oracle_prep(L, single)
    g = gpu_run(L, out_dtype=torch.float32, single=single)
    y = oracle_y(L, prep)
    assert np.array_equal(g["y"].cpu().numpy(), y)      # this layer's fp32 output
    x2 = oracle.gelu_bf16(y)
    s_next = _steps_next(x2)
    ref = oracle.quantize_act(x2, s_next.reshape(1, 1, 2), single=single_next)
    got = _run_fused(L, g, s_next, single_next, single)
    assert got.shape == ref.shape
    assert np.array_equal(got, ref)


def test_fused_full_size_ffn_sampled_rows():
    """SD3.5-medium fc1 (8858 x 1536 -> 6144) producing fc2's planes."""
    L = wl.config_layers("c4_sd35_ffn", seed=0)[0]
    prep = oracle_prep(L)
    g = gpu_run(L, out_dtype=torch.bfloat16)
    rows = sample_rows(L.M)
    y = oracle_y(L, prep, rows=rows)
    x2 = oracle.gelu_bf16(y)
    s_next = _steps_next(x2)
    ref = oracle.quantize_act(x2, s_next.reshape(1, 1, 2))
    got = _run_fused(L, g, s_next, False, False)
    assert np.array_equal(got[:, :, rows, :], ref)
