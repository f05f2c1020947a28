"""The host-to-host entry point (chunked rows, copies overlapped with the
kernels on three streams) against the device calls on the whole layer: rows
are independent in both kernels, so the outputs must be identical bit for
bit, for ragged chunk counts, strided host rows, every segment mode, single
scale and W4A8 weights."""
import numpy as np
import pytest
import torch

from w8a8_gemm_b200 import binding as B
from w8a8_gemm_b200 import workloads as wl

from parity import gpu_run, oracle_prep, oracle_y, segments

pytestmark = pytest.mark.gpu

LAYERS = {
    "none_tails": lambda: wl.gelu_layer("none", 300, 416, 520, seed=31, bias=True),
    "input_heads": lambda: wl.outproj_layer("heads", 300, 448, 264, 64, seed=32),
    "output_groups": lambda: wl.adanorm_layer("og", 300, 256, 768, 3, seed=33, G=3),
    "one_row": lambda: wl.gelu_layer("one", 1, 64, 40, seed=34, bias=True),
}


def _host_run(L, g, out_dtype, single, weight_bits, chunk_rows, pad_x=0, pad_y=0):
    seg = segments(L, single, weight_bits)
    wq = g["wq16"] if weight_bits == 4 else g["wq"]
    pl = B.HostPipeline(chunk_rows, L.K, L.N, max_G=L.G, max_P=seg.P)
    x_host = torch.zeros(L.M, L.K + pad_x, dtype=torch.bfloat16).pin_memory()
    x_host[:, :L.K] = L.x
    y_host = torch.full((L.M, L.N + pad_y), float("nan"), dtype=out_dtype).pin_memory()
    d = None if L.d is None else L.d.cuda()
    bias = None if L.bias is None else L.bias.cuda()
    B.sq_dualscale_seglinear_host(pl, x_host[:, :L.K], d, g["s_act"], wq, g["s_w"], bias,
                                  y_host[:, :L.N], seg)
    torch.cuda.current_stream().synchronize()
    assert B.sq_get_device_status() == 0
    pl.close()
    if pad_y:
        assert torch.isnan(y_host[:, L.N:].float()).all()   # nothing written past N
    return y_host[:, :L.N]


@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("name", sorted(LAYERS))
def test_host_path_equals_device_path(name, out_dtype):
    L = LAYERS[name]()
    g = gpu_run(L, out_dtype=out_dtype)
    y = _host_run(L, g, out_dtype, False, 8, chunk_rows=128, pad_x=16, pad_y=3)
    assert torch.equal(y.view(torch.int16) if out_dtype == torch.bfloat16 else y,
                       g["y"].cpu().view(torch.int16) if out_dtype == torch.bfloat16
                       else g["y"].cpu())


@pytest.mark.parametrize("single,weight_bits", [(True, 8), (False, 4), (True, 4)])
def test_host_path_single_scale_and_w4(single, weight_bits):
    L = LAYERS["none_tails"]()
    g = gpu_run(L, out_dtype=torch.float32, single=single, weight_bits=weight_bits)
    y = _host_run(L, g, torch.float32, single, weight_bits, chunk_rows=64)
    assert torch.equal(y, g["y"].cpu())
    # and the oracle, directly
    prep = oracle_prep(L, single, weight_bits=weight_bits)
    assert np.array_equal(y.numpy(), oracle_y(L, prep))


def test_host_path_empty_batch_is_noop():
    L = LAYERS["none_tails"]()
    g = gpu_run(L)
    seg = segments(L)
    pl = B.HostPipeline(128, L.K, L.N)
    x = torch.empty(0, L.K, dtype=torch.bfloat16).pin_memory()
    y = torch.empty(0, L.N, dtype=torch.float32).pin_memory()
    B.sq_dualscale_seglinear_host(pl, x, None, g["s_act"], g["wq"], g["s_w"], None, y, seg)
    torch.cuda.synchronize()
    pl.close()


def test_host_calls_on_two_streams_do_not_race_on_the_workspace():
    """Two calls on one pipeline, each on its own stream, with no ordering
    between the streams: the second call's first chunks reuse the workspace
    slots the first call's last chunks used, and must wait for them.  Both
    outputs must still equal the device path's bit for bit."""
    La = wl.gelu_layer("race_a", 700, 416, 520, seed=41, bias=True)
    Lb = wl.gelu_layer("race_b", 700, 416, 520, seed=42, bias=True)
    ga, gb = gpu_run(La), gpu_run(Lb)
    seg = segments(La)
    pl = B.HostPipeline(64, La.K, La.N)
    outs = []
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    for L, g, st in ((La, ga, streams[0]), (Lb, gb, streams[1])):
        x_host = L.x.contiguous().pin_memory()
        y_host = torch.full((L.M, L.N), float("nan"), dtype=torch.float32).pin_memory()
        with torch.cuda.stream(st):
            B.sq_dualscale_seglinear_host(pl, x_host, None, g["s_act"], g["wq"], g["s_w"],
                                          L.bias.cuda(), y_host, seg)
        outs.append((x_host, y_host))
    torch.cuda.synchronize()
    assert B.sq_get_device_status() == 0
    pl.close()
    assert torch.equal(outs[0][1], ga["y"].cpu())
    assert torch.equal(outs[1][1], gb["y"].cpu())
