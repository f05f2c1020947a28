"""The no-allocation host entry point, sq_dualscale_seglinear_host_noalloc.

It exists for callers that may not allocate device memory (a plug-in inside
an application that owns the device-memory budget, a latency-critical loop
that cannot take cudaMalloc's and cudaFree's device-wide synchronisation, a
process at the edge of the device's memory).  It runs one layer from host rows
to host rows through the library's fixed device scratch instead of a
caller-provided workspace.

The GPU test calls it through the C ABI twice in a row, on two different
layers, without synchronising between the calls: the second call reuses the
scratch the first one left behind.  Both outputs must equal, bit for bit, those
of the pipelined entry point sq_dualscale_seglinear_host on the same inputs
(rows are independent, so chunking cannot change a result).  The first layer
needs several scratch chunks and ends in a ragged one.

This file is named so that pytest collects it last; the test also passes when
run alone in a fresh process.
"""
import ctypes

import pytest
import torch

from w8a8_gemm_b200 import binding as B
from w8a8_gemm_b200 import build as sqbuild
from w8a8_gemm_b200 import workloads as wl


def _noalloc_layers():
    # 12288 bytes per row of scratch at K = N = 1536: 2688 rows per chunk, so
    # 6000 rows take three chunks, the last one ragged.
    big = wl.gelu_layer("noalloc_big", 6000, 1536, 1536, seed=71, bias=True)
    # an input-segmented layer (per-head divisors and steps), one chunk
    heads = wl.outproj_layer("noalloc_heads", 333, 448, 264, 64, seed=72)
    return big, heads


def _device_inputs(L):
    """Weight codes, weight steps and activation steps from the library's own
    offline calls, as a user of the host entry points would hold them."""
    from parity import segments
    dev = torch.device("cuda")
    seg = segments(L)
    d = None if L.d is None else L.d.to(dev)
    wq = torch.empty(L.N, L.K, dtype=torch.int8, device=dev)
    s_w = torch.empty(L.S, L.N, dtype=torch.float32, device=dev)
    B.sq_quantize_weight_seg(L.w.to(dev), d, seg, wq, s_w)
    s_act = torch.empty(L.G, L.S, 2, dtype=torch.float32, device=dev)
    B.sq_calibrate_act(L.x_cal.to(dev), d, seg, s_act)
    bias = None if L.bias is None else L.bias.to(dev)
    return seg, d, wq, s_w, s_act, bias


@pytest.mark.gpu
def test_noalloc_equals_pipeline_on_two_calls_in_a_row():
    sqbuild.build()
    layers = _noalloc_layers()
    prepared = [_device_inputs(L) for L in layers]
    outs = []
    # two calls in a row, no synchronisation in between
    for L, (seg, d, wq, s_w, s_act, bias) in zip(layers, prepared):
        x_host = L.x.contiguous().pin_memory()
        y_host = torch.full((L.M, L.N), float("nan"), dtype=torch.float32).pin_memory()
        B.sq_dualscale_seglinear_host_noalloc(x_host, d, s_act, wq, s_w, bias, y_host, seg)
        outs.append(y_host)
    torch.cuda.current_stream().synchronize()
    assert B.sq_get_device_status() == 0
    for L, (seg, d, wq, s_w, s_act, bias), y in zip(layers, prepared, outs):
        pl = B.HostPipeline(256, L.K, L.N, max_G=L.G, max_P=seg.P)
        ref = torch.full((L.M, L.N), float("nan"), dtype=torch.float32).pin_memory()
        B.sq_dualscale_seglinear_host(pl, L.x.contiguous().pin_memory(), d, s_act, wq, s_w, bias,
                                      ref, seg)
        torch.cuda.current_stream().synchronize()
        pl.close()
        assert not torch.isnan(ref).any()
        assert torch.equal(y, ref), L.name


def test_noalloc_rejects_rows_larger_than_the_scratch():
    """One row of x (2K bytes), its two planes (2K) and its output (4 bytes per
    column) must fit the fixed scratch; otherwise SQ_ERR_TOO_LARGE, before any
    pointer is looked at or anything is enqueued (no GPU needed)."""
    sqbuild.build()
    L = B.lib()
    seg = B.Segments(B.SQ_SEG_NONE, None, 1, 0)
    cs, keep = seg._c()
    p = ctypes.c_void_p
    K = B.SQ_NOALLOC_SCRATCH_BYTES // 4   # 4K bytes per row: exactly the scratch
    rc = L.sq_dualscale_seglinear_host_noalloc(p(0), 1, K, K, p(0), p(0), p(0), p(0), p(0),
                                               p(0), B.SQ_OUT_F32, 16, 16, ctypes.byref(cs),
                                               p(0))
    assert rc == -8 and B.status_string(rc).startswith("SQ_ERR_TOO_LARGE")
