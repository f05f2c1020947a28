"""The balanced last wave of one-segment GEMMs (sq_dualscale_seglinear_gemm_ws,
sq_debug_gemm_s32_ws): the k-blocks of the last, partial wave's tiles are
shared out over all SMs, and the SM holding a tile's first k-block adds the
others' int32 partial sums before the epilogue.  Integer addition is exact, so
accumulators and outputs must equal the whole-tile schedule's bit for bit --
for tiles split over two SMs, over a dozen (one tail tile, 148 SMs), and for
tails whose pieces are whole tiles.  Every case runs twice on one workspace,
which must come back ready for the next call."""
import numpy as np
import pytest
import torch

from w8a8_gemm_b200 import binding as B
from w8a8_gemm_b200 import workloads as wl

from parity import oracle_acc, oracle_prep, sample_rows, segments

pytestmark = pytest.mark.gpu


def _layer(M, N, K, seed):
    return wl.gelu_layer(f"tail_{M}x{N}x{K}", M, K, N, seed=seed, bias=True)


def _prepare(L, single=False, fp8=False):
    dev = torch.device("cuda")
    seg = segments(L, single=single, fp8=fp8)
    wq = torch.empty(L.N, L.K, dtype=torch.int8, device=dev)
    s_w = torch.empty(L.S, L.N, device=dev)
    B.sq_quantize_weight_seg(L.w.to(dev), None, seg, wq, s_w)
    s_act = torch.empty(L.G, L.S, 2, device=dev)
    B.sq_calibrate_act(L.x_cal.to(dev), None, seg, s_act)
    planes = torch.empty(L.G, seg.P, L.M, L.K, dtype=torch.int8, device=dev)
    B.sq_quantize_act(L.x.to(dev), None, s_act, seg, planes)
    return seg, wq, s_w, s_act, planes, L.bias.to(dev)


# (M, N, K): tile counts 149 (one tail tile split over up to 12 SMs), 150 with
# ragged N and K = 6144 (two tail tiles), 222 (74 tail tiles, each over two
# SMs), and 152 with K = 128 (one k-block per tile: the tail pieces are whole
# tiles).
SHAPES = [(100, 149 * 256, 1536), (384, 50 * 256 - 40, 6144), (261, 74 * 256, 2048),
          (128 * 4, 38 * 256, 128)]


@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("single", [False, True])
def test_split_tail_accumulators_equal_whole_tiles(shape, single):
    M, N, K = shape
    L = _layer(M, N, K, seed=M + N + K)
    seg, wq, s_w, s_act, planes, bias = _prepare(L, single=single)
    ws = B.gemm_workspace()
    ref = torch.empty(1, seg.P, M, N, dtype=torch.int32, device="cuda")
    B.sq_debug_gemm_s32(planes, wq, seg, ref)
    for _ in range(2):
        acc = torch.full_like(ref, -7)
        B.sq_debug_gemm_s32(planes, wq, seg, acc, workspace=ws)
        torch.cuda.synchronize()
        assert B.sq_get_device_status() == 0
        assert torch.equal(acc, ref)


@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32])
def test_split_tail_outputs_equal_whole_tiles(shape, out_dtype):
    M, N, K = shape
    L = _layer(M, N, K, seed=M * 3 + N + K)
    seg, wq, s_w, s_act, planes, bias = _prepare(L)
    ws = B.gemm_workspace()
    ref = torch.empty(M, N, dtype=out_dtype, device="cuda")
    B.sq_dualscale_seglinear_gemm(planes, wq, s_w, s_act, bias, ref, seg)
    for _ in range(2):
        y = torch.full_like(ref, float("nan"))
        B.sq_dualscale_seglinear_gemm(planes, wq, s_w, s_act, bias, y, seg, workspace=ws)
        torch.cuda.synchronize()
        assert B.sq_get_device_status() == 0
        assert torch.equal(y.view(torch.int16) if out_dtype == torch.bfloat16 else y,
                           ref.view(torch.int16) if out_dtype == torch.bfloat16 else ref)


def test_split_tail_fp8_outputs_equal_whole_tiles():
    M, N, K = SHAPES[2]
    L = _layer(M, N, K, seed=91)
    seg, wq, s_w, s_act, planes, bias = _prepare(L, fp8=True)
    ws = B.gemm_workspace()
    ref = torch.empty(M, N, dtype=torch.float32, device="cuda")
    B.sq_dualscale_seglinear_gemm(planes, wq, s_w, s_act, bias, ref, seg)
    y = torch.full_like(ref, float("nan"))
    B.sq_dualscale_seglinear_gemm(planes, wq, s_w, s_act, bias, y, seg, workspace=ws)
    torch.cuda.synchronize()
    # FP8 partial sums are fp32: the split adds them in another order, so the
    # whole-tile result is matched within the accumulation bound, not bitwise.
    assert torch.allclose(y, ref, rtol=1e-5, atol=1e-5 * float(ref.abs().max()))


def test_split_tail_on_the_ffn_workload_against_the_oracle():
    """The SD3.5 FFN pair at full size (1680 and 420 tiles of 128 x 256 on 148
    SMs: both have a partial last wave): int32 accumulators of the balanced
    schedule equal the oracle's on the sampled rows, and the bf16 outputs
    equal the whole-tile schedule's everywhere."""
    ws = B.gemm_workspace()
    for L in wl.config_layers("c4_sd35_ffn", seed=0):
        seg, wq, s_w, s_act, planes, bias = _prepare(L)
        acc = torch.empty(1, 2, L.M, L.N, dtype=torch.int32, device="cuda")
        B.sq_debug_gemm_s32(planes, wq, seg, acc, workspace=ws)
        rows = sample_rows(L.M)
        prep = oracle_prep(L)
        assert np.array_equal(planes.cpu().numpy(), prep["planes"])
        got = acc[:, :, torch.from_numpy(rows).cuda()].cpu().numpy()
        assert np.array_equal(got, oracle_acc(L, prep, rows=rows)), L.name
        y0 = torch.empty(L.M, L.N, dtype=torch.bfloat16, device="cuda")
        y1 = torch.empty_like(y0)
        B.sq_dualscale_seglinear_gemm(planes, wq, s_w, s_act, bias, y0, seg)
        B.sq_dualscale_seglinear_gemm(planes, wq, s_w, s_act, bias, y1, seg, workspace=ws)
        torch.cuda.synchronize()
        assert B.sq_get_device_status() == 0
        assert torch.equal(y0.view(torch.int16), y1.view(torch.int16)), L.name
        del acc
        torch.cuda.empty_cache()
