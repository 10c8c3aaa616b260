"""The dtype boundary of a quantized base model (mlora_apply_ex), against the oracle.

Page "Multi-LoRA Serving: adapter batching", section "The dtype boundary between a
quantized base model and LoRA": the LoRA branch may read the FP8 activation codes the
base GEMM reads (value = code * per-tensor scale) instead of the activation from before
quantization, and adds once onto the base GEMM's output in that output's own dtype
(bf16, fp16 or fp32).  Each case runs the CUDA path through the C ABI and compares
every row with the fp64 oracle given the exact input values (decoded FP8 codes times
the scale, the base output's exact values): |gpu - oracle| <= 1e-2 (1 + |oracle|);
rows without a delta must keep Y0's bits.
"""
import numpy as np
import pytest
import torch

import oracle
import segmented_rank_gemm_02_b200 as mlora
import workloads as wl
from gpu_harness import DEVICE, RTOL, free
from segmented_rank_gemm_02_b200 import staging

pytestmark = pytest.mark.gpu

TORCH_Y = {"bf16": torch.bfloat16, "f16": torch.float16, "f32": torch.float32}


def _fp8_codes(X_bits):
    """FP8 e4m3 codes of a bf16 activation with one per-tensor scale (amax / 448), as the
    quantized base GEMM would read it; returns (codes tensor on the device, scale)."""
    x = mlora.as_bf16_tensor(X_bits, DEVICE).float()
    scale = float(x.abs().max().item()) / 448.0
    codes = (x / scale).to(torch.float8_e4m3fn)
    return codes, scale


def _y_values(Y):
    """Exact values of a device Y (bf16, fp16 or fp32) as float64 numpy."""
    if Y.dtype == torch.bfloat16:
        return oracle.bf16_to_f64(mlora.bf16_bits(Y))
    if Y.dtype == torch.float16:
        return oracle.f16_to_f64(Y.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16))
    return Y.detach().cpu().double().numpy()


def _run(W, proj, x_kind, y_kind, Y0_override=None):
    st = staging.upload(W, proj, DEVICE)
    if x_kind == "fp8":
        X, x_scale = _fp8_codes(proj.X)
        X_ref = oracle.e4m3_to_f64(X.view(torch.uint8).cpu().numpy()) * x_scale
    else:
        X, x_scale = st["X"], 1.0
        X_ref = oracle.bf16_to_f64(proj.X)
    Y = st["Y"].to(TORCH_Y[y_kind]) if Y0_override is None else Y0_override
    Y0_vals = _y_values(Y)
    Y0_bits = Y.detach().cpu().clone()
    mlora.apply_ex(st["pool"], st["segs"], X, Y, x_scale=x_scale)
    assert st["pool"].check() == 0
    got = _y_values(Y)
    ref, flags = oracle.apply_rows_xf64(X_ref, Y0_vals, W.row_slot, None, W.slot_rank, W.slot_alpha,
                                        proj.A, proj.B)
    assert flags == 0
    err = np.abs(got - ref)
    bad = err > RTOL * (1 + np.abs(ref))
    assert not bad.any(), (f"{x_kind}/{y_kind}: {int(bad.sum())} elements out of tolerance, worst "
                           f"{float((err / (1 + np.abs(ref))).max())}")
    base = np.nonzero(W.row_slot < 0)[0]
    if base.size:
        assert torch.equal(Y.detach().cpu()[base], Y0_bits[base]), "rows without a delta changed"
    del st
    return float((err / (RTOL * (1 + np.abs(ref)))).max())


COMBOS = [("bf16", "f16"), ("bf16", "f32"), ("fp8", "bf16"), ("fp8", "f16"), ("fp8", "f32")]


@pytest.mark.parametrize("x_kind,y_kind", COMBOS)
@pytest.mark.parametrize("cfg", [2, 3, 5])
def test_dtype_boundary_workloads(cfg, x_kind, y_kind):
    W = wl.make_small(cfg)
    worst = _run(W, W.projection(0), x_kind, y_kind)
    assert worst < 1.0
    free()


@pytest.mark.parametrize("x_kind,y_kind", [("fp8", "f16"), ("bf16", "f32")])
def test_dtype_boundary_ranks_and_ragged_widths(x_kind, y_kind):
    # every rank bucket in one pool, odd ranks, d_out not a multiple of 32
    W = wl.random_case(21, 70, 96, 200, 6, (1, 7, 12, 24, 40, 64))
    _run(W, W.projection(0), x_kind, y_kind)
    free()


@pytest.mark.parametrize("out", ["f16", "f32"])
def test_fp8_base_gemm_output_and_codes(out):
    # a real FP8 base GEMM (e4m3 weights and activations, per-tensor scales) producing an
    # fp16 / fp32 Y0; the LoRA branch reads the same FP8 codes and adds onto that output
    W = wl.make_small(2)
    proj = W.projection(0)
    X, x_scale = _fp8_codes(proj.X)
    g = torch.Generator().manual_seed(3)
    w = (torch.randn(proj.d_out, proj.d_in, generator=g) * 0.02).to(DEVICE)
    w_scale = float(w.abs().max().item()) / 448.0
    w8 = (w / w_scale).to(torch.float8_e4m3fn)
    Y0 = torch._scaled_mm(X, w8.t(), scale_a=torch.tensor(x_scale, device=DEVICE),
                          scale_b=torch.tensor(w_scale, device=DEVICE), out_dtype=TORCH_Y[out])
    _run(W, proj, "fp8", out, Y0_override=Y0.contiguous())
    free()


def test_dtype_boundary_argument_errors():
    W = wl.make_small(2)
    proj = W.projection(0)
    st = staging.upload(W, proj, DEVICE)
    X8, scale = _fp8_codes(proj.X)
    # FP8 X needs rows of 16-byte vectors: a row stride of 4104 codes is refused
    Xbad = torch.zeros((W.n_rows, proj.d_in + 8), dtype=torch.float8_e4m3fn, device=DEVICE)[:, :proj.d_in]
    Y = st["Y"].float()
    with pytest.raises(mlora.MloraError) as e:
        mlora.apply_ex(st["pool"], st["segs"], Xbad, Y, x_scale=scale)
    assert e.value.status == mlora.ERR_INVALID_ARG
    with pytest.raises(mlora.MloraError) as e:
        mlora.apply_ex(st["pool"], st["segs"], X8, Y, x_scale=float("nan"))
    assert e.value.status == mlora.ERR_INVALID_ARG
    with pytest.raises(ValueError):
        mlora.apply_ex(st["pool"], st["segs"], X8, Y.to(torch.float64), x_scale=scale)
    torch.cuda.synchronize()
    assert torch.equal(Y, st["Y"].float())
    del st
    free()
