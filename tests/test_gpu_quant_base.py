"""The LoRA delta on top of a quantized base layer (page "Multi-LoRA Serving: adapter
batching", section "The dtype boundary between a quantized base model and LoRA").

The base GEMM runs on FP8 weights and activations (per-tensor scales, fp32
accumulation, bf16 output: torch._scaled_mm, the caller's GEMM); the LoRA branch
takes the activation from before its quantization (bf16) and bf16 adapters, and the
two paths meet once, on the base GEMM's bf16 output: Y = bf16(Y0 + s (X A^T) B^T).
The oracle receives the same Y0 (read back from the device), so the check isolates
the library's part.  The last test captures the whole layer in a CUDA graph: the
graph holds the pool's fixed slot addresses, so reloading a slot between replays
changes the adapter the replay applies, with no re-capture.
"""
import numpy as np
import pytest
import torch

import oracle
import segmented_rank_gemm_02_b200 as mlora
import workloads as wl
from gpu_harness import DEVICE, assert_close, assert_untouched, free
from segmented_rank_gemm_02_b200 import staging

pytestmark = pytest.mark.gpu

E4M3_MAX = 448.0


def fp8_base_layer(X, Wt):
    """Y0 = X W^T with X and W quantized to e4m3 (per-tensor scales), bf16 out."""
    sx = (X.float().abs().amax() / E4M3_MAX).clamp(min=1e-12)
    sw = (Wt.float().abs().amax() / E4M3_MAX).clamp(min=1e-12)
    Xq = (X.float() / sx).to(torch.float8_e4m3fn)
    Wq = (Wt.float() / sw).to(torch.float8_e4m3fn)
    return torch._scaled_mm(Xq, Wq.t(), scale_a=sx.reshape(()), scale_b=sw.reshape(()),
                            out_dtype=torch.bfloat16)


def base_weight(seed, d_out, d_in):
    g = torch.Generator(device="cpu").manual_seed(seed)
    return (torch.randn(d_out, d_in, generator=g) * 0.02).to(torch.bfloat16).to(DEVICE)


@pytest.mark.parametrize("n_rows,shuffle,base", [(208, True, 0.1), (640, False, 0.0)])
def test_delta_on_fp8_base_output(n_rows, shuffle, base):
    # scattered decode rows, and sorted rows whose segments take the long kernels
    W = wl.random_case(51, n_rows, 1024, 512, 5, (16, 64), base_frac=base, shuffle=shuffle)
    proj = W.projection(0)
    X = mlora.as_bf16_tensor(proj.X, DEVICE)
    Y = fp8_base_layer(X, base_weight(1, 512, 1024)).contiguous()
    torch.cuda.synchronize()
    Y0_bits = mlora.bf16_bits(Y)
    pool = staging.make_pool(1024, 512, W.n_slots, W.r_max, W.slot_rank, W.slot_alpha, proj.A, proj.B)
    segs = mlora.DeviceSegments(mlora.build_segments(W.row_slot, pool), W.n_rows, DEVICE)
    mlora.apply(pool, segs, X, Y)
    assert pool.check() == 0
    got = mlora.bf16_bits(Y)
    ref, flags = oracle.apply_rows(proj.X, Y0_bits, W.row_slot, None, W.slot_rank, W.slot_alpha,
                                   proj.A, proj.B)
    assert flags == 0
    assert_close(got, ref, "delta on the FP8 base output")
    assert_untouched(got, Y0_bits, np.nonzero(W.row_slot < 0)[0], "base rows")
    pool.close()
    free()


def test_graph_keeps_slot_addresses_across_reload():
    W = wl.random_case(52, 96, 512, 512, 3, (16,), base_frac=0.0)
    proj = W.projection(0)
    pool = staging.make_pool(512, 512, W.n_slots, W.r_max, W.slot_rank, W.slot_alpha, proj.A, proj.B)
    segs = mlora.DeviceSegments(mlora.build_segments(W.row_slot, pool), W.n_rows, DEVICE)
    X = mlora.as_bf16_tensor(proj.X, DEVICE)
    Wt = base_weight(2, 512, 512)
    Y = torch.empty(W.n_rows, 512, dtype=torch.bfloat16, device=DEVICE)
    stream = torch.cuda.Stream()

    def layer():
        Y.copy_(fp8_base_layer(X, Wt))
        mlora.apply(pool, segs, X, Y, stream=stream)

    with torch.cuda.stream(stream):
        layer()   # warm-up outside capture
    stream.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        layer()
    A, B = dict(proj.A), dict(proj.B)
    for round_ in range(2):
        if round_ == 1:
            # a new adapter in slot 1 (same rank): the captured graph now applies it
            rng = np.random.default_rng(7)
            A[1] = wl.f32_to_bf16_bits(rng.standard_normal((16, 512), dtype=np.float32) * 0.02)
            B[1] = wl.f32_to_bf16_bits(rng.standard_normal((512, 16), dtype=np.float32) * 0.02)
            pool.load_slot(1, 16, float(W.slot_alpha[1]), A[1], B[1])
            torch.cuda.synchronize()
        graph.replay()
        torch.cuda.synchronize()
        assert pool.check() == 0
        with torch.cuda.stream(stream):
            Y0 = fp8_base_layer(X, Wt)
        stream.synchronize()
        ref, flags = oracle.apply_rows(proj.X, mlora.bf16_bits(Y0), W.row_slot, None, W.slot_rank,
                                       W.slot_alpha, A, B)
        assert flags == 0
        assert_close(mlora.bf16_bits(Y), ref, f"replay {round_}")
    assert (W.row_slot == 1).any()
    del graph
    pool.close()
    free()
