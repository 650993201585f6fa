"""TSA on the GPU against the oracle, through the C ABI: the ego-motion
reference points, and the fused forward that averages the queues
("【论文阅读】BEVFormer论文解析及Temporal Self-Attention、Spatial
Cross-Attention注意力机制详解及代码示例", section 二.2 and the BEV encoder
listing).

Reference points are computed in double on both sides and rounded once to
fp32, so they agree to within an ulp of fp32 (1e-6 absolute covers that for
coordinates of magnitude up to 2).  The forward takes the oracle's fp32
reference points as input on both sides and uses the tolerances of every
MSDA parity test (1e-5 + 1e-5 |x| for fp32 value, 2e-2 for bf16).
"""
import numpy as np
import pytest
import torch

import oracle
import scale_deformable_attention_03_b200 as msda
from scale_deformable_attention_03_b200 import inputs

from .gpu_util import assert_close, dev

pytestmark = pytest.mark.gpu


def _ego(rng, B, T, shift_m=2.56, yaw_deg=15.0):
    """Random motion for every queue but the last (the current frame)."""
    ego = np.zeros((B, T, 3), np.float32)
    ego[:, :-1, :2] = rng.uniform(-shift_m, shift_m, (B, T - 1, 2))
    ego[:, :-1, 2] = rng.uniform(-yaw_deg, yaw_deg, (B, T - 1))
    return ego


@pytest.mark.parametrize("B,T,bev,grid", [
    (2, 2, (50, 70), (0.512, 0.512)),
    (1, 3, (200, 200), (0.512, 0.512)),
    (3, 1, (17, 9), (0.3, 0.7)),
])
def test_tsa_reference_points(B, T, bev, grid):
    rng = np.random.Generator(np.random.PCG64(70 + T))
    ego = _ego(rng, B, T)
    if T > 1:
        ego[0, 0] = (0.0, 0.0, 90.0)  # exact quarter turn
    ref = msda.tsa_reference_points(dev(ego), bev[0], bev[1], grid)
    torch.cuda.synchronize()
    want = oracle.tsa_reference_points(bev[0], bev[1], ego, grid)
    err = np.abs(ref.cpu().numpy().astype(np.float64) - want)
    assert err.max() <= 1e-6, err.max()


def _problem(seed, B, T, shapes, H, P, R, bf16, bev=None):
    rng = np.random.Generator(np.random.PCG64(seed))
    s, starts, Nv = inputs.level_table(shapes)
    L = len(shapes)
    bev = bev or shapes[0]
    Nq = bev[0] * bev[1]
    value = rng.standard_normal((B * T, Nv, H, 32)).astype(np.float32)
    bits = None
    if bf16:
        bits = inputs.to_bf16_bits(value)
        value = inputs.bf16_bits_to_f32(bits)
    ego = _ego(rng, B, T)
    ref = oracle.tsa_reference_points(bev[0], bev[1], ego).astype(np.float32)
    ref = np.repeat(ref.reshape(B * T, Nq, 1, 2), R, axis=2)  # R anchors at the cell
    ref[..., 1:, :] += rng.uniform(-0.02, 0.02, ref[..., 1:, :].shape).astype(np.float32)
    off = (rng.standard_normal((B * T, Nq, H, L, P, 2)) * 1.5).astype(np.float32)
    logits = rng.standard_normal((B * T, Nq, H, L, P)).astype(np.float32)
    vt = dev(bits.view(np.int16)).view(torch.bfloat16) if bf16 else dev(value)
    return s, starts, value, vt, ref, off, logits


CASES = [
    # seed, B, T, shapes, H, P, R: the config-4 layout (one level, 4 points), more
    # queues, several levels (32 and 36 samples per head: the per-head kernel), one head
    (80, 2, 2, [(23, 31)], 8, 4, 1),
    (81, 1, 1, [(16, 16)], 8, 4, 1),
    (82, 1, 3, [(12, 20)], 8, 4, 1),
    (83, 1, 4, [(9, 11)], 4, 2, 2),
    (84, 1, 2, [(20, 24), (10, 12), (5, 6), (3, 3)], 8, 8, 4),
    (85, 2, 2, [(14, 10), (7, 5), (4, 3)], 2, 12, 3),
    (86, 1, 2, [(15, 13)], 1, 4, 1),
    (87, 1, 2, [(40, 40), (20, 20)], 3, 8, 1),
]


@pytest.mark.parametrize("case", CASES, ids=[f"case{c[0]}" for c in CASES])
@pytest.mark.parametrize("bf16", [False, True])
def test_tsa_forward(case, bf16):
    seed, B, T, shapes, H, P, R = case
    s, starts, value, vt, ref, off, logits = _problem(seed, B, T, shapes, H, P, R, bf16)
    out = msda.tsa_forward(vt, s, starts, dev(ref), dev(off), dev(logits), T)
    torch.cuda.synchronize()
    want = oracle.tsa_forward(value, s, starts, ref, off, logits, T)
    assert_close(out, want, bf16, f"tsa_forward T={T}")


def test_tsa_forward_bevformer_base_full_size():
    """The TSA layer of BEVFormer-base: one BEV sample, the previous and the
    current 200x200 BEV, 8 heads, 4 points, ego motion from the reference
    point kernel's own inputs."""
    w = inputs.workload4()
    ego = np.array([[[1.7, -0.9, 4.0], [0.0, 0.0, 0.0]]], np.float32)
    ref = oracle.tsa_reference_points(200, 200, ego).astype(np.float32).reshape(2, -1, 1, 2)
    out = msda.tsa_forward(dev(w.value), w.spatial_shapes, w.level_start_index, dev(ref),
                           dev(w.sampling_offsets), dev(w.attention_logits), 2)
    torch.cuda.synchronize()
    want = oracle.tsa_forward(w.value, w.spatial_shapes, w.level_start_index, ref,
                              w.sampling_offsets, w.attention_logits, 2)
    assert_close(out, want, False, "tsa_forward 200x200")
    # the queue mean equals the mean of msda_forward_fused's per-queue rows
    per_queue = msda.msda_forward_fused(dev(w.value), w.spatial_shapes, w.level_start_index,
                                        dev(ref), dev(w.sampling_offsets),
                                        dev(w.attention_logits))
    mean = per_queue.mean(0, keepdim=True)
    torch.cuda.synchronize()
    assert torch.allclose(out, mean, rtol=1e-6, atol=1e-6)


def test_tsa_forward_empty():
    s, starts, _ = inputs.level_table([(4, 4)])
    v = torch.zeros((0, 16, 8, 32), device="cuda")
    z = torch.zeros((0, 16, 8, 1, 4, 2), device="cuda")
    out = msda.tsa_forward(v, s, starts, torch.zeros((0, 16, 1, 2), device="cuda"), z,
                           torch.zeros((0, 16, 8, 1, 4), device="cuda"), 2)
    assert out.shape == (0, 16, 256)


@pytest.mark.parametrize("case", CASES, ids=[f"case{c[0]}" for c in CASES])
@pytest.mark.parametrize("bf16", [False, True])
def test_tsa_backward(case, bf16):
    seed, B, T, shapes, H, P, R = case
    s, starts, value, vt, ref, off, logits = _problem(seed, B, T, shapes, H, P, R, bf16)
    Nq = ref.shape[1]
    go = np.random.Generator(np.random.PCG64(seed + 500)).standard_normal(
        (B, Nq, H * 32)).astype(np.float32)
    gv, g_off, g_lg, g_ref = msda.tsa_backward(vt, s, starts, dev(ref), dev(off), dev(logits), T,
                                               dev(go))
    torch.cuda.synchronize()
    rv, r_off, r_lg, r_ref = oracle.tsa_backward(value, s, starts, ref, off, logits, T, go)
    assert_close(gv, rv, False, "tsa grad_value")
    assert_close(g_off, r_off, False, "tsa grad_sampling_offsets")
    assert_close(g_lg, r_lg, False, "tsa grad_attention_logits")
    assert_close(g_ref, r_ref, False, "tsa grad_reference_points")


def test_tsa_backward_bevformer_base_full_size():
    w = inputs.workload4()
    ego = np.array([[[1.7, -0.9, 4.0], [0.0, 0.0, 0.0]]], np.float32)
    ref = oracle.tsa_reference_points(200, 200, ego).astype(np.float32).reshape(2, -1, 1, 2)
    go = np.random.Generator(np.random.PCG64(89)).standard_normal(
        (1, w.Nq, w.H * 32)).astype(np.float32)
    gv, g_off, g_lg, g_ref = msda.tsa_backward(dev(w.value), w.spatial_shapes,
                                               w.level_start_index, dev(ref),
                                               dev(w.sampling_offsets), dev(w.attention_logits),
                                               2, dev(go))
    torch.cuda.synchronize()
    rv, r_off, r_lg, r_ref = oracle.tsa_backward(w.value, w.spatial_shapes, w.level_start_index,
                                                 ref, w.sampling_offsets, w.attention_logits, 2,
                                                 go)
    assert_close(gv, rv, False, "tsa 200x200 grad_value")
    assert_close(g_off, r_off, False, "tsa 200x200 grad_sampling_offsets")
    assert_close(g_lg, r_lg, False, "tsa 200x200 grad_attention_logits")
    assert_close(g_ref, r_ref, False, "tsa 200x200 grad_reference_points")
