"""MSDA and SCA backward on the GPU against the oracle's analytic derivative
(itself pinned to central finite differences), through the C ABI.

grad_value is accumulated with fp32 atomics, so its summation order differs
from the oracle's; the fp32 tolerance still applies at these sizes.
Workload 5 (the BEVFormer-base SCA training step, bf16 value) runs at full
size against the 2e-2 bf16 bound.
"""
import numpy as np
import pytest
import torch

import oracle
import scale_deformable_attention_03_b200 as msda
from scale_deformable_attention_03_b200 import inputs

from .gpu_util import assert_close, dev, softmax_weights, value_tensor

pytestmark = pytest.mark.gpu


def _problem(seed, B, Nq, H, shapes, P, lo=-0.2, hi=1.2):
    rng = np.random.Generator(np.random.PCG64(seed))
    s, starts, Nv = inputs.level_table(shapes)
    L = len(shapes)
    value = rng.standard_normal((B, Nv, H, 32)).astype(np.float32)
    loc = rng.uniform(lo, hi, (B, Nq, H, L, P, 2)).astype(np.float32)
    weights = softmax_weights(rng.standard_normal((B, Nq, H, L, P)), L * P)
    gout = rng.standard_normal((B, Nq, H * 32)).astype(np.float32)
    return s, starts, value, loc, weights, gout


CASES = [
    (1, 1, 29, 1, [(5, 7)], 2),
    (2, 2, 300, 8, [(20, 30), (10, 15), (5, 8), (3, 4)], 4),
    (3, 1, 77, 2, [(6, 5), (3, 3), (1, 9)], 12),     # two chunks
    (4, 1, 40, 3, [(7, 9)] * 8, 16),                 # four chunks
    # rows of <= 16 samples take the head-group kernel: eight heads of four
    # samples per warp, a partial group (H = 5 in groups of four), padded
    # sample slots (3 of 4, 12 of 16)
    (5, 2, 53, 8, [(9, 11)], 4),
    (6, 1, 41, 5, [(6, 7), (3, 4)], 3),
    (7, 3, 37, 6, [(5, 9)], 3),
    (8, 1, 33, 2, [(4, 4), (2, 3), (3, 2)], 4),
]


@pytest.mark.parametrize("case", CASES, ids=[f"case{c[0]}" for c in CASES])
@pytest.mark.parametrize("bf16", [False, True])
def test_msda_backward_random(case, bf16):
    seed, B, Nq, H, shapes, P = case
    s, starts, value, loc, weights, gout = _problem(seed, B, Nq, H, shapes, P)
    if bf16:
        bits = inputs.to_bf16_bits(value)
        value = inputs.bf16_bits_to_f32(bits)
        vt = dev(bits.view(np.int16)).view(torch.bfloat16)
    else:
        vt = dev(value)
    gv, gl, gw = msda.msda_backward(vt, s, starts, dev(loc), dev(weights), dev(gout))
    torch.cuda.synchronize()
    rv, rl, rw = oracle.msda_backward(value, s, starts, loc, weights, gout)
    assert_close(gw, rw, False, "grad_attention_weights")
    assert_close(gl, rl, False, "grad_sampling_locations")
    assert_close(gv, rv, False, "grad_value")


def test_msda_backward_workload2():
    """The Deformable-DETR encoder at full size (all 19 947 queries)."""
    w = inputs.workload2()
    loc, weights = oracle.fused_locations(w.spatial_shapes, w.reference_points,
                                          w.sampling_offsets, w.attention_logits)
    loc, weights = loc.astype(np.float32), weights.astype(np.float32)
    gout = np.random.Generator(np.random.PCG64(5)).standard_normal(
        (1, w.Nq, w.H * 32)).astype(np.float32)
    gv, gl, gw = msda.msda_backward(dev(w.value), w.spatial_shapes, w.level_start_index,
                                    dev(loc), dev(weights), dev(gout))
    torch.cuda.synchronize()
    rv, rl, rw = oracle.msda_backward(w.value, w.spatial_shapes, w.level_start_index, loc,
                                      weights, gout)
    assert_close(gw, rw, False, "grad_attention_weights")
    assert_close(gl, rl, False, "grad_sampling_locations")
    assert_close(gv, rv, False, "grad_value")


def test_msda_backward_tsa_queues_full_size():
    """The two 200x200 TSA queues as a plain MSDA batch of two (workload 4),
    locations and weights from the oracle's fused location step."""
    w = inputs.workload4()
    loc, weights = oracle.fused_locations(w.spatial_shapes, w.reference_points,
                                          w.sampling_offsets, w.attention_logits)
    loc, weights = loc.astype(np.float32), weights.astype(np.float32)
    gout = np.random.Generator(np.random.PCG64(6)).standard_normal(
        (w.B, w.Nq, w.H * 32)).astype(np.float32)
    gv, gl, gw = msda.msda_backward(dev(w.value), w.spatial_shapes, w.level_start_index,
                                    dev(loc), dev(weights), dev(gout))
    torch.cuda.synchronize()
    rv, rl, rw = oracle.msda_backward(w.value, w.spatial_shapes, w.level_start_index, loc,
                                      weights, gout)
    assert_close(gw, rw, False, "tsa queues grad_attention_weights")
    assert_close(gl, rl, False, "tsa queues grad_sampling_locations")
    assert_close(gv, rv, False, "tsa queues grad_value")


def _sca_bwd(w, bf16):
    grads = msda.sca_backward(value_tensor(w, bf16), w.spatial_shapes, w.level_start_index,
                              dev(w.reference_points), dev(w.bev_mask), dev(w.sampling_offsets),
                              dev(w.attention_logits), dev(w.grad_out))
    torch.cuda.synchronize()
    ref = oracle.sca_backward(w.value, w.spatial_shapes, w.level_start_index, w.reference_points,
                              w.bev_mask, w.sampling_offsets, w.attention_logits, w.grad_out)
    return grads, ref


@pytest.mark.parametrize("seed,B,Ncam,bev,shapes,H,P,R", [
    (31, 2, 3, (7, 9), [(9, 13), (4, 7)], 2, 4, 2),
    (32, 1, 6, (30, 40), [(16, 20), (8, 10), (4, 5), (2, 3)], 8, 8, 4),
    (33, 2, 2, (5, 13), [(6, 7)] * 3, 1, 12, 3),
])
def test_sca_backward_random(seed, B, Ncam, bev, shapes, H, P, R):
    w = inputs.workload3(seed=seed, B=B, Ncam=Ncam, bev_h=bev[0], bev_w=bev[1], shapes=shapes,
                         H=H, P=P, R=R, rho="uniform", same_mask=False, with_grad=True)
    (gv, gl, gw), (rv, rl, rw) = _sca_bwd(w, False)
    assert_close(gw, rw, False, "grad_attention_weights_rb")
    assert_close(gl, rl, False, "grad_sampling_locations_rb")
    assert_close(gv, rv, False, "grad_value")


@pytest.mark.parametrize("case", ["no camera sees anything", "one camera blind",
                                  "every camera sees everything", "sixteen heads"])
@pytest.mark.parametrize("deterministic", [False, True])
def test_sca_backward_padding_rows(case, deterministic):
    """The rebatched gradients' rows count .. Nq-1 of every (batch, camera)
    hold no row and must come back zero: outputs pre-filled with NaN,
    compared with the oracle element by element, including the case with no
    rebatched row at all and a head count above the warps per CTA."""
    H, P, R = (16, 4, 2) if case == "sixteen heads" else (4, 4, 2)
    w = inputs.workload3(seed=35, B=2, Ncam=3, bev_h=9, bev_w=11, shapes=[(7, 9), (3, 4)],
                         H=H, P=P, R=R, rho="uniform", same_mask=False, with_grad=True)
    if case == "no camera sees anything":
        w.bev_mask[:] = 0
    elif case == "one camera blind":
        w.bev_mask[1] = 0
    elif case == "every camera sees everything":
        w.bev_mask[:] = 1
    B, Ncam, Nq, L = w.B, w.Ncam, w.Nq, w.L
    gl = torch.full((B, Ncam, Nq, H, L, P, 2), float("nan"), device="cuda")
    gw = torch.full((B, Ncam, Nq, H, L, P), float("nan"), device="cuda")
    gv, gl, gw = msda.sca_backward(dev(w.value), w.spatial_shapes, w.level_start_index,
                                   dev(w.reference_points), dev(w.bev_mask),
                                   dev(w.sampling_offsets), dev(w.attention_logits),
                                   dev(w.grad_out), grad_sampling_locations_rb=gl,
                                   grad_attention_weights_rb=gw, deterministic=deterministic)
    torch.cuda.synchronize()
    rv, rl, rw = oracle.sca_backward(w.value, w.spatial_shapes, w.level_start_index,
                                     w.reference_points, w.bev_mask, w.sampling_offsets,
                                     w.attention_logits, w.grad_out)
    assert_close(gw, rw, False, f"{case}: grad_attention_weights_rb")
    assert_close(gl, rl, False, f"{case}: grad_sampling_locations_rb")
    assert_close(gv, rv, False, f"{case}: grad_value")


def test_sca_backward_workload3_full_size():
    """The BEVFormer-base SCA backward with fp32 value (B = 1) at full size:
    the rebatched gradients and grad_value at the fp32 bound."""
    w = inputs.workload3(seed=1003, with_grad=True)
    (gv, gl, gw), (rv, rl, rw) = _sca_bwd(w, False)
    assert_close(gw, rw, False, "workload 3 grad_attention_weights_rb")
    assert_close(gl, rl, False, "workload 3 grad_sampling_locations_rb")
    assert_close(gv, rv, False, "workload 3 grad_value")


def _full_both(w, bf16):
    """sca_backward_full on the GPU; the oracle's derivative and chain."""
    got = msda.sca_backward_full(value_tensor(w, bf16), w.spatial_shapes, w.level_start_index,
                                 dev(w.reference_points), dev(w.bev_mask),
                                 dev(w.sampling_offsets), dev(w.attention_logits),
                                 dev(w.grad_out))
    torch.cuda.synchronize()
    rv, rl, rw = oracle.sca_backward(w.value, w.spatial_shapes, w.level_start_index,
                                     w.reference_points, w.bev_mask, w.sampling_offsets,
                                     w.attention_logits, w.grad_out)
    want = (rv,) + tuple(oracle.sca_backward_inputs(w.spatial_shapes, w.bev_mask,
                                                    w.attention_logits, rl, rw))
    return got, want


FULL_NAMES = ("grad_value", "grad_sampling_offsets", "grad_attention_logits",
              "grad_reference_points_cam")


@pytest.mark.parametrize("seed,B,Ncam,bev,shapes,H,P,R", [
    (51, 2, 3, (7, 9), [(9, 13), (4, 7)], 2, 4, 2),
    (52, 1, 6, (30, 40), [(16, 20), (8, 10), (4, 5), (2, 3)], 8, 8, 4),
    (53, 2, 2, (5, 13), [(6, 7)] * 3, 1, 12, 3),       # R = 3: separate reference kernel
    (54, 1, 4, (9, 11), [(8, 9), (4, 5)], 12, 4, 2),   # 12 heads: two head chunks
    (55, 2, 3, (6, 8), [(10, 12)], 8, 4, 4),           # rows of 4 samples: group chain
    (56, 1, 2, (4, 6), [(5, 6)] * 5, 2, 16, 4),        # 80 samples: three chunks
])
@pytest.mark.parametrize("rho", ["uniform", "coherent"])
def test_sca_backward_full(seed, B, Ncam, bev, shapes, H, P, R, rho):
    """The whole SCA backward to its inputs, at the fp32 element bound."""
    w = inputs.workload3(seed=seed, B=B, Ncam=Ncam, bev_h=bev[0], bev_w=bev[1], shapes=shapes,
                         H=H, P=P, R=R, rho=rho, same_mask=False, with_grad=True)
    got, want = _full_both(w, False)
    for g, r, name in zip(got, want, FULL_NAMES):
        assert_close(g, r, False, name)


def test_sca_backward_full_workload3_full_size():
    """BEVFormer-base (fp32 value, B = 1): value, offset, logit and
    reference-point gradients at the fp32 element bound."""
    w = inputs.workload3(seed=1003, with_grad=True)
    got, want = _full_both(w, False)
    for g, r, name in zip(got, want, FULL_NAMES):
        assert_close(g, r, False, "workload 3 " + name)


def test_workload5_training_step_full_size():
    w = inputs.workload5()
    out = msda.sca_forward(value_tensor(w, True), w.spatial_shapes, w.level_start_index,
                           dev(w.reference_points), dev(w.bev_mask), dev(w.sampling_offsets),
                           dev(w.attention_logits))
    (gv, gl, gw), (rv, rl, rw) = _sca_bwd(w, True)
    ref_out = oracle.sca_forward(w.value, w.spatial_shapes, w.level_start_index,
                                 w.reference_points, w.bev_mask, w.sampling_offsets,
                                 w.attention_logits)
    assert_close(out, ref_out, True, "workload 5 forward")
    assert_close(gw, rw, True, "workload 5 grad_attention_weights_rb")
    assert_close(gl, rl, True, "workload 5 grad_sampling_locations_rb")
    assert_close(gv, rv, True, "workload 5 grad_value")


def _input_grads_both(w, pos, rl, rw):
    """sca_backward_inputs on the GPU and in the oracle, both fed the same
    fp32 rebatched gradients (the oracle's, rounded once)."""
    rl32, rw32 = rl.astype(np.float32), rw.astype(np.float32)
    got = msda.sca_backward_inputs(w.spatial_shapes, w.level_start_index,
                                   dev(w.attention_logits), pos, dev(rl32), dev(rw32), w.Ncam,
                                   w.R)
    torch.cuda.synchronize()
    want = oracle.sca_backward_inputs(w.spatial_shapes, w.bev_mask, w.attention_logits, rl32,
                                      rw32)
    return got, want


@pytest.mark.parametrize("seed,B,Ncam,bev,shapes,H,P,R", [
    (41, 2, 3, (7, 9), [(9, 13), (4, 7)], 2, 4, 2),
    (42, 1, 6, (30, 40), [(16, 20), (8, 10), (4, 5), (2, 3)], 8, 8, 4),
    (43, 2, 2, (5, 13), [(6, 7)] * 3, 1, 12, 3),       # R = 3: separate reference kernel
    (44, 1, 4, (9, 11), [(8, 9), (4, 5)], 12, 4, 2),   # 12 heads: two head chunks
    # rows of <= 16 samples (the head-group kernel): eight heads of four samples
    # with the reference points fused, padded slots (12 of 16) in three passes,
    # and R = 3 not dividing the four-lane segment (separate reference kernel)
    (45, 2, 3, (6, 8), [(10, 12)], 8, 4, 4),
    (46, 1, 5, (7, 7), [(6, 9), (3, 5), (2, 2)], 5, 4, 1),
    (47, 2, 4, (5, 9), [(7, 7)], 3, 3, 3),
])
@pytest.mark.parametrize("rho", ["uniform", "coherent"])
def test_sca_backward_inputs(seed, B, Ncam, bev, shapes, H, P, R, rho):
    """Offsets, logits and reference-point gradients from the rebatched ones,
    against the oracle's chain rule (itself pinned by finite differences)."""
    w = inputs.workload3(seed=seed, B=B, Ncam=Ncam, bev_h=bev[0], bev_w=bev[1], shapes=shapes,
                         H=H, P=P, R=R, rho=rho, same_mask=False, with_grad=True)
    idx, count, pos, hits = msda.sca_compact(dev(w.bev_mask))
    _, rl, rw = oracle.sca_backward(w.value, w.spatial_shapes, w.level_start_index,
                                    w.reference_points, w.bev_mask, w.sampling_offsets,
                                    w.attention_logits, w.grad_out)
    (g_off, g_lg, g_ref), (r_off, r_lg, r_ref) = _input_grads_both(w, pos, rl, rw)
    assert_close(g_off, r_off, False, "grad_sampling_offsets")
    assert_close(g_lg, r_lg, False, "grad_attention_logits")
    assert_close(g_ref, r_ref, False, "grad_reference_points_cam")


def test_sca_backward_inputs_workload5():
    w = inputs.workload5()
    mask = dev(w.bev_mask)
    idx, count, pos, hits = msda.sca_compact(mask)
    gv, gl, gw = msda.sca_rebatched_backward(
        value_tensor(w, True), w.spatial_shapes, w.level_start_index, dev(w.reference_points),
        dev(w.sampling_offsets), dev(w.attention_logits), dev(w.grad_out), idx, count, hits)
    torch.cuda.synchronize()
    _, rl, rw = oracle.sca_backward(w.value, w.spatial_shapes, w.level_start_index,
                                    w.reference_points, w.bev_mask, w.sampling_offsets,
                                    w.attention_logits, w.grad_out)
    # the second stage alone, on the oracle's first-stage gradients: fp32 bound
    (g_off, g_lg, g_ref), (r_off, r_lg, r_ref) = _input_grads_both(w, pos, rl, rw)
    assert_close(g_off, r_off, False, "workload 5 grad_sampling_offsets")
    assert_close(g_lg, r_lg, False, "workload 5 grad_attention_logits")
    assert_close(g_ref, r_ref, False, "workload 5 grad_reference_points_cam")
    # the whole GPU chain in one call (bf16 value): the bf16-path bound
    got, want = _full_both(w, True)
    for g, r, name in zip(got, want, FULL_NAMES):
        assert_close(g, r, True, "workload 5 sca_backward_full " + name)


@pytest.mark.parametrize("case", CASES, ids=[f"case{c[0]}" for c in CASES])
@pytest.mark.parametrize("bf16", [False, True])
def test_msda_backward_deterministic(case, bf16):
    """Fixed-point grad_value: the oracle's derivative within the fp32 bound,
    and two runs bitwise equal."""
    seed, B, Nq, H, shapes, P = case
    s, starts, value, loc, weights, gout = _problem(seed, B, Nq, H, shapes, P)
    if bf16:
        bits = inputs.to_bf16_bits(value)
        value = inputs.bf16_bits_to_f32(bits)
        vt = dev(bits.view(np.int16)).view(torch.bfloat16)
    else:
        vt = dev(value)
    args = (vt, s, starts, dev(loc), dev(weights), dev(gout))
    gv, gl, gw = msda.msda_backward(*args, deterministic=True)
    gv2, gl2, gw2 = msda.msda_backward(*args, deterministic=True)
    torch.cuda.synchronize()
    rv, rl, rw = oracle.msda_backward(value, s, starts, loc, weights, gout)
    assert_close(gv, rv, False, "deterministic grad_value")
    assert_close(gl, rl, False, "grad_sampling_locations")
    assert_close(gw, rw, False, "grad_attention_weights")
    assert torch.equal(gv, gv2) and torch.equal(gl, gl2) and torch.equal(gw, gw2)


def test_sca_backward_deterministic_workload5():
    """The SCA training step with fixed-point grad_value: parity at full size
    (bf16 value), bitwise equal runs, and within fp32 rounding of the atomic
    path."""
    w = inputs.workload5()
    args = (value_tensor(w, True), w.spatial_shapes, w.level_start_index,
            dev(w.reference_points), dev(w.bev_mask), dev(w.sampling_offsets),
            dev(w.attention_logits), dev(w.grad_out))
    gv, gl, gw = msda.sca_backward(*args, deterministic=True)
    gv2, _, _ = msda.sca_backward(*args, deterministic=True)
    ga, _, _ = msda.sca_backward(*args)
    torch.cuda.synchronize()
    assert torch.equal(gv, gv2)
    rv, rl, rw = oracle.sca_backward(w.value, w.spatial_shapes, w.level_start_index,
                                     w.reference_points, w.bev_mask, w.sampling_offsets,
                                     w.attention_logits, w.grad_out)
    assert_close(gv, rv, True, "workload 5 deterministic grad_value")
    assert_close(gl, rl, True, "workload 5 grad_sampling_locations_rb")
    assert_close(gw, rw, True, "workload 5 grad_attention_weights_rb")
    assert_close(gv, ga.cpu().numpy(), False, "deterministic vs atomic grad_value")
