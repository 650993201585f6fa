"""MSDA forward (msda_forward, msda_forward_fused) on the GPU against the
oracle, element by element, through the C ABI.

Workloads 1, 2 and 4 at their full sizes (the oracle finishes each in about a
second), fp32 and bf16 value, plus randomised shapes covering several sample
chunks per row (L*P up to 128), ragged query counts, odd level sizes,
locations partly or wholly outside the maps, and a non-finite location.
"""
import numpy as np
import pytest
import torch

import oracle
import scale_deformable_attention_03_b200 as msda
from scale_deformable_attention_03_b200 import inputs

from .gpu_util import assert_close, dev, softmax_weights, value_tensor

pytestmark = pytest.mark.gpu


def _run_fused(w, bf16):
    out = msda.msda_forward_fused(value_tensor(w, bf16), w.spatial_shapes, w.level_start_index,
                                  dev(w.reference_points), dev(w.sampling_offsets),
                                  dev(w.attention_logits))
    torch.cuda.synchronize()
    ref = oracle.msda_forward_fused(w.value, w.spatial_shapes, w.level_start_index,
                                    w.reference_points, w.sampling_offsets, w.attention_logits)
    return out, ref


@pytest.mark.parametrize("bf16", [False, True])
def test_workload1_given_locations(bf16):
    w = inputs.workload1(value_dtype="bf16" if bf16 else "f32")
    weights = softmax_weights(w.attention_logits, w.L * w.P)
    out = msda.msda_forward(value_tensor(w, bf16), w.spatial_shapes, w.level_start_index,
                            dev(w.sampling_locations), dev(weights))
    torch.cuda.synchronize()
    ref = oracle.msda_forward(w.value, w.spatial_shapes, w.level_start_index,
                              w.sampling_locations, weights)
    assert_close(out, ref, bf16, "workload 1 msda_forward")


@pytest.mark.parametrize("bf16", [False, True])
def test_workload1_fused(bf16):
    w = inputs.workload1(value_dtype="bf16" if bf16 else "f32")
    out, ref = _run_fused(w, bf16)
    assert_close(out, ref, bf16, "workload 1 fused")


@pytest.mark.parametrize("bf16", [False, True])
def test_workload2_detr_encoder(bf16):
    w = inputs.workload2(value_dtype="bf16" if bf16 else "f32")
    out, ref = _run_fused(w, bf16)
    assert_close(out, ref, bf16, "workload 2 fused")


def test_workload2_given_locations_from_fused_inputs():
    w = inputs.workload2()
    loc, weights = oracle.fused_locations(w.spatial_shapes, w.reference_points,
                                          w.sampling_offsets, w.attention_logits)
    loc = loc.astype(np.float32)
    weights = weights.astype(np.float32)
    out = msda.msda_forward(dev(w.value), w.spatial_shapes, w.level_start_index, dev(loc),
                            dev(weights))
    torch.cuda.synchronize()
    ref = oracle.msda_forward(w.value, w.spatial_shapes, w.level_start_index, loc, weights)
    assert_close(out, ref, False, "workload 2 msda_forward")


def test_workload4_tsa():
    w = inputs.workload4()
    out, ref = _run_fused(w, False)
    assert_close(out, ref, False, "workload 4 fused")


def _random_problem(seed, B, Nq, H, shapes, P, R, lo=-0.2, hi=1.2):
    rng = np.random.Generator(np.random.PCG64(seed))
    s, starts, Nv = inputs.level_table(shapes)
    L = len(shapes)
    value = rng.standard_normal((B, Nv, H, 32)).astype(np.float32)
    loc = rng.uniform(lo, hi, (B, Nq, H, L, P, 2)).astype(np.float32)
    logits = rng.standard_normal((B, Nq, H, L, P)).astype(np.float32)
    ref = rng.uniform(lo, hi, (B, Nq, R, 2)).astype(np.float32)
    off = (rng.standard_normal((B, Nq, H, L, P, 2)) * 3).astype(np.float32)
    return s, starts, value, loc, logits, ref, off


CASES = [
    # seed, B, Nq, H, shapes, P, R
    (1, 1, 37, 1, [(5, 7)], 1, 1),
    (2, 2, 65, 2, [(9, 13), (4, 7)], 3, 1),
    (3, 1, 100, 8, [(17, 23), (8, 11), (4, 6), (2, 3)], 8, 4),   # L*P = 32
    (4, 3, 33, 3, [(6, 5), (3, 3), (1, 9)], 12, 6),              # L*P = 36: two chunks
    (5, 1, 41, 2, [(7, 9)] * 4 + [(3, 5)] * 4, 16, 8),           # L*P = 128: four chunks
    (6, 2, 129, 4, [(1, 1), (2, 1), (1, 2)], 5, 5),              # 1-pixel levels
]


@pytest.mark.parametrize("case", CASES, ids=[f"case{c[0]}" for c in CASES])
@pytest.mark.parametrize("bf16", [False, True])
def test_random_shapes(case, bf16):
    """Every kernel layout: one head per warp (one to four sample chunks),
    head pairs (bf16, even H), several heads per warp (L*P <= 16), 1-pixel
    levels, 8 levels of 16 points."""
    seed, B, Nq, H, shapes, P, R = case
    s, starts, value, loc, logits, ref, off = _random_problem(seed, B, Nq, H, shapes, P, R)
    L = len(shapes)
    vt = dev(value)
    if bf16:
        bits = inputs.to_bf16_bits(value)
        value = inputs.bf16_bits_to_f32(bits)
        vt = dev(bits.view(np.int16)).view(torch.bfloat16)
    weights = softmax_weights(logits, L * P)
    out = msda.msda_forward(vt, s, starts, dev(loc), dev(weights))
    out_f = msda.msda_forward_fused(vt, s, starts, dev(ref), dev(off), dev(logits))
    torch.cuda.synchronize()
    assert_close(out, oracle.msda_forward(value, s, starts, loc, weights), bf16, "given")
    assert_close(out_f, oracle.msda_forward_fused(value, s, starts, ref, off, logits), bf16,
                 "fused")


def test_level_start_index_with_gaps():
    """Levels need not be packed: starts are honoured as given."""
    rng = np.random.Generator(np.random.PCG64(7))
    shapes = np.array([[4, 6], [3, 3]], np.int64)
    starts = np.array([5, 40], np.int64)
    Nv, B, Nq, H, L, P = 60, 1, 50, 2, 2, 4
    value = rng.standard_normal((B, Nv, H, 32)).astype(np.float32)
    loc = rng.uniform(-0.1, 1.1, (B, Nq, H, L, P, 2)).astype(np.float32)
    weights = rng.uniform(0, 1, (B, Nq, H, L, P)).astype(np.float32)
    out = msda.msda_forward(dev(value), shapes, starts, dev(loc), dev(weights))
    torch.cuda.synchronize()
    assert_close(out, oracle.msda_forward(value, shapes, starts, loc, weights), False, "gaps")


def test_non_finite_and_outside_locations():
    s, starts, value, loc, logits, ref, off = _random_problem(8, 1, 16, 2, [(5, 6)], 4, 1)
    loc[0, 0, :, 0, 0, 0] = np.nan
    loc[0, 1, :, 0, 1, 1] = np.inf
    loc[0, 2, :, 0, 2, 0] = -np.inf
    loc[0, 3, :, 0, :, 0] = -0.5   # wholly left of the map
    loc[0, 4, :, 0, :, 1] = 1.2    # wholly below
    loc[0, 5, :, 0, :, 0] = 1e30
    weights = softmax_weights(logits, 4)
    out = msda.msda_forward(dev(value), s, starts, dev(loc), dev(weights))
    torch.cuda.synchronize()
    ref_out = oracle.msda_forward(value, s, starts, loc, weights)
    assert np.all(np.isfinite(ref_out))
    assert_close(out, ref_out, False, "non-finite")


def test_empty_batch_and_queries():
    s, starts = np.array([[3, 4]], np.int64), np.array([0], np.int64)
    value = torch.zeros((1, 12, 2, 32), device="cuda")
    out = msda.msda_forward(value, s, starts, torch.zeros((1, 0, 2, 1, 2, 2), device="cuda"),
                            torch.zeros((1, 0, 2, 1, 2), device="cuda"))
    assert out.shape == (1, 0, 64)
    out = msda.msda_forward(torch.zeros((0, 12, 2, 32), device="cuda"), s, starts,
                            torch.zeros((0, 5, 2, 1, 2, 2), device="cuda"),
                            torch.zeros((0, 5, 2, 1, 2), device="cuda"))
    assert out.shape == (0, 5, 64)
    torch.cuda.synchronize()


def test_repeat_calls_identical():
    """The forward has no atomics: two calls give identical bits."""
    w = inputs.workload2(max_queries=3000)
    args = (dev(w.value), w.spatial_shapes, w.level_start_index, dev(w.reference_points),
            dev(w.sampling_offsets), dev(w.attention_logits))
    a = msda.msda_forward_fused(*args)
    b = msda.msda_forward_fused(*args)
    torch.cuda.synchronize()
    assert torch.equal(a, b)
