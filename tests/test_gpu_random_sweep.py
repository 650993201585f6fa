"""Seeded sweeps over the problem space.  SCA: batch, cameras, BEV size, level
count and shapes (one-pixel levels included), heads, points and anchors,
reference points and value dtype, drawn once from a fixed generator, plus two
problems at the compiled limits (L = 8, P = 16, 32 cameras; B * Ncam = 1024).  Each
problem runs every SCA entry point (the one-call forward, the staged calls,
the query-major kernel, the training backward in both accumulation modes and
the whole backward chain) against the oracle: fp32 value at the fp32 element
bound, bf16 value at the bf16 bound (the oracle reading the same bf16
values); the staged calls must equal the one-call
forward bit for bit (both run the rebatched kernels), and the two grad_value
accumulations must agree with each other within the fp32 bound.  Plain MSDA:
batch, queries, heads, levels, points and anchors, locations partly outside
their levels, through msda_forward, msda_forward_fused and msda_backward (both
accumulation modes).
"""
import numpy as np
import pytest
import torch

import oracle
import scale_deformable_attention_03_b200 as msda
from scale_deformable_attention_03_b200 import inputs

from .gpu_util import assert_close, dev, value_tensor

pytestmark = pytest.mark.gpu


def _draw(n, seed=2024):
    """n problems (seed, B, Ncam, (bev_h, bev_w), shapes, H, P, R, rho)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    out = []
    for i in range(n):
        L = int(rng.integers(1, 5))
        shapes = [(int(rng.integers(1, 24)), int(rng.integers(1, 24))) for _ in range(L)]
        H = int(rng.choice([1, 2, 3, 4, 6, 8, 12, 16]))
        R = int(rng.choice([1, 2, 4]))
        P = R * int(rng.integers(1, 16 // R + 1))
        out.append((3000 + i, int(rng.integers(1, 3)), int(rng.integers(1, 9)),
                    (int(rng.integers(1, 17)), int(rng.integers(1, 17))), shapes, H, P, R,
                    str(rng.choice(["uniform", "coherent"]))))
    return out


# The compiled limits, beside the drawn problems: eight levels of sixteen
# points (rows of 128 samples, four sample chunks) with sixteen anchors over 32
# cameras, and B * Ncam = 1024 batch-cameras (the largest row-prefix table).
LIMITS = [
    (3900, 1, 32, (4, 5), [(9, 11), (7, 8), (5, 6), (4, 4), (3, 3), (2, 2), (1, 2), (1, 1)],
     2, 16, 16, "uniform"),
    (3901, 32, 32, (2, 3), [(3, 4)], 1, 2, 2, "uniform"),
]

PROBLEMS = _draw(24) + LIMITS


def _workload(case, bf16):
    seed, B, Ncam, bev, shapes, H, P, R, rho = case
    return inputs.workload3(seed=seed, B=B, Ncam=Ncam, bev_h=bev[0], bev_w=bev[1],
                            shapes=shapes, H=H, P=P, R=R, rho=rho, same_mask=False,
                            with_grad=True, value_dtype="bf16" if bf16 else "f32")


@pytest.mark.parametrize("case", PROBLEMS, ids=[f"p{c[0]}" for c in PROBLEMS])
@pytest.mark.parametrize("bf16", [False, True])
def test_forward_entry_points(case, bf16):
    w = _workload(case, bf16)
    v = value_tensor(w, bf16)
    args = (v, w.spatial_shapes, w.level_start_index, dev(w.reference_points))
    mask, off, lg = dev(w.bev_mask), dev(w.sampling_offsets), dev(w.attention_logits)
    whole = msda.sca_forward(*args, mask, off, lg)
    qm = msda.sca_forward_query_major(*args, mask, off, lg)
    idx, count, pos, hits = msda.sca_compact(mask)
    rows = msda.sca_rebatched_forward(*args, off, lg, idx, count)
    staged = msda.sca_camera_average(rows, pos, hits)
    torch.cuda.synchronize()
    ref = oracle.sca_forward(w.value, w.spatial_shapes, w.level_start_index, w.reference_points,
                             w.bev_mask, w.sampling_offsets, w.attention_logits)
    assert_close(whole, ref, bf16, "sca_forward")
    assert_close(qm, ref, bf16, "sca_forward_query_major")
    assert_close(staged, ref, bf16, "staged forward")
    assert torch.equal(staged, whole)  # the same kernels, the same bits


@pytest.mark.parametrize("case", PROBLEMS, ids=[f"p{c[0]}" for c in PROBLEMS])
@pytest.mark.parametrize("bf16", [False, True])
def test_backward_entry_points(case, bf16):
    w = _workload(case, bf16)
    args = (value_tensor(w, bf16), w.spatial_shapes, w.level_start_index,
            dev(w.reference_points), dev(w.bev_mask), dev(w.sampling_offsets),
            dev(w.attention_logits), dev(w.grad_out))
    gv, gl, gw = msda.sca_backward(*args)
    gvd, gld, gwd = msda.sca_backward(*args, deterministic=True)
    full = msda.sca_backward_full(*args)
    torch.cuda.synchronize()
    rv, rl, rw = oracle.sca_backward(w.value, w.spatial_shapes, w.level_start_index,
                                     w.reference_points, w.bev_mask, w.sampling_offsets,
                                     w.attention_logits, w.grad_out)
    for name, g, r in (("grad_value", gv, rv), ("grad_sampling_locations_rb", gl, rl),
                       ("grad_attention_weights_rb", gw, rw),
                       ("deterministic grad_value", gvd, rv),
                       ("deterministic grad_sampling_locations_rb", gld, rl),
                       ("deterministic grad_attention_weights_rb", gwd, rw)):
        assert_close(g, r, bf16, name)
    assert_close(gv, gvd.cpu().numpy(), False, "atomic vs fixed-point grad_value")
    want = (rv,) + tuple(oracle.sca_backward_inputs(w.spatial_shapes, w.bev_mask,
                                                    w.attention_logits, rl, rw))
    for g, r, name in zip(full, want, ("grad_value", "grad_sampling_offsets",
                                       "grad_attention_logits", "grad_reference_points_cam")):
        assert_close(g, r, bf16, f"sca_backward_full {name}")


def _draw_msda(n, seed=2025):
    """n plain-MSDA problems (seed, B, Nq, H, shapes, P, R)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    out = []
    for i in range(n):
        L = int(rng.integers(1, 5))
        shapes = [(int(rng.integers(1, 24)), int(rng.integers(1, 24))) for _ in range(L)]
        R = int(rng.choice([1, 2, 4]))
        P = R * int(rng.integers(1, 16 // R + 1))
        out.append((4000 + i, int(rng.integers(1, 4)), int(rng.integers(1, 300)),
                    int(rng.choice([1, 2, 3, 4, 5, 8, 12, 16])), shapes, P, R))
    return out


MSDA_PROBLEMS = _draw_msda(24)


@pytest.mark.parametrize("case", MSDA_PROBLEMS, ids=[f"m{c[0]}" for c in MSDA_PROBLEMS])
@pytest.mark.parametrize("bf16", [False, True])
def test_msda_entry_points(case, bf16):
    """msda_forward (given locations and weights; about a third of the
    locations lie partly or wholly outside their level), msda_forward_fused,
    msda_backward in both accumulation modes, against the oracle."""
    seed, B, Nq, H, shapes, P, R = case
    rng = np.random.Generator(np.random.PCG64(seed))
    s, starts, Nv = inputs.level_table(shapes)
    L = len(shapes)
    value = rng.standard_normal((B, Nv, H, 32)).astype(np.float32)
    if bf16:
        bits = inputs.to_bf16_bits(value)
        value = inputs.bf16_bits_to_f32(bits)
        vt = dev(bits.view(np.int16)).view(torch.bfloat16)
    else:
        vt = dev(value)
    loc = rng.uniform(-0.2, 1.2, (B, Nq, H, L, P, 2)).astype(np.float32)
    logits = rng.standard_normal((B, Nq, H, L, P)).astype(np.float32)
    weights = oracle.softmax(logits, L * P).reshape(logits.shape).astype(np.float32)
    ref = rng.uniform(-0.2, 1.2, (B, Nq, R, 2)).astype(np.float32)
    off = (rng.standard_normal((B, Nq, H, L, P, 2)) * 3).astype(np.float32)
    gout = rng.standard_normal((B, Nq, H * 32)).astype(np.float32)

    out = msda.msda_forward(vt, s, starts, dev(loc), dev(weights))
    fused = msda.msda_forward_fused(vt, s, starts, dev(ref), dev(off), dev(logits))
    gv, gl, gw = msda.msda_backward(vt, s, starts, dev(loc), dev(weights), dev(gout))
    gvd, gld, gwd = msda.msda_backward(vt, s, starts, dev(loc), dev(weights), dev(gout),
                                       deterministic=True)
    torch.cuda.synchronize()
    assert_close(out, oracle.msda_forward(value, s, starts, loc, weights), bf16, "msda_forward")
    assert_close(fused, oracle.msda_forward_fused(value, s, starts, ref, off, logits), bf16,
                 "msda_forward_fused")
    rv, rl, rw = oracle.msda_backward(value, s, starts, loc, weights, gout)
    for name, g, r in (("grad_value", gv, rv), ("grad_sampling_locations", gl, rl),
                       ("grad_attention_weights", gw, rw),
                       ("deterministic grad_value", gvd, rv),
                       ("deterministic grad_sampling_locations", gld, rl),
                       ("deterministic grad_attention_weights", gwd, rw)):
        assert_close(g, r, bf16, name)
