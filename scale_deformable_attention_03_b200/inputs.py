"""Seeded synthetic inputs for the five MSDA / SCA workloads.

This module draws random numbers and lays them out; it holds none of the
method's arithmetic (no softmax, no location, no sampling).  Both the CUDA
path (tests, benchmark) and the oracle (tests) consume what it returns, so it
is the only code the two sides share.

Workloads (seed = 1000 + workload number; NumPy PCG64; fp32 unless stated):

1 tiny MSDA: B=1, one 16x16 level, H=2, P=4, Nq=256; value ~N(0,1);
  locations ~U(-0.1, 1.1); logits ~N(0,1).  For the fused call: R=4 reference
  points ~U(-0.1, 1.1) and offsets ~N(0, 1) level pixels.
2 Deformable-DETR encoder MSDA: B=1, H=8, levels 100x150, 50x75, 25x38, 13x19
  (Nv=19947), Nq=Nv, P=4, R=1.  The reference point of query q is the centre
  of q's own pixel on q's own level, normalised; offsets ~N(0, 2) level pixels;
  logits ~N(0,1); value ~N(0,1).
3 BEVFormer-base SCA: B=1, 6 cameras, levels 116x200, 58x100, 29x50, 15x25
  (Nv=30825 per camera), H=8, P=8, R=4, 200x200 BEV queries (row-major).
  bev_mask: every query is seen by 1 + Bernoulli(0.5) cameras drawn without
  replacement; in a seeing camera its R anchor bits are uniform over the
  non-zero patterns (Bernoulli(0.5) each, conditioned on at least one).
  Reference points ("coherent"): rho_x = frac((j+0.5)/200 + c/6),
  rho_y = 0.25 + 0.5 (i+0.5)/200 + 0.06 (m - 1.5) for BEV cell (i, j),
  camera c, anchor m, so that neighbouring cells read neighbouring pixels;
  ("uniform"): U(0,1)^2.  Offsets ~N(0, 2) level pixels; logits ~N(0,1);
  value ~N(0,1), fp32 or bf16.
4 BEVFormer TSA MSDA: two queues (prev_bev, bev) of one 200x200 level, H=8,
  P=4, R=1, Nq=40000.  Reference points are BEV cell centres; the prev_bev
  queue's are shifted by one (sx, sy) ~U(-5, 5) cells per draw.  Offsets
  ~N(0, 1.5) cells; logits ~N(0,1); value ~N(0,1).
5 BEVFormer-base SCA training step: workload 3 with B=2 (the same bev_mask for
  both batch items, independent everything else), bf16 value, upstream
  gradient ~N(0,1) [2, 40000, 256].

bf16 values are rounded from fp32 once, round-to-nearest-even; ``value`` then
holds the bf16 values widened exactly to fp32, and ``value_bf16`` their bits.
"""
from dataclasses import dataclass, field
from typing import Dict, Optional

import numpy as np

DH = 32  # channels per head

SHAPES_DETR = [(100, 150), (50, 75), (25, 38), (13, 19)]
SHAPES_BEVFORMER = [(116, 200), (58, 100), (29, 50), (15, 25)]


@dataclass
class Workload:
    """Arrays of one synthetic problem; absent entries are None."""
    name: str
    B: int
    Ncam: int
    Nq: int
    Nv: int
    H: int
    L: int
    P: int
    R: int
    spatial_shapes: np.ndarray              # [L, 2] int64, rows (H_l, W_l)
    level_start_index: np.ndarray           # [L] int64
    value: np.ndarray                       # fp32 (bf16-exact when value_bf16 is set)
    value_bf16: Optional[np.ndarray] = None  # uint16 bits, same shape as value
    sampling_locations: Optional[np.ndarray] = None
    attention_logits: Optional[np.ndarray] = None
    reference_points: Optional[np.ndarray] = None
    sampling_offsets: Optional[np.ndarray] = None
    bev_mask: Optional[np.ndarray] = None
    grad_out: Optional[np.ndarray] = None
    extra: Dict[str, object] = field(default_factory=dict)

    @property
    def dims(self):
        return dict(B=self.B, Ncam=self.Ncam, Nq=self.Nq, Nv=self.Nv, H=self.H, L=self.L,
                    P=self.P, R=self.R)


def level_table(shapes):
    s = np.asarray(shapes, dtype=np.int64).reshape(-1, 2)
    sizes = s[:, 0] * s[:, 1]
    starts = np.concatenate([[0], np.cumsum(sizes)[:-1]]).astype(np.int64)
    return s, starts, int(sizes.sum())


def to_bf16_bits(x):
    """fp32 -> bf16 bit patterns, round to nearest even (finite inputs)."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    rounding = ((u >> 16) & 1) + np.uint32(0x7FFF)
    return ((u + rounding) >> 16).astype(np.uint16)


def bf16_bits_to_f32(b):
    return (b.astype(np.uint32) << 16).view(np.float32)


def _normal(rng, shape, std=1.0):
    return (rng.standard_normal(shape) * std).astype(np.float32)


def _value(rng, shape, value_dtype):
    v = _normal(rng, shape)
    if value_dtype == "bf16":
        bits = to_bf16_bits(v)
        return bf16_bits_to_f32(bits), bits
    if value_dtype != "f32":
        raise ValueError(value_dtype)
    return v, None


def workload1(seed=1001, value_dtype="f32", Nq=256, side=16, H=2, P=4, R=4):
    rng = np.random.Generator(np.random.PCG64(seed))
    shapes, starts, Nv = level_table([(side, side)])
    B, L = 1, 1
    value, bits = _value(rng, (B, Nv, H, DH), value_dtype)
    loc = rng.uniform(-0.1, 1.1, (B, Nq, H, L, P, 2)).astype(np.float32)
    logits = _normal(rng, (B, Nq, H, L, P))
    ref = rng.uniform(-0.1, 1.1, (B, Nq, R, 2)).astype(np.float32)
    off = _normal(rng, (B, Nq, H, L, P, 2), 1.0)
    return Workload("tiny-msda", B, 1, Nq, Nv, H, L, P, R, shapes, starts, value, bits,
                    sampling_locations=loc, attention_logits=logits, reference_points=ref,
                    sampling_offsets=off)


def workload2(seed=1002, value_dtype="f32", shapes=SHAPES_DETR, H=8, P=4, max_queries=None):
    """Queries are the pixels of every level, in value-row order (optionally the
    first ``max_queries`` of them)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    shapes, starts, Nv = level_table(shapes)
    B, L, R = 1, len(shapes), 1
    value, bits = _value(rng, (B, Nv, H, DH), value_dtype)
    centres = []
    for (Hl, Wl) in shapes:
        ys, xs = np.meshgrid(np.arange(Hl), np.arange(Wl), indexing="ij")
        centres.append(np.stack([(xs + 0.5) / Wl, (ys + 0.5) / Hl], -1).reshape(-1, 2))
    ref = np.concatenate(centres)[None, :, None, :].astype(np.float32)  # [1, Nv, 1, 2]
    Nq = Nv if max_queries is None else min(Nv, max_queries)
    ref = np.ascontiguousarray(ref[:, :Nq])
    off = _normal(rng, (B, Nq, H, L, P, 2), 2.0)
    logits = _normal(rng, (B, Nq, H, L, P))
    return Workload("detr-encoder-msda", B, 1, Nq, Nv, H, L, P, R, shapes, starts, value, bits,
                    attention_logits=logits, reference_points=ref, sampling_offsets=off)


def sca_mask(rng, Ncam, B, Nq, R, same_for_batch=True):
    """bev_mask [Ncam, B, Nq, R] uint8: 1 + Bernoulli(0.5) seeing cameras per
    query, drawn without replacement; non-zero anchor pattern per seeing camera."""
    def one():
        n_hit = 1 + rng.binomial(1, 0.5, size=Nq)
        order = np.argsort(rng.random((Nq, Ncam)), axis=1)
        seen = np.zeros((Nq, Ncam), dtype=bool)
        rows = np.arange(Nq)
        for r in range(min(2, Ncam)):
            sel = n_hit > r
            seen[rows[sel], order[sel, r]] = True
        pattern = rng.integers(1, 2 ** R, size=(Ncam, Nq))
        bitsel = (pattern[:, :, None] >> np.arange(R)[None, None, :]) & 1
        return (seen.T[:, :, None] & (bitsel == 1)).astype(np.uint8)  # [Ncam, Nq, R]
    first = one()
    per_b = [first] + [first if same_for_batch else one() for _ in range(B - 1)]
    return np.ascontiguousarray(np.stack(per_b, axis=1))


def sca_reference_points(rng, Ncam, B, bev_h, bev_w, R, kind="coherent"):
    Nq = bev_h * bev_w
    if kind == "uniform":
        return rng.random((Ncam, B, Nq, R, 2)).astype(np.float32)
    if kind != "coherent":
        raise ValueError(kind)
    i, j = np.meshgrid(np.arange(bev_h), np.arange(bev_w), indexing="ij")
    i, j = i.reshape(-1), j.reshape(-1)
    ref = np.empty((Ncam, B, Nq, R, 2), dtype=np.float64)
    for c in range(Ncam):
        rx = np.mod((j + 0.5) / bev_w + c / Ncam, 1.0)
        for m in range(R):
            ry = 0.25 + 0.5 * (i + 0.5) / bev_h + 0.06 * (m - (R - 1) / 2.0)
            ref[c, :, :, m, 0] = rx
            ref[c, :, :, m, 1] = ry
    return ref.astype(np.float32)


def workload3(seed=1003, value_dtype="f32", B=1, Ncam=6, bev_h=200, bev_w=200,
              shapes=SHAPES_BEVFORMER, H=8, P=8, R=4, rho="coherent", same_mask=True,
              with_grad=False):
    rng = np.random.Generator(np.random.PCG64(seed))
    shapes, starts, Nv = level_table(shapes)
    L, Nq = len(shapes), bev_h * bev_w
    value, bits = _value(rng, (B, Ncam, Nv, H, DH), value_dtype)
    mask = sca_mask(rng, Ncam, B, Nq, R, same_for_batch=same_mask)
    ref = sca_reference_points(rng, Ncam, B, bev_h, bev_w, R, rho)
    off = _normal(rng, (B, Nq, H, L, P, 2), 2.0)
    logits = _normal(rng, (B, Nq, H, L, P))
    gout = _normal(rng, (B, Nq, H * DH)) if with_grad else None
    return Workload("bevformer-base-sca", B, Ncam, Nq, Nv, H, L, P, R, shapes, starts, value,
                    bits, attention_logits=logits, reference_points=ref, sampling_offsets=off,
                    bev_mask=mask, grad_out=gout, extra=dict(bev_h=bev_h, bev_w=bev_w, rho=rho))


def workload4(seed=1004, value_dtype="f32", bev_h=200, bev_w=200, H=8, P=4, max_shift=5.0):
    rng = np.random.Generator(np.random.PCG64(seed))
    shapes, starts, Nv = level_table([(bev_h, bev_w)])
    B, L, R, Nq = 2, 1, 1, bev_h * bev_w
    value, bits = _value(rng, (B, Nv, H, DH), value_dtype)
    sx, sy = rng.uniform(-max_shift, max_shift, 2)
    i, j = np.meshgrid(np.arange(bev_h), np.arange(bev_w), indexing="ij")
    i, j = i.reshape(-1).astype(np.float64), j.reshape(-1).astype(np.float64)
    ref = np.empty((B, Nq, R, 2))
    ref[0, :, 0, 0] = (j + 0.5 + sx) / bev_w   # prev_bev queue, ego-shifted
    ref[0, :, 0, 1] = (i + 0.5 + sy) / bev_h
    ref[1, :, 0, 0] = (j + 0.5) / bev_w        # current bev queue
    ref[1, :, 0, 1] = (i + 0.5) / bev_h
    off = _normal(rng, (B, Nq, H, L, P, 2), 1.5)
    logits = _normal(rng, (B, Nq, H, L, P))
    return Workload("bevformer-tsa-msda", B, 1, Nq, Nv, H, L, P, R, shapes, starts, value, bits,
                    attention_logits=logits, reference_points=ref.astype(np.float32),
                    sampling_offsets=off, extra=dict(shift=(float(sx), float(sy))))


def workload5(seed=1005, bev_h=200, bev_w=200, **kw):
    return workload3(seed=seed, value_dtype="bf16", B=2, bev_h=bev_h, bev_w=bev_w,
                     same_mask=True, with_grad=True, **kw)


def make(n, **kw):
    return {1: workload1, 2: workload2, 3: workload3, 4: workload4, 5: workload5}[n](**kw)
