"""Pins of the oracle against facts fixed by the pages and by mathematics.

Every test here runs on the CPU.  None of them re-types the oracle's formula:
each checks it against a worked example from the pages, a closed form, an
invariant, a library routine the special case reduces to (torch's
grid_sample), a brute-force loop with a different structure, or central
finite differences.

Sources: "BEV(三) BEVFormer: how the Query interacts with the 8 Heads of the
Feature" (sections 4.2, 5, 6, 7, 10, 15) and the Tencent Cloud "Spatial
Cross-Attention" walkthrough (rebatch and average listings).
"""
import json
import os

import numpy as np
import pytest
import torch

import oracle
from scale_deformable_attention_03_b200 import inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rng(seed):
    return np.random.Generator(np.random.PCG64(seed))


def _levels(shapes):
    s, starts, nv = inputs.level_table(shapes)
    return s, starts, nv


def _value_rows(value_b, starts, shapes, l, h):
    """[Dh, H_l, W_l] view of head h of level l of one batch item's value."""
    Hl, Wl = shapes[l]
    rows = value_b[starts[l]:starts[l] + Hl * Wl, h, :]
    return rows.reshape(Hl, Wl, -1).transpose(2, 0, 1)


def _grid_sample_msda(value, shapes, starts, loc, attn):
    """Brute force with torch's grid_sample (bilinear, zero padding,
    align_corners=False) for every (b, q, h, l, k), summed with the weights."""
    B, Nv, H, Dh = value.shape
    _, Nq, _, L, P, _ = loc.shape
    out = np.zeros((B, Nq, H, Dh))
    for b in range(B):
        for h in range(H):
            for l in range(L):
                img = torch.from_numpy(np.ascontiguousarray(
                    _value_rows(value[b], starts, shapes, l, h)))[None]
                grid = torch.from_numpy(2.0 * loc[b, :, h, l, :, :] - 1.0)[None]  # [1, Nq, P, 2]
                f = torch.nn.functional.grid_sample(img, grid, mode="bilinear",
                                                    padding_mode="zeros", align_corners=False)
                f = f[0].numpy().transpose(1, 2, 0)  # [Nq, P, Dh]
                out[b, :, h, :] += np.einsum("qp,qpd->qd", attn[b, :, h, l, :], f)
    return out.reshape(B, Nq, H * Dh)


# --------------------------------------------------------------------------
# softmax (section 4.2)
# --------------------------------------------------------------------------

def test_softmax_sums_to_one_per_head():
    a = _rng(1).standard_normal((7, 3, 32)) * 4
    w = oracle.softmax(a, 32)
    assert np.all(w > 0)
    np.testing.assert_allclose(w.sum(-1), 1.0, rtol=0, atol=1e-12)
    # ordering is preserved and a shift of all logits changes nothing
    np.testing.assert_array_equal(np.argsort(w, -1), np.argsort(a, -1))
    np.testing.assert_allclose(oracle.softmax(a + 123.0, 32), w, rtol=1e-12, atol=0)


def test_softmax_zero_logits_uniform():
    # zero-initialised weight head: every one of the L*P = 32 weights is 1/32
    w = oracle.softmax(np.zeros((5, 8, 32)), 32)
    assert np.all(w == 1.0 / 32.0)
    w = oracle.softmax(np.zeros((2, 12)), 12)
    np.testing.assert_allclose(w, 1.0 / 12.0, rtol=1e-15)


def test_softmax_large_logits_stable():
    w = oracle.softmax(np.array([[1000.0, 1000.0, -1000.0, 999.0]]), 4)
    e = np.exp([0.0, 0.0, -2000.0, -1.0])
    np.testing.assert_allclose(w[0], e / e.sum(), rtol=1e-14)


# --------------------------------------------------------------------------
# bilinear read (section 6)
# --------------------------------------------------------------------------

@pytest.mark.parametrize("coord_f32", [True, False])
def test_pixel_centres_reproduce_pixels(coord_f32):
    shapes, starts, Nv = _levels([(5, 7), (3, 4), (2, 9)])
    H, Dh = 3, 5
    rng = _rng(2)
    value = rng.standard_normal((1, Nv, H, Dh))
    L, P = len(shapes), 1
    targets = [(l, y, x) for l in range(L) for y in range(shapes[l][0]) for x in range(shapes[l][1])]
    Nq = len(targets)
    loc = rng.uniform(0.2, 0.8, (1, Nq, H, L, P, 2)).astype(np.float32)
    attn = np.zeros((1, Nq, H, L, P))
    expect = np.zeros((1, Nq, H, Dh))
    for q, (l, y, x) in enumerate(targets):
        Hl, Wl = shapes[l]
        loc[0, q, :, l, 0, 0] = np.float32((x + 0.5) / Wl)
        loc[0, q, :, l, 0, 1] = np.float32((y + 0.5) / Hl)
        attn[0, q, :, l, 0] = 1.0
        expect[0, q] = value[0, starts[l] + y * Wl + x]
    out = oracle.msda_forward(value, shapes, starts, loc, attn, coord_f32=coord_f32)
    np.testing.assert_allclose(out, expect.reshape(1, Nq, H * Dh), rtol=1e-6, atol=1e-6)


def test_constant_map_gives_constant():
    shapes, starts, Nv = _levels([(6, 9), (3, 5)])
    H, Dh, L, P, Nq = 2, 4, 2, 3, 40
    rng = _rng(3)
    value = np.full((1, Nv, H, Dh), 2.5)
    loc = np.empty((1, Nq, H, L, P, 2), np.float32)
    for l, (Hl, Wl) in enumerate(shapes):
        # x = W s - 1/2 in [0, W-1]: all four neighbours inside the map
        loc[..., l, :, 0] = rng.uniform(0.5 / Wl, 1 - 0.5 / Wl, (1, Nq, H, P))
        loc[..., l, :, 1] = rng.uniform(0.5 / Hl, 1 - 0.5 / Hl, (1, Nq, H, P))
    attn = rng.uniform(0, 1, (1, Nq, H, L, P))
    out = oracle.msda_forward(value, shapes, starts, loc, attn).reshape(1, Nq, H, Dh)
    expect = 2.5 * attn.sum(axis=(3, 4))[..., None]
    np.testing.assert_allclose(out, np.broadcast_to(expect, out.shape), rtol=1e-12)


def test_fully_out_of_bounds_is_zero():
    shapes, starts, Nv = _levels([(4, 6)])
    H, Dh, L, P, Nq = 2, 3, 1, 4, 64
    rng = _rng(4)
    value = rng.standard_normal((1, Nv, H, Dh)) + 10.0
    Hl, Wl = shapes[0]
    loc = rng.uniform(0.0, 1.0, (1, Nq, H, L, P, 2))
    side = rng.integers(0, 4, (1, Nq, H, L, P))
    # x <= -1 (s_x <= -0.5/W), x >= W (s_x >= 1 + 0.5/W), same for y
    loc[..., 0] = np.where(side == 0, rng.uniform(-2.0, -0.5 / Wl, side.shape), loc[..., 0])
    loc[..., 0] = np.where(side == 1, rng.uniform(1 + 0.5 / Wl, 3.0, side.shape), loc[..., 0])
    loc[..., 1] = np.where(side == 2, rng.uniform(-2.0, -0.5 / Hl, side.shape), loc[..., 1])
    loc[..., 1] = np.where(side == 3, rng.uniform(1 + 0.5 / Hl, 3.0, side.shape), loc[..., 1])
    loc = loc.astype(np.float32)
    attn = rng.uniform(0.1, 1, (1, Nq, H, L, P))
    out = oracle.msda_forward(value, shapes, starts, loc, attn)
    assert np.all(out == 0.0)


def test_non_finite_location_reads_nothing():
    shapes, starts, Nv = _levels([(4, 6)])
    value = _rng(5).standard_normal((1, Nv, 1, 2))
    loc = np.full((1, 3, 1, 1, 1, 2), 0.5, np.float32)
    loc[0, 0, 0, 0, 0, 0] = np.nan
    loc[0, 1, 0, 0, 0, 1] = np.inf
    attn = np.ones((1, 3, 1, 1, 1))
    out = oracle.msda_forward(value, shapes, starts, loc, attn)
    assert np.all(out[0, :2] == 0.0) and np.any(out[0, 2] != 0.0)
    go = np.ones_like(out)
    gv, gl, gw = oracle.msda_backward(value, shapes, starts, loc, attn, go)
    assert np.all(gl[0, :2] == 0.0) and np.all(gw[0, :2] == 0.0)


@pytest.mark.parametrize("coord_f32,tol", [(False, 1e-12), (True, 2e-5)])
def test_matches_torch_grid_sample(coord_f32, tol):
    """The bilinear read with zero padding and align_corners=False is exactly
    torch.nn.functional.grid_sample (bilinear, zeros) at grid = 2 s - 1."""
    shapes, starts, Nv = _levels([(7, 11), (4, 5), (3, 2), (1, 1)])
    B, H, Dh, L, P, Nq = 2, 3, 6, 4, 5, 23
    rng = _rng(6)
    value = rng.standard_normal((B, Nv, H, Dh))
    loc = rng.uniform(-0.25, 1.25, (B, Nq, H, L, P, 2)).astype(np.float32).astype(np.float64)
    attn = rng.standard_normal((B, Nq, H, L, P))
    out = oracle.msda_forward(value, shapes, starts, loc, attn, coord_f32=coord_f32)
    ref = _grid_sample_msda(value, shapes, starts, loc, attn)
    np.testing.assert_allclose(out, ref, rtol=0, atol=tol)


def test_one_hot_weight_returns_the_sample():
    shapes, starts, Nv = _levels([(5, 8), (3, 3)])
    B, H, Dh, L, P, Nq = 1, 2, 4, 2, 3, 12
    rng = _rng(7)
    value = rng.standard_normal((B, Nv, H, Dh))
    loc = rng.uniform(-0.1, 1.1, (B, Nq, H, L, P, 2))
    pick = rng.integers(0, L * P, (B, Nq, H))
    attn = np.zeros((B, Nq, H, L * P))
    np.put_along_axis(attn, pick[..., None], 1.0, axis=-1)
    attn = attn.reshape(B, Nq, H, L, P)
    out = oracle.msda_forward(value, shapes, starts, loc, attn, coord_f32=False)
    ref = _grid_sample_msda(value, shapes, starts, loc, attn)
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)


# --------------------------------------------------------------------------
# weighted sum and head concat (sections 7-9, 15)
# --------------------------------------------------------------------------

def _pixel_centre(x, y, W, H):
    return np.float32((x + 0.5) / W), np.float32((y + 0.5) / H)


def test_section7_alpha_times_f():
    g = json.load(open(os.path.join(GOLDEN, "bq_s7_alpha_times_f.json")))
    f = np.asarray(g["f"])
    shapes, starts, Nv = _levels([(1, 1)])
    value = f.reshape(1, 1, 1, 3)
    loc = np.full((1, 1, 1, 1, 1, 2), 0.5, np.float32)
    attn = np.full((1, 1, 1, 1, 1), g["alpha"])
    out = oracle.msda_forward(value, shapes, starts, loc, attn)
    np.testing.assert_allclose(out.reshape(-1), g["expected"], rtol=1e-15)


def _section15_problem(g):
    """A 1x2 value map whose pixel centres hold the example's sampled vectors:
    pixel 0 holds f_1 and pixel 1 holds f_2 of each head."""
    f = np.asarray(g["f"])                  # [head, sample, channel]
    H, S, Dh = f.shape
    shapes, starts, Nv = _levels([(1, S)])
    value = f.transpose(1, 0, 2)[None]      # [1, Nv = S, H, Dh]
    loc = np.zeros((1, 1, H, 1, S, 2), np.float32)
    for k in range(S):
        loc[0, 0, :, 0, k, :] = _pixel_centre(k, 0, S, 1)
    return value, shapes, starts, loc


def test_section15_two_head_example():
    g = json.load(open(os.path.join(GOLDEN, "bq_s15_two_head_example.json")))
    value, shapes, starts, loc = _section15_problem(g)
    attn = np.asarray(g["alpha"])[None, None, :, None, :]
    out = oracle.msda_forward(value, shapes, starts, loc, attn)
    np.testing.assert_allclose(out.reshape(-1), g["g"], rtol=1e-14)
    # identity output projection, dropout off: q_hat = q + g
    np.testing.assert_allclose(np.asarray(g["q"]) + out.reshape(-1), g["q_hat"], rtol=1e-14)


def test_section15_through_the_fused_path():
    """Logits log(alpha) softmax back to alpha; zero offsets from the pixel
    centres (one reference point per sample, R = 2) read the same vectors."""
    g = json.load(open(os.path.join(GOLDEN, "bq_s15_two_head_example.json")))
    value, shapes, starts, loc = _section15_problem(g)
    H, S = np.asarray(g["alpha"]).shape
    ref = loc[:, :, 0, 0, :, :].copy()            # [1, 1, R = S, 2]
    off = np.zeros((1, 1, H, 1, S, 2))
    logits = np.log(np.asarray(g["alpha"]))[None, None, :, None, :]
    out = oracle.msda_forward_fused(value, shapes, starts, ref, off, logits)
    np.testing.assert_allclose(out.reshape(-1), g["g"], rtol=1e-12)


# --------------------------------------------------------------------------
# location (section 5)
# --------------------------------------------------------------------------

def test_anchor_of_point_k_is_k_mod_R():
    """Section 5: with 4 anchors, point k = 4 j + m starts from anchor m.
    Each anchor sits on a pixel centre holding a distinct value; a one-hot
    weight on point k must read the pixel of anchor k mod 4."""
    shapes, starts, Nv = _levels([(3, 10)])
    R, P, H, Dh = 4, 8, 1, 1
    value = np.arange(Nv, dtype=np.float64).reshape(1, Nv, 1, 1) + 100
    anchors = [(1, 0), (4, 1), (7, 2), (9, 1)]   # (x, y) per anchor
    ref = np.array([[_pixel_centre(x, y, 10, 3) for (x, y) in anchors]], np.float32)[None]
    off = np.zeros((1, P, H, 1, P, 2))
    logits = np.full((1, P, H, 1, P), -1e30)
    for q in range(P):
        logits[0, q, 0, 0, q] = 0.0
    ref = np.repeat(ref, P, axis=1)
    out = oracle.msda_forward_fused(value, shapes, starts, ref, off, logits).reshape(-1)
    expect = [100 + anchors[k % 4][1] * 10 + anchors[k % 4][0] for k in range(P)]
    np.testing.assert_array_equal(out, expect)


def test_offsets_are_in_level_pixels():
    """Section 5: the offset is divided by the level's width (x) and height
    (y), so an offset of (+1, 0) / (0, +1) moves the read by exactly one pixel
    on every level, whatever its size."""
    shapes, starts, Nv = _levels([(6, 10), (3, 5), (2, 7)])
    L, P, R, H, Dh = 3, 3, 1, 1, 1
    value = np.arange(Nv, dtype=np.float64).reshape(1, Nv, 1, 1)
    # anchor on the centre of pixel (2, 1) of a 10x6 grid: normalised, it is a
    # different pixel on each level; read one level at a time
    for l, (Hl, Wl) in enumerate(shapes):
        x, y = 1, 0
        ref = np.array(_pixel_centre(x, y, Wl, Hl), np.float32).reshape(1, 1, 1, 2)
        ref = np.repeat(ref, P, axis=1)
        off = np.zeros((1, P, H, L, P, 2))
        off[0, 1, 0, :, 1, 0] = 1.0       # query 1: point 1 one pixel right
        off[0, 2, 0, :, 2, 1] = 1.0       # query 2: point 2 one pixel down
        logits = np.full((1, P, H, L, P), -1e30)
        for q in range(P):
            logits[0, q, 0, l, q] = 0.0
        out = oracle.msda_forward_fused(value, shapes, starts, ref, off, logits).reshape(-1)
        base = starts[l] + y * Wl + x
        np.testing.assert_allclose(out, [base, base + 1, base + Wl], rtol=0, atol=1e-4)


# --------------------------------------------------------------------------
# compaction (rebatch listing) and camera average (section 10, average listing)
# --------------------------------------------------------------------------

def _random_mask(rng, Ncam, B, Nq, R, p=0.3):
    return (rng.random((Ncam, B, Nq, R)) < p).astype(np.uint8)


def test_compaction_brute_force():
    rng = _rng(8)
    Ncam, B, Nq, R = 5, 3, 97, 3
    mask = _random_mask(rng, Ncam, B, Nq, R, 0.2)
    idx, cnt, pos, hits = oracle.sca_compact(mask)
    for b in range(B):
        for c in range(Ncam):
            seen = [q for q in range(Nq) if any(mask[c, b, q, r] for r in range(R))]
            n = len(seen)
            assert cnt[b, c] == n
            assert list(idx[b, c, :n]) == seen
            assert np.all(idx[b, c, n:] == -1)
            # numpy's nonzero of the summed mask, as the rebatch listing does
            np.testing.assert_array_equal(idx[b, c, :n], np.nonzero(mask[c, b].sum(-1))[0])
            for q in range(Nq):
                assert pos[b, c, q] == (seen.index(q) if q in seen else -1)
    np.testing.assert_array_equal(hits, (mask.sum(-1) > 0).transpose(1, 2, 0).sum(-1))
    assert cnt.sum() == hits.sum()


def test_compaction_edge_cases():
    for (Ncam, B, Nq, R) in [(1, 1, 1, 1), (3, 2, 0, 2), (2, 1, 33, 4)]:
        for fill in (0, 1):
            mask = np.full((Ncam, B, Nq, R), fill, np.uint8)
            idx, cnt, pos, hits = oracle.sca_compact(mask)
            assert np.all(cnt == (Nq if fill else 0))
            if Nq:
                assert np.all(hits == (Ncam if fill else 0))
                if fill:
                    assert np.all(idx == np.arange(Nq)) and np.all(pos == np.arange(Nq))
                else:
                    assert np.all(idx == -1) and np.all(pos == -1)


def _tiny_sca(seed, B=2, Ncam=3, bev=(2, 4), shapes=((3, 5), (2, 2)), H=2, Dh=3, P=4, R=2,
              p_mask=0.35):
    rng = _rng(seed)
    shapes, starts, Nv = _levels(list(shapes))
    L = len(shapes)
    Nq = bev[0] * bev[1]
    value = rng.standard_normal((B, Ncam, Nv, H, Dh))
    ref = rng.uniform(0.05, 0.95, (Ncam, B, Nq, R, 2))
    mask = _random_mask(rng, Ncam, B, Nq, R, p_mask)
    mask[:, 0, 0, :] = 0          # a query no camera sees
    mask[:, 0, 1, 0] = 1          # a query every camera sees
    off = rng.standard_normal((B, Nq, H, L, P, 2)) * 0.7
    logits = rng.standard_normal((B, Nq, H, L, P))
    return dict(value=value, shapes=shapes, starts=starts, ref=ref, mask=mask, off=off,
                logits=logits, B=B, Ncam=Ncam, Nq=Nq, H=H, Dh=Dh, L=L, P=P, R=R)


@pytest.mark.parametrize("coord_f32", [True, False])
def test_sca_equals_per_query_camera_mean(coord_f32):
    """The rebatch / scatter-add / clamp(count, 1) pipeline equals a direct
    per-query mean over the cameras that see the query, with no rebatching."""
    t = _tiny_sca(9)
    ref32 = t["ref"].astype(np.float32) if coord_f32 else t["ref"]
    off32 = t["off"].astype(np.float32) if coord_f32 else t["off"]
    out = oracle.sca_forward(t["value"], t["shapes"], t["starts"], ref32, t["mask"], off32,
                             t["logits"], coord_f32=coord_f32)
    expect = np.zeros_like(out)
    for b in range(t["B"]):
        for q in range(t["Nq"]):
            cams = [c for c in range(t["Ncam"]) if t["mask"][c, b, q].any()]
            for c in cams:
                one = oracle.msda_forward_fused(
                    t["value"][b:b + 1, c], t["shapes"], t["starts"],
                    ref32[c, b:b + 1, q:q + 1], off32[b:b + 1, q:q + 1],
                    t["logits"][b:b + 1, q:q + 1], coord_f32=coord_f32)
                expect[b, q] += one[0, 0] / len(cams)
    np.testing.assert_allclose(out, expect, rtol=1e-12, atol=1e-14)
    assert np.all(out[0, 0] == 0.0)  # seen by no camera: zero


def test_sca_single_camera_is_plain_msda():
    t = _tiny_sca(10)
    mask = np.zeros_like(t["mask"])
    mask[1, :, :, 0] = 1          # only camera 1 sees every query
    out = oracle.sca_forward(t["value"], t["shapes"], t["starts"], t["ref"], mask, t["off"],
                             t["logits"], coord_f32=False)
    plain = oracle.msda_forward_fused(t["value"][:, 1], t["shapes"], t["starts"], t["ref"][1],
                                      t["off"], t["logits"], coord_f32=False)
    np.testing.assert_allclose(out, plain, rtol=1e-14, atol=0)


def test_sca_rebatched_rows_follow_compaction():
    t = _tiny_sca(11)
    out, rb = oracle.sca_forward(t["value"], t["shapes"], t["starts"], t["ref"], t["mask"],
                                 t["off"], t["logits"], coord_f32=False, return_rebatched=True)
    idx, cnt, pos, hits = oracle.sca_compact(t["mask"])
    for b in range(t["B"]):
        acc = np.zeros_like(out[b])
        for c in range(t["Ncam"]):
            n = cnt[b, c]
            assert np.all(rb[b, c, n:] == 0.0)
            acc[idx[b, c, :n]] += rb[b, c, :n]
        np.testing.assert_allclose(out[b], acc / np.maximum(hits[b], 1)[:, None], rtol=1e-14)


def test_camera_average_is_the_mean_of_the_seeing_cameras():
    """The average step on its own: for every query, numpy's mean over the
    rows of the cameras whose mask sees it (each row found through idx, not
    through pos), zero for a query no camera sees."""
    rng = _rng(12)
    Ncam, B, Nq, R, HD = 4, 2, 37, 2, 5
    mask = _random_mask(rng, Ncam, B, Nq, R, 0.3)
    mask[:, 0, 0, :] = 0          # a query no camera sees
    mask[:, 0, 1, 0] = 1          # a query every camera sees
    idx, _, pos, hits = oracle.sca_compact(mask)
    rb = rng.standard_normal((B, Ncam, Nq, HD))
    out = oracle.sca_camera_average(rb, pos, hits)
    for b in range(B):
        for q in range(Nq):
            cams = [c for c in range(Ncam) if mask[c, b, q].any()]
            rows = [rb[b, c, list(idx[b, c]).index(q)] for c in cams]
            expect = np.mean(rows, axis=0) if rows else np.zeros(HD)
            np.testing.assert_allclose(out[b, q], expect, rtol=1e-13, atol=1e-15)
    assert np.all(out[0, 0] == 0.0)


def test_camera_average_closed_forms():
    """One seeing camera returns its row unchanged; six cameras with equal
    rows of small integers return that row exactly; rows past a camera's
    count are never read."""
    Ncam, B, Nq, HD = 6, 1, 3, 4
    mask = np.zeros((Ncam, B, Nq, 1), np.uint8)
    mask[2, 0, 0, 0] = 1          # query 0: camera 2 only
    mask[:, 0, 1, 0] = 1          # query 1: all six
    _, cnt, pos, hits = oracle.sca_compact(mask)
    rb = np.full((B, Ncam, Nq, HD), np.nan)
    for c in range(Ncam):
        rb[0, c, :cnt[0, c]] = 3.0
    rb[0, 2, 0] = [1.0, -2.0, 0.5, 7.0]
    out = oracle.sca_camera_average(rb, pos, hits)
    np.testing.assert_array_equal(out[0, 0], [1.0, -2.0, 0.5, 7.0])
    np.testing.assert_array_equal(out[0, 1], np.full(HD, 3.0))
    np.testing.assert_array_equal(out[0, 2], np.zeros(HD))


def test_camera_average_of_the_rebatched_rows_is_sca_forward():
    t = _tiny_sca(13)
    out, rb = oracle.sca_forward(t["value"], t["shapes"], t["starts"], t["ref"], t["mask"],
                                 t["off"], t["logits"], coord_f32=False, return_rebatched=True)
    _, _, pos, hits = oracle.sca_compact(t["mask"])
    np.testing.assert_array_equal(oracle.sca_camera_average(rb, pos, hits), out)


# --------------------------------------------------------------------------
# backward: central finite differences and linearity
# --------------------------------------------------------------------------

def _fd_locations(rng, shape, shapes, margin=1e-3):
    """Locations whose pixel coordinates stay >= margin away from integers,
    so that +-h never crosses a cell boundary."""
    loc = rng.uniform(-0.15, 1.15, shape)
    L = shape[3]
    for l in range(L):
        Hl, Wl = shapes[l]
        for ax, n in ((0, Wl), (1, Hl)):
            x = loc[..., l, :, ax] * n - 0.5
            fr = x - np.floor(x)
            x = np.floor(x) + np.clip(fr, margin, 1 - margin)
            loc[..., l, :, ax] = (x + 0.5) / n
    return loc


def _tiny_msda(seed):
    rng = _rng(seed)
    shapes, starts, Nv = _levels([(3, 5), (2, 2)])
    B, H, Dh, L, P, Nq = 1, 2, 3, 2, 2, 3
    value = rng.standard_normal((B, Nv, H, Dh))
    loc = _fd_locations(rng, (B, Nq, H, L, P, 2), shapes)
    attn = rng.uniform(0.1, 1.0, (B, Nq, H, L, P))
    go = rng.standard_normal((B, Nq, H * Dh))
    return value, shapes, starts, loc, attn, go


def _central_fd(f, x, h):
    g = np.zeros_like(x)
    flat = x.reshape(-1)
    gf = g.reshape(-1)
    for i in range(flat.size):
        keep = flat[i]
        flat[i] = keep + h
        up = f()
        flat[i] = keep - h
        dn = f()
        flat[i] = keep
        gf[i] = (up - dn) / (2 * h)
    return g


def test_msda_backward_matches_finite_differences():
    value, shapes, starts, loc, attn, go = _tiny_msda(12)

    def loss():
        return float(np.sum(go * oracle.msda_forward(value, shapes, starts, loc, attn,
                                                     coord_f32=False)))

    gv, gl, gw = oracle.msda_backward(value, shapes, starts, loc, attn, go, coord_f32=False)
    h = 1e-6
    np.testing.assert_allclose(gv, _central_fd(loss, value, h), rtol=1e-6, atol=1e-8)
    np.testing.assert_allclose(gw, _central_fd(loss, attn, h), rtol=1e-6, atol=1e-8)
    np.testing.assert_allclose(gl, _central_fd(loss, loc, h), rtol=1e-6, atol=1e-7)
    assert np.abs(gl).max() > 0.1  # the check is not vacuous


def test_msda_backward_with_partly_outside_samples():
    """Samples whose neighbourhood straddles the border (zero padding)."""
    rng = _rng(13)
    shapes, starts, Nv = _levels([(3, 4)])
    B, H, Dh, L, P, Nq = 1, 1, 2, 1, 6, 4
    value = rng.standard_normal((B, Nv, H, Dh))
    # pixel coordinates in (-1, 0) or (W-1, W): one neighbour column outside
    loc = _fd_locations(rng, (B, Nq, H, L, P, 2), shapes)
    loc[..., 0, 0::2, 0] = (rng.uniform(-0.9, -0.1, (B, Nq, H, 3)) + 0.5) / 4
    loc[..., 0, 1::2, 1] = (rng.uniform(2.1, 2.9, (B, Nq, H, 3)) + 0.5) / 3
    attn = rng.uniform(0.1, 1.0, (B, Nq, H, L, P))
    go = rng.standard_normal((B, Nq, H * Dh))

    def loss():
        return float(np.sum(go * oracle.msda_forward(value, shapes, starts, loc, attn,
                                                     coord_f32=False)))

    gv, gl, gw = oracle.msda_backward(value, shapes, starts, loc, attn, go, coord_f32=False)
    h = 1e-6
    np.testing.assert_allclose(gv, _central_fd(loss, value, h), rtol=1e-6, atol=1e-8)
    np.testing.assert_allclose(gl, _central_fd(loss, loc, h), rtol=1e-6, atol=1e-7)
    np.testing.assert_allclose(gw, _central_fd(loss, attn, h), rtol=1e-6, atol=1e-8)


def test_msda_backward_linearity():
    """out is linear in the weights and in the value: <gO, out> equals
    sum(gW * alpha) and sum(gV * V)."""
    rng = _rng(14)
    shapes, starts, Nv = _levels([(9, 13), (4, 7), (2, 3)])
    B, H, Dh, L, P, Nq = 2, 3, 8, 3, 4, 31
    value = rng.standard_normal((B, Nv, H, Dh))
    loc = rng.uniform(-0.1, 1.1, (B, Nq, H, L, P, 2)).astype(np.float32)
    attn = rng.uniform(0, 1, (B, Nq, H, L, P))
    go = rng.standard_normal((B, Nq, H * Dh))
    out = oracle.msda_forward(value, shapes, starts, loc, attn)
    gv, gl, gw = oracle.msda_backward(value, shapes, starts, loc, attn, go)
    lhs = np.sum(go * out)
    np.testing.assert_allclose(np.sum(gw * attn), lhs, rtol=1e-12)
    np.testing.assert_allclose(np.sum(gv * value), lhs, rtol=1e-12)


def test_sca_backward_matches_finite_differences():
    """FD through the whole SCA forward: grad_value directly, and the
    gradients of the offsets, reference points and logits that
    oracle.sca_backward_inputs forms from the rebatched location and weight
    gradients."""
    t = _tiny_sca(15)
    rng = _rng(16)
    B, Ncam, Nq, H, Dh, L, P, R = (t[k] for k in ("B", "Ncam", "Nq", "H", "Dh", "L", "P", "R"))
    go = rng.standard_normal((B, Nq, H * Dh))
    shapes, starts = t["shapes"], t["starts"]
    # keep pixel coordinates away from cell boundaries
    for _ in range(50):
        loc, _w = oracle.fused_locations(shapes, t["ref"][0], t["off"], t["logits"], coord_f32=False)
        ok = True
        for c in range(Ncam):
            loc_c, _ = oracle.fused_locations(shapes, t["ref"][c], t["off"], t["logits"],
                                              coord_f32=False)
            for l, (Hl, Wl) in enumerate(shapes):
                for ax, n in ((0, Wl), (1, Hl)):
                    x = loc_c[..., l, :, ax] * n - 0.5
                    fr = x - np.floor(x)
                    ok &= bool(np.all((fr > 1e-3) & (fr < 1 - 1e-3)))
        if ok:
            break
        t["off"] += rng.uniform(-0.05, 0.05, t["off"].shape)
    assert ok

    def loss():
        return float(np.sum(go * oracle.sca_forward(t["value"], shapes, starts, t["ref"],
                                                     t["mask"], t["off"], t["logits"],
                                                     coord_f32=False)))

    gv, gl_rb, gw_rb = oracle.sca_backward(t["value"], shapes, starts, t["ref"], t["mask"],
                                           t["off"], t["logits"], go, coord_f32=False)
    h = 1e-6
    np.testing.assert_allclose(gv, _central_fd(loss, t["value"], h), rtol=1e-6, atol=1e-8)

    idx, cnt, pos, hits = oracle.sca_compact(t["mask"])
    for b in range(B):
        for c in range(Ncam):
            assert np.all(gl_rb[b, c, cnt[b, c]:] == 0) and np.all(gw_rb[b, c, cnt[b, c]:] == 0)
    g_off, g_logits, g_ref = oracle.sca_backward_inputs(shapes, t["mask"], t["logits"], gl_rb,
                                                        gw_rb)
    np.testing.assert_allclose(g_off, _central_fd(loss, t["off"], h), rtol=1e-6, atol=1e-7)
    np.testing.assert_allclose(g_ref, _central_fd(loss, t["ref"], h), rtol=1e-6, atol=1e-7)
    np.testing.assert_allclose(g_logits, _central_fd(loss, t["logits"], h), rtol=1e-6, atol=1e-8)
    assert np.abs(g_off).max() > 0.05


def test_empty_problems():
    shapes, starts, Nv = _levels([(2, 3)])
    value = np.zeros((1, Nv, 1, 2))
    out = oracle.msda_forward(value, shapes, starts, np.zeros((1, 0, 1, 1, 1, 2)),
                              np.zeros((1, 0, 1, 1, 1)))
    assert out.shape == (1, 0, 2)
    with pytest.raises(ValueError):
        oracle.msda_forward(value, [(3, 3)], [0], np.zeros((1, 1, 1, 1, 1, 2)),
                            np.zeros((1, 1, 1, 1, 1)))  # level larger than the value map


# --------------------------------------------------------------------------
# dense projections (sections 3, 4.1, 4.2, 11, 13)
# --------------------------------------------------------------------------

def test_linear_matches_numpy_matmul():
    rng = _rng(40)
    x = rng.standard_normal((37, 24))
    w = rng.standard_normal((11, 24))
    b = rng.standard_normal(11)
    r = rng.standard_normal((37, 11))
    np.testing.assert_allclose(oracle.linear(x, w, b, r), x @ w.T + b + r, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(oracle.linear(x, w), x @ w.T, rtol=1e-12, atol=1e-12)


def test_linear_identity_weight():
    x = _rng(41).standard_normal((5, 8))
    np.testing.assert_array_equal(oracle.linear(x, np.eye(8)), x)


def test_section15_output_projection_and_residual():
    """Identity W_o, dropout off: q_hat = q + W_o g = [9, 3.6, 9, 3]."""
    g = json.load(open(os.path.join(GOLDEN, "bq_s15_two_head_example.json")))
    q_hat = oracle.linear(np.asarray(g["g"])[None], np.eye(4), None, np.asarray(g["q"])[None])
    np.testing.assert_allclose(q_hat[0], g["q_hat"], rtol=1e-15)


def test_round_bf16_ties_to_even():
    # 1 + 2^-8 is halfway between the bf16 neighbours 1 and 1 + 2^-7: to even (1)
    x = np.array([1.0, 1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -2.5, 3.0e-3])
    r = oracle.round_bf16(x)
    assert r[0] == 1.0 and r[1] == 1.0 and r[2] == 1.0 + 2.0 ** -6 and r[3] == -2.5
    assert abs(r[4] - 3.0e-3) <= 2.0 ** -8 * 3.0e-3  # half an ulp of an 8-bit significand


def test_module_with_identity_projections_is_residual_plus_sca():
    """W_v = I, zero offset/weight heads except their biases, W_o = I: the
    module returns q + bf16(SCA(V = F~)) (sections 13 and 10)."""
    rng = _rng(42)
    B, Ncam, Nq, C, L, P, R = 1, 2, 6, 32, 2, 2, 2
    shapes, starts, Nv = _levels([(3, 4), (2, 2)])
    q = rng.standard_normal((B, Nq, C))
    feats = oracle.round_bf16(rng.standard_normal((B, Ncam, Nv, C)))
    ref = rng.uniform(0.1, 0.9, (Ncam, B, Nq, R, 2))
    mask = (rng.random((Ncam, B, Nq, R)) < 0.6).astype(np.uint8)
    S = 1 * L * P
    b_off = rng.standard_normal(S * 2) * 0.5
    b_w = rng.standard_normal(S)
    y = oracle.sca_module_forward(q, None, feats, np.eye(C), None, np.zeros((2 * S, C)), b_off,
                                  np.zeros((S, C)), b_w, np.eye(C), None, ref, mask, shapes,
                                  starts, L, P)
    off = np.broadcast_to(b_off.reshape(1, 1, 1, L, P, 2), (B, Nq, 1, L, P, 2))
    lg = np.broadcast_to(b_w.reshape(1, 1, 1, L, P), (B, Nq, 1, L, P))
    g = oracle.sca_forward(feats.reshape(B, Ncam, Nv, 1, C), shapes, starts, ref, mask, off, lg)
    np.testing.assert_allclose(y, q + oracle.round_bf16(g), rtol=1e-12, atol=1e-12)


# --------------------------------------------------------------------------
# TSA: ego-motion reference points and the queue mean ("【论文阅读】BEVFormer
# 论文解析及Temporal Self-Attention、Spatial Cross-Attention注意力机制详解及
# 代码示例", section 二.2 and the BEV encoder listing)
# --------------------------------------------------------------------------

def _cell_centres(bev_h, bev_w):
    i, j = np.meshgrid(np.arange(bev_h), np.arange(bev_w), indexing="ij")
    return np.stack([(j + 0.5) / bev_w, (i + 0.5) / bev_h], -1).reshape(-1, 2)


def test_tsa_reference_points_without_motion_are_cell_centres():
    ref = oracle.tsa_reference_points(5, 7, np.zeros((2, 2, 3)))
    for b in range(2):
        for t in range(2):
            np.testing.assert_allclose(ref[b, t], _cell_centres(5, 7), rtol=0, atol=1e-15)


def test_tsa_reference_points_whole_cell_translation():
    """No rotation, a motion of (3 cells, -2 cells): the point seen is the
    centre of cell (i - 2, j + 3).  Unequal grid lengths pin x to the width."""
    gy, gx = 0.3, 0.512
    ego = np.array([[[3 * gx, -2 * gy, 0.0]]])
    ref = oracle.tsa_reference_points(6, 9, ego, grid_length=(gy, gx))[0, 0]
    want = _cell_centres(6, 9) + np.array([3 / 9, -2 / 6])
    np.testing.assert_allclose(ref, want, rtol=0, atol=1e-14)


def test_tsa_reference_points_are_a_rigid_motion():
    """Distances in metres are kept, and the centroid of the cell centres
    (the BEV centre) lands on the translation."""
    gy, gx = 0.4, 0.512
    H, W = 7, 10
    ego = np.array([[[1.3, -0.7, 33.0]]])
    ref = oracle.tsa_reference_points(H, W, ego, grid_length=(gy, gx))[0, 0]
    metres = (ref - 0.5) * np.array([W * gx, H * gy])
    base = (_cell_centres(H, W) - 0.5) * np.array([W * gx, H * gy])
    d_new = np.linalg.norm(metres[:, None] - metres[None], axis=-1)
    d_old = np.linalg.norm(base[:, None] - base[None], axis=-1)
    np.testing.assert_allclose(d_new, d_old, rtol=0, atol=1e-12)
    np.testing.assert_allclose(metres.mean(0), [1.3, -0.7], rtol=0, atol=1e-12)


def _tsa_point_sampler(prev, cur, ego_prev):
    """Both queues sampled with one point, zero offsets: the output is the
    mean of the two maps read at each queue's reference point."""
    N, _, D = prev.shape
    shapes, starts, Nv = _levels([(N, N)])
    value = np.stack([prev.reshape(Nv, 1, D), cur.reshape(Nv, 1, D)])
    ego = np.array([[ego_prev, [0.0, 0.0, 0.0]]])
    ref = oracle.tsa_reference_points(N, N, ego).reshape(2, N * N, 1, 2)
    off = np.zeros((2, N * N, 1, 1, 1, 2))
    lg = np.zeros((2, N * N, 1, 1, 1))
    return oracle.tsa_forward(value, shapes, starts, ref, off, lg, 2)[0].reshape(N, N, D)


@pytest.mark.parametrize("angle,turns", [(90.0, 1), (180.0, 2), (-90.0, 3)])
def test_tsa_quarter_turns_rotate_the_previous_map(angle, turns):
    """A yaw of k * 90 degrees about the BEV centre moves cell centres onto
    cell centres: the previous queue then returns its map turned like
    numpy's rot90 (x along the columns, counter-clockwise from +x to +y), and
    the output is the mean with the current map."""
    rng = _rng(60)
    N, D = 6, 3
    prev, cur = rng.standard_normal((N, N, D)), rng.standard_normal((N, N, D))
    out = _tsa_point_sampler(prev, cur, [0.0, 0.0, angle])
    want = 0.5 * (np.rot90(prev, turns, axes=(0, 1)) + cur)
    np.testing.assert_allclose(out, want, rtol=0, atol=1e-6)


def test_tsa_whole_cell_shift_moves_the_previous_map():
    """A motion of one cell along +x and two along -y reads cell (i - 2, j + 1)
    of the previous map; cells whose source leaves the map read zero."""
    rng = _rng(61)
    N, D = 7, 2
    prev, cur = rng.standard_normal((N, N, D)), rng.standard_normal((N, N, D))
    out = _tsa_point_sampler(prev, cur, [0.512, -2 * 0.512, 0.0])
    shifted = np.zeros_like(prev)
    shifted[2:, :N - 1] = prev[:N - 2, 1:]
    np.testing.assert_allclose(out, 0.5 * (shifted + cur), rtol=0, atol=1e-6)


def test_tsa_single_queue_is_the_fused_msda():
    w = inputs.workload4(bev_h=9, bev_w=11)
    out = oracle.tsa_forward(w.value[:1], w.spatial_shapes, w.level_start_index,
                             w.reference_points[:1], w.sampling_offsets[:1],
                             w.attention_logits[:1], 1)
    ref = oracle.msda_forward_fused(w.value[:1], w.spatial_shapes, w.level_start_index,
                                    w.reference_points[:1], w.sampling_offsets[:1],
                                    w.attention_logits[:1])
    np.testing.assert_array_equal(out, ref)


def test_tsa_mean_is_symmetric_in_the_queues():
    w = inputs.workload4(bev_h=9, bev_w=11)
    args = (w.value, w.reference_points, w.sampling_offsets, w.attention_logits)
    a = oracle.tsa_forward(args[0], w.spatial_shapes, w.level_start_index, *args[1:], 2)
    b = oracle.tsa_forward(*(x[::-1] for x in args[:1]), w.spatial_shapes, w.level_start_index,
                           *(x[::-1] for x in args[1:]), 2)
    np.testing.assert_allclose(a, b, rtol=0, atol=1e-14)
    same = oracle.tsa_forward(np.concatenate([args[0][:1]] * 2), w.spatial_shapes,
                              w.level_start_index,
                              *(np.concatenate([x[:1]] * 2) for x in args[1:]), 2)
    one = oracle.msda_forward_fused(args[0][:1], w.spatial_shapes, w.level_start_index,
                                    *(x[:1] for x in args[1:]))
    np.testing.assert_allclose(same, one, rtol=0, atol=1e-14)


# --------------------------------------------------------------------------
# training-time dropout (section 12) with Philox4x32-10 (Salmon, Moraes,
# Dror, Shaw, "Parallel random numbers: as easy as 1, 2, 3", SC 2011)
# --------------------------------------------------------------------------

# the generator's published known-answer vectors: (counter, key) -> output
PHILOX_KAT = [
    ((0, 0, 0, 0), (0, 0), (0x6627E8D5, 0xE169C58D, 0xBC57AC4C, 0x9B00DBD8)),
    ((0xFFFFFFFF,) * 4, (0xFFFFFFFF,) * 2, (0x408F276D, 0x41C83B0E, 0xA20BC7C6, 0x6D5451FD)),
    ((0x243F6A88, 0x85A308D3, 0x13198A2E, 0x03707344), (0xA4093822, 0x299F31D0),
     (0xD16CFE09, 0x94FDCCEB, 0x5001E420, 0x24126EA1)),
]


@pytest.mark.parametrize("ctr,key,want", PHILOX_KAT)
def test_philox_known_answers(ctr, key, want):
    assert [int(x) for x in oracle.philox4x32_10(ctr, key)] == list(want)


def test_dropout_zero_rate_is_identity():
    o = _rng(70).standard_normal((13, 7))
    np.testing.assert_array_equal(oracle.dropout(o, 0.0, 123), o)


def test_dropout_keeps_and_scales():
    """Kept elements are o / (1 - p) exactly, dropped ones 0, the kept
    fraction is 1 - p within five standard deviations, the mask follows the
    element index only (not the values), and another seed gives another mask."""
    p, n = 0.1, 1 << 18
    o = _rng(71).uniform(1.0, 2.0, n)
    y = oracle.dropout(o, p, 2024)
    kept = y != 0
    np.testing.assert_array_equal(y[kept], o[kept] / (1 - p))
    sigma = np.sqrt(n * p * (1 - p))
    assert abs(kept.sum() - n * (1 - p)) < 5 * sigma
    y2 = oracle.dropout(o * 3.0 + 1.0, p, 2024)
    np.testing.assert_array_equal(y2 != 0, kept)
    y3 = oracle.dropout(o, p, 2025)
    assert 0.1 * n < np.count_nonzero((y3 != 0) != kept) < 0.3 * n


def test_dropout_mask_is_the_generator_words():
    """Element e is kept iff word e mod 4 of Philox at counter (e div 4) and
    key (seed) is at least p * 2^32 (checked on a few elements by hand)."""
    p, seed = 0.25, (7 << 32) | 5
    y = oracle.dropout(np.ones(40), p, seed)
    for e in (0, 1, 2, 3, 4, 17, 39):
        u = oracle.philox4x32_10((e // 4, 0, 0, 0), (5, 7))[e % 4]
        assert (y[e] != 0) == (int(u) >= int(p * 2 ** 32))


def test_module_embeddings_are_added_to_the_features():
    """[BQ] 3: F~ = F + e_cam + e_level.  Passing the embeddings equals passing
    features that already hold them, built here by indexing each pixel's
    camera and level independently (a level per row from the level table)."""
    rng = _rng(43)
    B, Ncam, Nq, C, L, P, R = 1, 3, 5, 32, 2, 2, 1
    shapes, starts, Nv = _levels([(3, 4), (2, 2)])
    q = rng.standard_normal((B, Nq, C))
    feats = oracle.round_bf16(rng.standard_normal((B, Ncam, Nv, C)))
    e_cam = rng.standard_normal((Ncam, C))
    e_lvl = rng.standard_normal((L, C))
    ref = rng.uniform(0.1, 0.9, (Ncam, B, Nq, R, 2))
    mask = np.ones((Ncam, B, Nq, R), np.uint8)
    S = L * P
    wv, wo = rng.standard_normal((C, C)) / 8, rng.standard_normal((C, C)) / 8
    woff, ww = rng.standard_normal((2 * S, C)) / 8, rng.standard_normal((S, C)) / 8
    level_of_row = np.concatenate([np.full(h * w, l) for l, (h, w) in enumerate(shapes)])
    tilde = feats + e_cam[None, :, None, :] + e_lvl[level_of_row][None, None, :, :]
    common = (None, wv, None, woff, None, ww, None, wo, None, ref, mask, shapes, starts, L, P)
    a = oracle.sca_module_forward(q, None, feats, *common[1:], camera_embeds=e_cam,
                                  level_embeds=e_lvl)
    b = oracle.sca_module_forward(q, None, tilde, *common[1:])
    np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-12)


def test_tsa_backward_matches_finite_differences():
    """Central differences through the whole TSA forward (two queues, two
    levels, R = 2) for the value, offsets, logits and reference points."""
    rng = _rng(62)
    B, T, Nq, H, Dh, P, R = 1, 2, 3, 2, 3, 2, 2
    shapes, starts, Nv = _levels([(4, 5), (2, 3)])
    L = 2
    value = rng.standard_normal((B * T, Nv, H, Dh))
    ref = rng.uniform(0.2, 0.8, (B * T, Nq, R, 2))
    off = rng.uniform(-0.7, 0.7, (B * T, Nq, H, L, P, 2))
    logits = rng.standard_normal((B * T, Nq, H, L, P))
    go = rng.standard_normal((B, Nq, H * Dh))
    for _ in range(50):  # keep pixel coordinates away from cell boundaries
        loc, _w = oracle.fused_locations(shapes, ref, off, logits, coord_f32=False)
        ok = True
        for l, (Hl, Wl) in enumerate(shapes):
            for ax, n in ((0, Wl), (1, Hl)):
                x = loc[..., l, :, ax] * n - 0.5
                fr = x - np.floor(x)
                ok &= bool(np.all((fr > 1e-3) & (fr < 1 - 1e-3)))
        if ok:
            break
        off += rng.uniform(-0.05, 0.05, off.shape)
    assert ok

    def loss():
        return float(np.sum(go * oracle.tsa_forward(value, shapes, starts, ref, off, logits, T,
                                                     coord_f32=False)))

    gv, g_off, g_lg, g_ref = oracle.tsa_backward(value, shapes, starts, ref, off, logits, T, go,
                                                 coord_f32=False)
    h = 1e-6
    np.testing.assert_allclose(gv, _central_fd(loss, value, h), rtol=1e-6, atol=1e-8)
    np.testing.assert_allclose(g_off, _central_fd(loss, off, h), rtol=1e-6, atol=1e-7)
    np.testing.assert_allclose(g_lg, _central_fd(loss, logits, h), rtol=1e-6, atol=1e-8)
    np.testing.assert_allclose(g_ref, _central_fd(loss, ref, h), rtol=1e-6, atol=1e-7)
    assert np.abs(g_off).max() > 0.02
