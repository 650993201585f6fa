"""The oracle's pins catch plausible mistakes.

Each case below plants one mistake in a private copy of the oracle's C source
(a dropped term, a swapped axis, a wrong sign or index, a transposed
operand), compiles it into a temporary library, points the oracle's NumPy
front end at it and runs the pins of test_oracle_pins.py.  At least one pin
must fail for every mutant.  CPU only; the committed oracle is not touched.
"""
import ctypes
import os
import subprocess

import pytest

import oracle
from . import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "msda_oracle.c")

# (name, text in the oracle, planted replacement, occurrence: 0 = all)
MUTANTS = [
    ("no half-pixel shift", "volatile float c = prod - 0.5f;", "volatile float c = prod;", 0),
    ("half-pixel shift dropped in double", "return (double)n * s - 0.5;", "return (double)n * s;", 0),
    ("y scaled by the width", "pixel_coord(loc_row[2 * s + 1], Hl, coord_f32)",
     "pixel_coord(loc_row[2 * s + 1], Wl, coord_f32)", 0),
    ("neighbours transposed", "int64_t xc = x0 + (g & 1), yc = y0 + (g >> 1);",
     "int64_t xc = x0 + (g >> 1), yc = y0 + (g & 1);", 0),
    ("x weights swapped", "double wx = (g & 1) ? c->lx : 1.0 - c->lx;",
     "double wx = (g & 1) ? 1.0 - c->lx : c->lx;", 0),
    ("border clamp instead of zero padding",
     "if (xc >= 0 && xc < Wl && yc >= 0 && yc < Hl) c.row[g] = start + yc * Wl + xc;",
     "{ int64_t cx = xc < 0 ? 0 : (xc >= Wl ? Wl - 1 : xc); int64_t cy = yc < 0 ? 0 : "
     "(yc >= Hl ? Hl - 1 : yc); c.row[g] = start + cy * Wl + cx; }", 0),
    ("column-major pixel rows", "c.row[g] = start + yc * Wl + xc;",
     "c.row[g] = start + xc * Hl + yc;", 0),
    ("level start ignored", "c.row[g] = start + yc * Wl + xc;", "c.row[g] = yc * Wl + xc;", 0),
    ("head index ignored", "const double* v = vb + (c.row[q] * H + h) * Dh;",
     "const double* v = vb + (c.row[q] * H + 0) * Dh;", 1),
    ("batch offset ignored", "row_forward(value + (int64_t)b * Nv * H * Dh,", "row_forward(value,", 0),
    ("anchor index k / (P/R)", "int m = k % R;", "int m = k / (P / R);", 0),
    ("offset x normalised by the height",
     "fused_location(ref_row[2 * m + 0], off_row[2 * s + 0], Wl, coord_f32)",
     "fused_location(ref_row[2 * m + 0], off_row[2 * s + 0], Hl, coord_f32)", 0),
    ("offset normaliser dropped (binary32)", "volatile float q = (float)d / (float)n;",
     "volatile float q = (float)d;", 0),
    ("offset normaliser dropped (double)", "return rho + d / (double)n;", "return rho + d;", 0),
    ("softmax per level instead of per head", "oracle_softmax(logit_row, H, L * P, attn_row);",
     "oracle_softmax(logit_row, H * L, P, attn_row);", 0),
    ("softmax without normalisation", "for (int i = 0; i < n; ++i) w[i] /= z;", "", 0),
    ("average over all cameras", "int n = sc.hits[bq] > 1 ? sc.hits[bq] : 1;", "int n = Ncam;", 1),
    ("average step over all cameras", "const int n = hits[bq] > 1 ? hits[bq] : 1;",
     "const int n = Ncam;", 0),
    ("average step without the clamp", "const int n = hits[bq] > 1 ? hits[bq] : 1;",
     "const int n = hits[bq];", 0),
    ("average step reads camera 0's positions", "const int32_t i = pos[bc * Nq + q];",
     "const int32_t i = pos[(int64_t)b * Ncam * Nq + q];", 0),
    ("average step reads the query's row", "o[d] += out_rb[(bc * Nq + i) * HD + d];",
     "o[d] += out_rb[(bc * Nq + q) * HD + d];", 0),
    ("only anchor 0 decides a hit", "for (int r = 0; r < R; ++r)\n                    if (bev_mask",
     "for (int r = 0; r < 1; ++r)\n                    if (bev_mask", 0),
    ("camera 0 reference points everywhere",
     "const double* ref_row = ref_cam + (((int64_t)c * B + b) * Nq + q) * R * 2;",
     "const double* ref_row = ref_cam + (((int64_t)0 * B + b) * Nq + q) * R * 2;", 0),
    ("d/dy sign flipped", "double dfdy = (1.0 - c.lx) * (dot[2] - dot[0]) + c.lx * (dot[3] - dot[1]);",
     "double dfdy = (1.0 - c.lx) * (dot[0] - dot[2]) + c.lx * (dot[3] - dot[1]);", 0),
    ("d/dx missing the width", "gloc_row[2 * s + 0] = alpha * (double)Wl * dfdx;",
     "gloc_row[2 * s + 0] = alpha * dfdx;", 0),
    ("grad_value missing the weight", "double w = alpha * corner_weight(&c, q);",
     "double w = corner_weight(&c, q);", 0),
    ("grad_attn missing the bilinear weight", "gw += corner_weight(&c, q) * dot[q];", "gw += dot[q];", 0),
    ("projection weight transposed", "acc += x[(int64_t)m * K + k] * w[(int64_t)n * K + k];",
     "acc += x[(int64_t)m * K + k] * w[(int64_t)k * N + n];", 0),
    ("projection bias dropped", "if (bias) acc += bias[n];", "", 0),
    ("offset gradient not divided by the width",
     "grad_off[(bq * S + s) * 2 + 0] += gl[2 * s + 0] / Wl;", "grad_off[(bq * S + s) * 2 + 0] += gl[2 * s + 0];", 0),
    ("softmax backward without the centring",
     "grad_logits[base + j] = alpha[j] * (G[base + j] - dot);", "grad_logits[base + j] = alpha[j] * G[base + j];", 0),
    ("reference gradient on anchor k / (P/R)", "gr[2 * (k % R) + 0] += gl[2 * s + 0];",
     "gr[2 * (k / (P / R)) + 0] += gl[2 * s + 0];", 0),
    ("SCA backward not divided by the count",
     "sc.row[d] = grad_out[bq * HD + d] / (double)n;", "sc.row[d] = grad_out[bq * HD + d];", 0),
    ("ego rotation sign flipped", "const double qx = cs * px - sn * py + dx;",
     "const double qx = cs * px + sn * py + dx;", 0),
    ("ego rotation about the corner", "const double px = ((double)j + 0.5 - 0.5 * bev_w) * gx;",
     "const double px = ((double)j + 0.5) * gx;", 0),
    ("ego translation in cells", "const double qy = sn * px + cs * py + dy;",
     "const double qy = sn * px + cs * py + dy * gy;", 0),
    ("BEV x normalised by the height grid", "r[0] = qx / (bev_w * gx) + 0.5;",
     "r[0] = qx / (bev_w * gy) + 0.5;", 0),
    ("queue mean not divided", "out[((int64_t)b * Nq + q) * HD + d] = sum / T;",
     "out[((int64_t)b * Nq + q) * HD + d] = sum;", 0),
    ("every queue reads queue 0", "sum += per_queue[(((int64_t)b * T + t) * Nq + q) * HD + d];",
     "sum += per_queue[(((int64_t)b * T + 0) * Nq + q) * HD + d];", 0),
    ("Philox multiplier digits swapped", "(uint64_t)0xD2511F53u * c0", "(uint64_t)0xD2511F35u * c0", 0),
    ("Philox key not bumped", "k0 += 0x9E3779B9u;", "", 0),
    ("dropout without the rescale", "? o[e] / (1.0 - p) : 0.0", "? o[e] : 0.0", 0),
    ("dropout keeps the low draws", "(uint64_t)u[e & 3] >= thr", "(uint64_t)u[e & 3] < thr", 0),
    ("dropout reads the wrong word", "(uint64_t)u[e & 3] >= thr", "(uint64_t)u[(e >> 2) & 3] >= thr", 0),
]

PIN_CALLS = [
    ("softmax_sums", lambda: pins.test_softmax_sums_to_one_per_head()),
    ("softmax_zero", lambda: pins.test_softmax_zero_logits_uniform()),
    ("centres_f32", lambda: pins.test_pixel_centres_reproduce_pixels(True)),
    ("centres_f64", lambda: pins.test_pixel_centres_reproduce_pixels(False)),
    ("constant", lambda: pins.test_constant_map_gives_constant()),
    ("outside", lambda: pins.test_fully_out_of_bounds_is_zero()),
    ("grid_sample_f64", lambda: pins.test_matches_torch_grid_sample(False, 1e-12)),
    ("grid_sample_f32", lambda: pins.test_matches_torch_grid_sample(True, 2e-5)),
    ("section7", lambda: pins.test_section7_alpha_times_f()),
    ("section15", lambda: pins.test_section15_two_head_example()),
    ("section15_fused", lambda: pins.test_section15_through_the_fused_path()),
    ("anchor", lambda: pins.test_anchor_of_point_k_is_k_mod_R()),
    ("offset_pixels", lambda: pins.test_offsets_are_in_level_pixels()),
    ("compaction", lambda: pins.test_compaction_brute_force()),
    ("sca_mean", lambda: pins.test_sca_equals_per_query_camera_mean(False)),
    ("sca_rebatch", lambda: pins.test_sca_rebatched_rows_follow_compaction()),
    ("average_mean", lambda: pins.test_camera_average_is_the_mean_of_the_seeing_cameras()),
    ("average_closed", lambda: pins.test_camera_average_closed_forms()),
    ("msda_fd", lambda: pins.test_msda_backward_matches_finite_differences()),
    ("msda_fd_border", lambda: pins.test_msda_backward_with_partly_outside_samples()),
    ("linearity", lambda: pins.test_msda_backward_linearity()),
    ("sca_fd", lambda: pins.test_sca_backward_matches_finite_differences()),
    ("linear_numpy", lambda: pins.test_linear_matches_numpy_matmul()),
    ("linear_s15", lambda: pins.test_section15_output_projection_and_residual()),
    ("tsa_centres", lambda: pins.test_tsa_reference_points_without_motion_are_cell_centres()),
    ("tsa_translation", lambda: pins.test_tsa_reference_points_whole_cell_translation()),
    ("tsa_rigid", lambda: pins.test_tsa_reference_points_are_a_rigid_motion()),
    ("tsa_rot90", lambda: pins.test_tsa_quarter_turns_rotate_the_previous_map(90.0, 1)),
    ("tsa_shift", lambda: pins.test_tsa_whole_cell_shift_moves_the_previous_map()),
    ("philox_kat", lambda: [pins.test_philox_known_answers(*k) for k in pins.PHILOX_KAT]),
    ("dropout_scale", lambda: pins.test_dropout_keeps_and_scales()),
    ("dropout_words", lambda: pins.test_dropout_mask_is_the_generator_words()),
]


def _plant(text, old, new, occurrence):
    assert old in text, f"mutation site not found: {old!r}"
    if occurrence == 0:
        return text.replace(old, new)
    parts = text.split(old)
    assert len(parts) > occurrence
    return old.join(parts[:occurrence]) + new + old.join(parts[occurrence:])


@pytest.mark.parametrize("name,old,new,occ", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_planted_mistake(tmp_path, monkeypatch, name, old, new, occ):
    text = open(SRC).read()
    src = tmp_path / "mutant.c"
    src.write_text(_plant(text, old, new, occ))
    hdr = os.path.join(os.path.dirname(SRC), "msda_oracle.h")
    so = tmp_path / "libmutant.so"
    subprocess.run(["gcc", "-O1", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off",
                    "-I", os.path.dirname(hdr), "-o", str(so), str(src), "-lm"], check=True)
    good = oracle.lib()
    mutant = ctypes.CDLL(str(so))
    for fname in ("oracle_softmax", "oracle_msda_forward", "oracle_msda_forward_fused",
                  "oracle_fused_locations", "oracle_msda_backward", "oracle_sca_compact",
                  "oracle_sca_forward", "oracle_sca_backward", "oracle_linear",
                  "oracle_sca_backward_inputs", "oracle_tsa_reference_points",
                  "oracle_tsa_forward", "oracle_dropout", "oracle_philox4x32_10",
                  "oracle_sca_camera_average"):
        fn = getattr(mutant, fname)
        fn.argtypes = getattr(good, fname).argtypes
        fn.restype = getattr(good, fname).restype
    monkeypatch.setattr(oracle, "_lib", mutant)
    caught = []
    for pin_name, call in PIN_CALLS:
        try:
            call()
        except (AssertionError, ValueError):
            caught.append(pin_name)
            break
    assert caught, f"no pin fails for the planted mistake '{name}'"
