"""NumPy front end of the C oracle (``msda_oracle.c``).

TEST INFRASTRUCTURE ONLY: the test suite, the smoke check and the benchmark's
CPU-baseline leg may import this package; the library itself never does.

Every function takes NumPy arrays (any float dtype is widened exactly to
float64), returns float64 results and follows the layouts documented in
``msda_oracle.h``.  ``coord_f32=True`` takes the corner decision in binary32,
as the CUDA kernels do; ``False`` takes it in double (finite differences).
"""
import ctypes
import os

import numpy as np

from . import build as _build

_lib = None

_D = ctypes.POINTER(ctypes.c_double)
_I64 = ctypes.POINTER(ctypes.c_int64)
_I32 = ctypes.POINTER(ctypes.c_int32)
_U8 = ctypes.POINTER(ctypes.c_uint8)
_i = ctypes.c_int


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        L.oracle_softmax.argtypes = [_D, ctypes.c_int64, _i, _D]
        L.oracle_msda_forward.argtypes = [_D, _i, _i, _i, _i, _i, _I64, _I64, _i, _i, _D, _D, _i, _D]
        L.oracle_msda_forward_fused.argtypes = [_D, _i, _i, _i, _i, _i, _I64, _I64, _i, _i, _i,
                                                _D, _D, _D, _i, _D]
        L.oracle_fused_locations.argtypes = [_i, _i, _i, _I64, _i, _i, _i, _D, _D, _D, _i, _D, _D]
        L.oracle_msda_backward.argtypes = [_D, _i, _i, _i, _i, _i, _I64, _I64, _i, _i, _D, _D, _D,
                                           _i, _D, _D, _D]
        L.oracle_sca_compact.argtypes = [_U8, _i, _i, _i, _i, _I32, _I32, _I32, _I32]
        L.oracle_sca_forward.argtypes = [_D, _i, _i, _i, _i, _i, _i, _I64, _I64, _i, _i, _i, _D,
                                         _U8, _D, _D, _i, _D, _D]
        L.oracle_sca_backward.argtypes = [_D, _i, _i, _i, _i, _i, _i, _I64, _I64, _i, _i, _i, _D,
                                          _U8, _D, _D, _D, _i, _D, _D, _D]
        L.oracle_linear.argtypes = [_D, _D, _D, _D, _i, _i, _i, _D]
        L.oracle_sca_camera_average.argtypes = [_D, _I32, _I32, _i, _i, _i, ctypes.c_int64, _D]
        L.oracle_sca_backward_inputs.argtypes = [_i, _i, _i, _i, _i, _I64, _i, _i, _U8, _D, _D,
                                                 _D, _D, _D, _D]
        L.oracle_tsa_reference_points.argtypes = [_i, _i, _i, _i, ctypes.c_double,
                                                  ctypes.c_double, _D, _D]
        L.oracle_tsa_forward.argtypes = [_D, _i, _i, _i, _i, _i, _i, _I64, _I64, _i, _i, _i, _D,
                                         _D, _D, _i, _D]
        _U32 = ctypes.POINTER(ctypes.c_uint32)
        L.oracle_philox4x32_10.argtypes = [_U32, _U32, _U32]
        L.oracle_philox4x32_10.restype = None
        L.oracle_dropout.argtypes = [_D, ctypes.c_int64, ctypes.c_double, ctypes.c_uint64, _D]
        for f in ("oracle_softmax", "oracle_msda_forward", "oracle_msda_forward_fused",
                  "oracle_fused_locations", "oracle_msda_backward", "oracle_sca_compact",
                  "oracle_sca_forward", "oracle_sca_backward", "oracle_linear",
                  "oracle_sca_camera_average",
                  "oracle_sca_backward_inputs", "oracle_tsa_reference_points",
                  "oracle_tsa_forward", "oracle_dropout"):
            getattr(L, f).restype = ctypes.c_int
        _lib = L
    return _lib


def _d(a):
    return np.ascontiguousarray(a, dtype=np.float64)


def _p(a, t):
    return a.ctypes.data_as(t)


def _levels(spatial_shapes, level_start_index):
    shapes = np.ascontiguousarray(spatial_shapes, dtype=np.int64).reshape(-1, 2)
    if level_start_index is None:
        sizes = shapes[:, 0] * shapes[:, 1]
        level_start_index = np.concatenate([[0], np.cumsum(sizes)[:-1]])
    starts = np.ascontiguousarray(level_start_index, dtype=np.int64).reshape(-1)
    return shapes, starts


def _check(rc, name):
    if rc != 0:
        raise ValueError(f"{name}: invalid arguments")


def softmax(logits, axis_len):
    a = _d(logits)
    out = np.empty_like(a)
    _check(lib().oracle_softmax(_p(a, _D), a.size // axis_len, axis_len, _p(out, _D)), "softmax")
    return out


def msda_forward(value, spatial_shapes, level_start_index, sampling_locations,
                 attention_weights, coord_f32=True):
    """value [B, Nv, H, Dh]; locations [B, Nq, H, L, P, 2]; weights [B, Nq, H, L, P]
    -> out [B, Nq, H*Dh]."""
    v, loc, w = _d(value), _d(sampling_locations), _d(attention_weights)
    shapes, starts = _levels(spatial_shapes, level_start_index)
    B, Nv, H, Dh = v.shape
    _, Nq, _, L, P, _ = loc.shape
    out = np.empty((B, Nq, H * Dh))
    rc = lib().oracle_msda_forward(_p(v, _D), B, Nv, H, Dh, L, _p(shapes, _I64), _p(starts, _I64),
                                   Nq, P, _p(loc, _D), _p(w, _D), int(coord_f32), _p(out, _D))
    _check(rc, "msda_forward")
    return out


def fused_locations(spatial_shapes, reference_points, sampling_offsets, attention_logits,
                    coord_f32=True):
    """-> (sampling_locations [B, Nq, H, L, P, 2], attention_weights [B, Nq, H, L, P])."""
    shapes, _ = _levels(spatial_shapes, None)
    ref, off, lg = _d(reference_points), _d(sampling_offsets), _d(attention_logits)
    B, Nq, H, L, P, _ = off.shape
    R = ref.shape[2]
    loc = np.empty(off.shape)
    w = np.empty(lg.shape)
    rc = lib().oracle_fused_locations(B, H, L, _p(shapes, _I64), Nq, P, R, _p(ref, _D),
                                      _p(off, _D), _p(lg, _D), int(coord_f32), _p(loc, _D),
                                      _p(w, _D))
    _check(rc, "fused_locations")
    return loc, w


def msda_forward_fused(value, spatial_shapes, level_start_index, reference_points,
                       sampling_offsets, attention_logits, coord_f32=True):
    """ref [B, Nq, R, 2]; offsets [B, Nq, H, L, P, 2] (level pixels);
    logits [B, Nq, H, L, P] -> out [B, Nq, H*Dh]."""
    v = _d(value)
    shapes, starts = _levels(spatial_shapes, level_start_index)
    ref, off, lg = _d(reference_points), _d(sampling_offsets), _d(attention_logits)
    B, Nv, H, Dh = v.shape
    _, Nq, _, L, P, _ = off.shape
    R = ref.shape[2]
    out = np.empty((B, Nq, H * Dh))
    rc = lib().oracle_msda_forward_fused(_p(v, _D), B, Nv, H, Dh, L, _p(shapes, _I64),
                                         _p(starts, _I64), Nq, P, R, _p(ref, _D), _p(off, _D),
                                         _p(lg, _D), int(coord_f32), _p(out, _D))
    _check(rc, "msda_forward_fused")
    return out


def msda_backward(value, spatial_shapes, level_start_index, sampling_locations,
                  attention_weights, grad_out, coord_f32=True):
    """-> (grad_value [B, Nv, H, Dh], grad_locations, grad_weights)."""
    v, loc, w, go = _d(value), _d(sampling_locations), _d(attention_weights), _d(grad_out)
    shapes, starts = _levels(spatial_shapes, level_start_index)
    B, Nv, H, Dh = v.shape
    _, Nq, _, L, P, _ = loc.shape
    gv = np.empty(v.shape)
    gl = np.empty(loc.shape)
    gw = np.empty(w.shape)
    rc = lib().oracle_msda_backward(_p(v, _D), B, Nv, H, Dh, L, _p(shapes, _I64), _p(starts, _I64),
                                    Nq, P, _p(loc, _D), _p(w, _D), _p(go, _D), int(coord_f32),
                                    _p(gv, _D), _p(gl, _D), _p(gw, _D))
    _check(rc, "msda_backward")
    return gv, gl, gw


def sca_compact(bev_mask):
    """bev_mask [Ncam, B, Nq, R] -> (idx [B, Ncam, Nq], count [B, Ncam],
    pos [B, Ncam, Nq], hits [B, Nq]), all int32."""
    m = np.ascontiguousarray(bev_mask).astype(np.uint8)
    Ncam, B, Nq, R = m.shape
    idx = np.empty((B, Ncam, Nq), np.int32)
    cnt = np.empty((B, Ncam), np.int32)
    pos = np.empty((B, Ncam, Nq), np.int32)
    hits = np.empty((B, Nq), np.int32)
    rc = lib().oracle_sca_compact(_p(m, _U8), Ncam, B, Nq, R, _p(idx, _I32), _p(cnt, _I32),
                                  _p(pos, _I32), _p(hits, _I32))
    _check(rc, "sca_compact")
    return idx, cnt, pos, hits


def sca_forward(value, spatial_shapes, level_start_index, reference_points_cam, bev_mask,
                sampling_offsets, attention_logits, coord_f32=True, return_rebatched=False):
    """value [B, Ncam, Nv, H, Dh]; ref [Ncam, B, Nq, R, 2]; mask [Ncam, B, Nq, R];
    offsets [B, Nq, H, L, P, 2]; logits [B, Nq, H, L, P] -> out [B, Nq, H*Dh]
    (and the rebatched rows [B, Ncam, Nq, H*Dh] when asked)."""
    v = _d(value)
    shapes, starts = _levels(spatial_shapes, level_start_index)
    ref, off, lg = _d(reference_points_cam), _d(sampling_offsets), _d(attention_logits)
    m = np.ascontiguousarray(bev_mask).astype(np.uint8)
    B, Ncam, Nv, H, Dh = v.shape
    _, Nq, _, L, P, _ = off.shape
    R = ref.shape[3]
    out = np.empty((B, Nq, H * Dh))
    rb = np.empty((B, Ncam, Nq, H * Dh)) if return_rebatched else None
    rc = lib().oracle_sca_forward(_p(v, _D), B, Ncam, Nv, H, Dh, L, _p(shapes, _I64),
                                  _p(starts, _I64), Nq, P, R, _p(ref, _D), _p(m, _U8), _p(off, _D),
                                  _p(lg, _D), int(coord_f32), _p(out, _D),
                                  _p(rb, _D) if rb is not None else None)
    _check(rc, "sca_forward")
    return (out, rb) if return_rebatched else out


def sca_camera_average(out_rb, pos, hits):
    """out_rb [B, Ncam, Nq, HD], pos [B, Ncam, Nq], hits [B, Nq] (int32, as
    sca_compact gives them) -> out [B, Nq, HD]: the seeing cameras' rows
    summed in ascending camera order, divided by max(1, hits)."""
    rb = _d(out_rb)
    B, Ncam, Nq, HD = rb.shape
    p = np.ascontiguousarray(pos, dtype=np.int32)
    h = np.ascontiguousarray(hits, dtype=np.int32)
    out = np.empty((B, Nq, HD))
    rc = lib().oracle_sca_camera_average(_p(rb, _D), _p(p, _I32), _p(h, _I32), B, Ncam, Nq, HD,
                                         _p(out, _D))
    _check(rc, "sca_camera_average")
    return out


def sca_backward(value, spatial_shapes, level_start_index, reference_points_cam, bev_mask,
                 sampling_offsets, attention_logits, grad_out, coord_f32=True):
    """-> (grad_value [B, Ncam, Nv, H, Dh], grad_loc_rb [B, Ncam, Nq, H, L, P, 2],
    grad_attn_rb [B, Ncam, Nq, H, L, P])."""
    v = _d(value)
    shapes, starts = _levels(spatial_shapes, level_start_index)
    ref, off, lg = _d(reference_points_cam), _d(sampling_offsets), _d(attention_logits)
    go = _d(grad_out)
    m = np.ascontiguousarray(bev_mask).astype(np.uint8)
    B, Ncam, Nv, H, Dh = v.shape
    _, Nq, _, L, P, _ = off.shape
    R = ref.shape[3]
    gv = np.empty(v.shape)
    gl = np.empty((B, Ncam, Nq, H, L, P, 2))
    gw = np.empty((B, Ncam, Nq, H, L, P))
    rc = lib().oracle_sca_backward(_p(v, _D), B, Ncam, Nv, H, Dh, L, _p(shapes, _I64),
                                   _p(starts, _I64), Nq, P, R, _p(ref, _D), _p(m, _U8),
                                   _p(off, _D), _p(lg, _D), _p(go, _D), int(coord_f32),
                                   _p(gv, _D), _p(gl, _D), _p(gw, _D))
    _check(rc, "sca_backward")
    return gv, gl, gw


def linear(x, w, bias=None, residual=None):
    """y = x w^T (+ bias) (+ residual); x [M, K], w [N, K] -> y [M, N]."""
    xd, wd = _d(x), _d(w)
    M, K = xd.shape
    N = wd.shape[0]
    b = _d(bias) if bias is not None else None
    r = _d(residual) if residual is not None else None
    y = np.empty((M, N))
    rc = lib().oracle_linear(_p(xd, _D), _p(wd, _D), _p(b, _D) if b is not None else None,
                             _p(r, _D) if r is not None else None, M, N, K, _p(y, _D))
    _check(rc, "linear")
    return y


def round_bf16(a):
    """Round to the nearest bfloat16 (ties to even), returned as float64: the
    storage step of the module's bf16 operands."""
    f = np.ascontiguousarray(a, dtype=np.float32)
    u = f.view(np.uint32)
    u = ((u + ((u >> 16) & 1) + np.uint32(0x7FFF)) >> 16) << 16
    return u.astype(np.uint32).view(np.float32).astype(np.float64)


def sca_module_forward(query, query_pos, features, w_value, b_value, w_offsets, b_offsets,
                       w_weights, b_weights, w_output, b_output, reference_points_cam, bev_mask,
                       spatial_shapes, level_start_index, num_levels, num_points,
                       value_bf16=False, dropout_p=0.0, dropout_seed=0, camera_embeds=None,
                       level_embeds=None):
    """The SCA module forward ([BQ] 3, 4, 10-13), composed of the oracle's
    projection and SCA: F~ = F + e_cam + e_level ([BQ] 3; the embeddings are
    optional, absent = already in F); q~ = bf16(q + pos); V = F~ W_v^T + b_v;
    Delta, a from q~; g = SCA; q_hat = q + dropout(bf16(g) W_o^T + b_o).
    features [B, Ncam, Nv, C]; camera_embeds [Ncam, C]; level_embeds [L, C]
    (added to the rows of level l: start_l .. start_l + H_l W_l - 1);
    dropout_p = 0 is the inference identity."""
    q = _d(query)
    B, Nq, C = q.shape
    _, Ncam, Nv, _ = features.shape
    H, L, P = C // 32, num_levels, num_points
    qt = round_bf16(q + (0.0 if query_pos is None else _d(query_pos))).reshape(B * Nq, C)
    F = _d(features).copy()
    if camera_embeds is not None:
        F += _d(camera_embeds)[None, :, None, :]
    if level_embeds is not None:
        shapes, starts = _levels(spatial_shapes, level_start_index)
        e = _d(level_embeds)
        for l in range(L):
            n = int(shapes[l, 0] * shapes[l, 1])
            F[:, :, starts[l]:starts[l] + n, :] += e[l]
    V = linear(F.reshape(-1, C), w_value, b_value)
    if value_bf16:
        V = round_bf16(V)
    off = linear(qt, w_offsets, b_offsets).reshape(B, Nq, H, L, P, 2)
    lg = linear(qt, w_weights, b_weights).reshape(B, Nq, H, L, P)
    g = sca_forward(V.reshape(B, Ncam, Nv, H, 32), spatial_shapes, level_start_index,
                    reference_points_cam, bev_mask, off, lg)
    o = linear(round_bf16(g).reshape(B * Nq, C), w_output, b_output)
    y = q.reshape(B * Nq, C) + (dropout(o, dropout_p, dropout_seed) if dropout_p > 0 else o)
    return y.reshape(B, Nq, C)


def sca_backward_inputs(spatial_shapes, bev_mask, attention_logits, grad_loc_rb, grad_attn_rb):
    """-> (grad_sampling_offsets [B, Nq, H, L, P, 2], grad_attention_logits
    [B, Nq, H, L, P], grad_reference_points_cam [Ncam, B, Nq, R, 2])."""
    shapes, _ = _levels(spatial_shapes, None)
    m = np.ascontiguousarray(bev_mask).astype(np.uint8)
    Ncam, B, Nq, R = m.shape
    lg, gl, gw = _d(attention_logits), _d(grad_loc_rb), _d(grad_attn_rb)
    _, _, H, L, P = lg.shape
    g_off = np.empty((B, Nq, H, L, P, 2))
    g_lg = np.empty((B, Nq, H, L, P))
    g_ref = np.empty((Ncam, B, Nq, R, 2))
    rc = lib().oracle_sca_backward_inputs(B, Ncam, Nq, H, L, _p(shapes, _I64), P, R, _p(m, _U8),
                                          _p(lg, _D), _p(gl, _D), _p(gw, _D), _p(g_off, _D),
                                          _p(g_lg, _D), _p(g_ref, _D))
    _check(rc, "sca_backward_inputs")
    return g_off, g_lg, g_ref


def tsa_reference_points(bev_h, bev_w, ego_motion, grid_length=(0.512, 0.512)):
    """ego_motion [B, T, 3] = (dx m, dy m, angle degrees) of each queue;
    grid_length = (gy, gx) metres per cell -> ref [B, T, bev_h * bev_w, 2]."""
    e = _d(ego_motion)
    B, T, _ = e.shape
    gy, gx = grid_length
    ref = np.empty((B, T, bev_h * bev_w, 2))
    rc = lib().oracle_tsa_reference_points(B, T, bev_h, bev_w, float(gx), float(gy), _p(e, _D),
                                           _p(ref, _D))
    _check(rc, "tsa_reference_points")
    return ref


def tsa_forward(value, spatial_shapes, level_start_index, reference_points, sampling_offsets,
                attention_logits, num_queues, coord_f32=True):
    """value [B*T, Nv, H, Dh] (row b*T + t); ref [B*T, Nq, R, 2];
    offsets [B*T, Nq, H, L, P, 2]; logits [B*T, Nq, H, L, P] -> out [B, Nq, H*Dh],
    the mean over the T queues."""
    v = _d(value)
    shapes, starts = _levels(spatial_shapes, level_start_index)
    ref, off, lg = _d(reference_points), _d(sampling_offsets), _d(attention_logits)
    BT, Nv, H, Dh = v.shape
    T = int(num_queues)
    if T < 1 or BT % T:
        raise ValueError("tsa_forward: batch is not a multiple of num_queues")
    _, Nq, _, L, P, _ = off.shape
    R = ref.shape[2]
    out = np.empty((BT // T, Nq, H * Dh))
    rc = lib().oracle_tsa_forward(_p(v, _D), BT // T, T, Nv, H, Dh, L, _p(shapes, _I64),
                                  _p(starts, _I64), Nq, P, R, _p(ref, _D), _p(off, _D),
                                  _p(lg, _D), int(coord_f32), _p(out, _D))
    _check(rc, "tsa_forward")
    return out


def philox4x32_10(counter, key):
    """The four 32-bit output words of Philox4x32-10 (Salmon et al., SC 2011)."""
    c = np.ascontiguousarray(counter, dtype=np.uint32)
    k = np.ascontiguousarray(key, dtype=np.uint32)
    out = np.empty(4, dtype=np.uint32)
    u32 = ctypes.POINTER(ctypes.c_uint32)
    lib().oracle_philox4x32_10(_p(c, u32), _p(k, u32), _p(out, u32))
    return out


def dropout(o, p, seed):
    """Training-time dropout of o (any shape, row-major element order)."""
    a = _d(o)
    out = np.empty_like(a)
    _check(lib().oracle_dropout(_p(a, _D), a.size, float(p), int(seed), _p(out, _D)), "dropout")
    return out


def tsa_backward(value, spatial_shapes, level_start_index, reference_points, sampling_offsets,
                 attention_logits, num_queues, grad_out, coord_f32=True):
    """Derivative of tsa_forward (the pages give no backward): queue t of
    sample b receives grad_out[b] / T; the fused MSDA backward of every queue
    gives the location and weight gradients, and the chain through the
    location and the softmax (oracle_sca_backward_inputs with one camera that
    sees every query) gives those of the offsets, logits and reference points.
    -> (grad_value [B*T, Nv, H, Dh], grad_offsets [B*T, Nq, H, L, P, 2],
        grad_logits [B*T, Nq, H, L, P], grad_reference_points [B*T, Nq, R, 2])."""
    T = int(num_queues)
    v, ref, off, lg = _d(value), _d(reference_points), _d(sampling_offsets), _d(attention_logits)
    BT, Nq, R = ref.shape[0], ref.shape[1], ref.shape[2]
    loc, w = fused_locations(spatial_shapes, ref, off, lg, coord_f32)
    go = np.repeat(_d(grad_out) / T, T, axis=0)
    gv, gl, gw = msda_backward(v, spatial_shapes, level_start_index, loc, w, go, coord_f32)
    seen = np.ones((1, BT, Nq, R), np.uint8)
    g_off, g_lg, g_ref = sca_backward_inputs(spatial_shapes, seen, lg, gl[:, None], gw[:, None])
    return gv, g_off, g_lg, g_ref[0]
