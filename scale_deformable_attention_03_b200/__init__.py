"""B200-native multi-scale deformable attention (MSDA) and BEVFormer Spatial
Cross-Attention (SCA).

The compute lives in ``libmsda.so`` (hand-written sm_100a CUDA kernels behind
the C ABI of ``include/msda.h``).  This module only marshals arguments: it
reads shapes and device pointers from torch tensors, allocates outputs with
torch, passes the current CUDA stream and raises ``MsdaError`` on a non-zero
status.  There is no fallback: without the built library every call raises.

Functions (same names as the C ABI): ``msda_forward``, ``msda_forward_fused``,
``msda_backward``, ``sca_compact``, ``sca_rebatched_forward``,
``sca_camera_average``, ``sca_camera_average_linear``, ``sca_forward``,
``sca_forward_query_major``, ``sca_rebatched_backward``, ``sca_backward``
and ``msda_backward`` (``deterministic=True``: the fixed-point variants),
``sca_backward_full``,
``sca_backward_inputs``, ``tsa_reference_points``, ``tsa_forward``,
``tsa_backward``, ``msda_linear`` (with dropout), ``sca_module_forward``,
``msda_workspace_size``, ``sca_compact_workspace_size``; the remaining C
entry points (workspace sizes, status strings, the no-alloc compaction, the
GEMM's timeout counter and test switch) are reached through ``lib()``.
"""
import ctypes
import os

import numpy as np

HEAD_DIM = 32
_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmsda.so")

MSDA_F32, MSDA_BF16 = 0, 1


class MsdaError(RuntimeError):
    pass


class Dims(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in ("B", "Ncam", "Nq", "Nv", "H", "L", "P", "R")]


_vp = ctypes.c_void_p


class ScaModuleParams(ctypes.Structure):
    _fields_ = [("query", _vp), ("query_pos", _vp), ("features", _vp), ("w_value", _vp),
                ("b_value", _vp), ("w_offsets", _vp), ("b_offsets", _vp), ("w_weights", _vp),
                ("b_weights", _vp), ("w_output", _vp), ("b_output", _vp),
                ("reference_points_cam", _vp), ("bev_mask", _vp), ("value_dtype", ctypes.c_int),
                ("dropout_p", ctypes.c_float), ("dropout_seed", ctypes.c_uint64),
                ("camera_embeds", _vp), ("level_embeds", _vp)]


_lib = None
_i64p = ctypes.POINTER(ctypes.c_int64)


def lib():
    """The loaded libmsda.so (raises MsdaError when it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise MsdaError(f"{LIB_PATH} is missing: build it with "
                            "`python -m scale_deformable_attention_03_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        st = ctypes.c_int
        L.msda_forward.argtypes = [_vp, st, _i64p, _i64p, _vp, _vp, Dims, _vp, _vp]
        L.msda_forward_fused.argtypes = [_vp, st, _i64p, _i64p, _vp, _vp, _vp, Dims, _vp, _vp]
        L.msda_backward.argtypes = [_vp, st, _i64p, _i64p, _vp, _vp, _vp, Dims, _vp, _vp, _vp, _vp]
        L.msda_backward_deterministic.argtypes = [_vp, st, _i64p, _i64p, _vp, _vp, _vp, Dims,
                                                  _vp, ctypes.c_size_t, _vp, _vp, _vp, _vp]
        L.msda_backward_deterministic.restype = ctypes.c_int
        L.msda_backward_deterministic_workspace_size.argtypes = [Dims]
        L.msda_backward_deterministic_workspace_size.restype = ctypes.c_size_t
        L.sca_backward_deterministic.argtypes = [_vp, st, _i64p, _i64p, _vp, _vp, _vp, _vp, _vp,
                                                 Dims, _vp, ctypes.c_size_t, _vp, _vp, _vp, _vp]
        L.sca_backward_deterministic.restype = ctypes.c_int
        L.sca_backward_deterministic_workspace_size.argtypes = [Dims]
        L.sca_backward_deterministic_workspace_size.restype = ctypes.c_size_t
        L.msda_workspace_size.argtypes = [Dims]
        L.msda_workspace_size.restype = ctypes.c_size_t
        L.sca_compact_workspace_size.argtypes = [Dims]
        L.sca_compact_workspace_size.restype = ctypes.c_size_t
        L.sca_compact.argtypes = [_vp, Dims, _vp, ctypes.c_size_t, _vp, _vp, _vp, _vp, _vp]
        L.sca_forward.argtypes = [_vp, st, _i64p, _i64p, _vp, _vp, _vp, _vp, Dims, _vp,
                                  ctypes.c_size_t, _vp, _vp]
        L.sca_backward.argtypes = [_vp, st, _i64p, _i64p, _vp, _vp, _vp, _vp, _vp, Dims, _vp,
                                   ctypes.c_size_t, _vp, _vp, _vp, _vp]
        L.sca_rebatched_forward.argtypes = [_vp, st, _i64p, _i64p, _vp, _vp, _vp, _vp, _vp, Dims,
                                            _vp, _vp]
        L.sca_camera_average.argtypes = [_vp, _vp, _vp, Dims, _vp, _vp]
        L.sca_rebatched_backward.argtypes = [_vp, st, _i64p, _i64p, _vp, _vp, _vp, _vp, _vp, _vp,
                                             _vp, Dims, _vp, _vp, _vp, _vp]
        for f in ("msda_forward", "msda_forward_fused", "msda_backward", "sca_compact",
                  "sca_forward", "sca_backward", "sca_rebatched_forward", "sca_camera_average",
                  "sca_rebatched_backward"):
            getattr(L, f).restype = ctypes.c_int
        L.msda_linear.argtypes = [_vp, _vp, _vp, _vp, ctypes.c_int32, ctypes.c_int32,
                                  ctypes.c_int32, st, _vp, _vp]
        L.msda_linear.restype = ctypes.c_int
        L.msda_linear_dropout.argtypes = [_vp, _vp, _vp, _vp, ctypes.c_int32, ctypes.c_int32,
                                          ctypes.c_int32, st, _vp, ctypes.c_float,
                                          ctypes.c_uint64, _vp]
        L.msda_linear_dropout.restype = ctypes.c_int
        L.sca_camera_average_linear.argtypes = [_vp, _vp, _vp, Dims, _vp, _vp, _vp,
                                                ctypes.c_int32, st, _vp, ctypes.c_float,
                                                ctypes.c_uint64, _vp]
        L.sca_camera_average_linear.restype = ctypes.c_int
        L.msda_linear_timeouts.restype = ctypes.c_uint32
        L.msda_linear_test_withhold_load.restype = ctypes.c_int
        L.sca_module_workspace_size.argtypes = [Dims, ctypes.c_int]
        L.sca_module_workspace_size.restype = ctypes.c_size_t
        L.sca_module_forward.argtypes = [ctypes.POINTER(ScaModuleParams), _i64p, _i64p, Dims, _vp,
                                         ctypes.c_size_t, _vp, _vp]
        L.sca_module_forward.restype = ctypes.c_int
        L.sca_backward_inputs.argtypes = [_i64p, _i64p, _vp, _vp, _vp, _vp, Dims, _vp, _vp, _vp,
                                          _vp]
        L.sca_backward_inputs.restype = ctypes.c_int
        L.sca_backward_full_workspace_size.argtypes = [Dims]
        L.sca_backward_full_workspace_size.restype = ctypes.c_size_t
        L.sca_backward_full.argtypes = [_vp, st, _i64p, _i64p, _vp, _vp, _vp, _vp, _vp, Dims,
                                        _vp, ctypes.c_size_t, _vp, _vp, _vp, _vp, _vp]
        L.sca_backward_full.restype = ctypes.c_int
        i32, f64 = ctypes.c_int32, ctypes.c_double
        L.tsa_reference_points.argtypes = [_vp, i32, i32, i32, i32, f64, f64, _vp, _vp]
        L.tsa_reference_points.restype = ctypes.c_int
        L.tsa_forward.argtypes = [_vp, st, _i64p, _i64p, _vp, _vp, _vp, i32, Dims, _vp, _vp]
        L.tsa_forward.restype = ctypes.c_int
        L.tsa_backward_workspace_size.argtypes = [Dims, i32]
        L.tsa_backward_workspace_size.restype = ctypes.c_size_t
        L.tsa_backward.argtypes = [_vp, st, _i64p, _i64p, _vp, _vp, _vp, i32, _vp, Dims, _vp,
                                   ctypes.c_size_t, _vp, _vp, _vp, _vp, _vp]
        L.tsa_backward.restype = ctypes.c_int
        L.sca_forward_query_major.argtypes = [_vp, st, _i64p, _i64p, _vp, _vp, _vp, _vp, Dims,
                                              _vp, _vp]
        L.sca_forward_query_major.restype = ctypes.c_int
        L.msda_status_string.argtypes = [ctypes.c_int]
        L.msda_status_string.restype = ctypes.c_char_p
        L.msda_last_error.restype = ctypes.c_char_p
        L.msda_version.restype = ctypes.c_int32
        _lib = L
    return _lib


def _check(status, name):
    if status != 0:
        L = lib()
        raise MsdaError(f"{name}: {L.msda_status_string(status).decode()}: "
                        f"{L.msda_last_error().decode()}")


def _torch():
    import torch
    return torch


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    torch = _torch()
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _levels(spatial_shapes, level_start_index):
    """Host int64 copies of the level tables (kept alive by the caller)."""
    torch = _torch()

    def host(a):
        if isinstance(a, torch.Tensor):
            a = a.detach().cpu().numpy()
        return np.ascontiguousarray(np.asarray(a, dtype=np.int64))
    shapes = host(spatial_shapes).reshape(-1, 2)
    if level_start_index is None:
        sizes = shapes[:, 0] * shapes[:, 1]
        level_start_index = np.concatenate([[0], np.cumsum(sizes)[:-1]])
    starts = host(level_start_index).reshape(-1)
    return shapes, starts


def _vdt(value):
    torch = _torch()
    if value.dtype == torch.float32:
        return MSDA_F32
    if value.dtype == torch.bfloat16:
        return MSDA_BF16
    raise MsdaError(f"value dtype {value.dtype} is not float32 or bfloat16")


def _contig(*ts):
    for t in ts:
        if t is not None and not t.is_contiguous():
            raise MsdaError("tensors must be contiguous")


def msda_forward(value, spatial_shapes, level_start_index, sampling_locations,
                 attention_weights, out=None, stream=None):
    """value [B, Nv, H, 32] (f32/bf16); locations [B, Nq, H, L, P, 2];
    weights [B, Nq, H, L, P] -> out [B, Nq, H*32] fp32."""
    torch = _torch()
    _contig(value, sampling_locations, attention_weights, out)
    B, Nv, H, _ = value.shape
    _, Nq, _, L, P, _ = sampling_locations.shape
    shapes, starts = _levels(spatial_shapes, level_start_index)
    if out is None:
        out = torch.empty((B, Nq, H * HEAD_DIM), device=value.device, dtype=torch.float32)
    d = Dims(B, 1, Nq, Nv, H, L, P, 1)
    _check(lib().msda_forward(_ptr(value), _vdt(value), shapes.ctypes.data_as(_i64p),
                              starts.ctypes.data_as(_i64p), _ptr(sampling_locations),
                              _ptr(attention_weights), d, _ptr(out), _stream(stream)),
           "msda_forward")
    return out


def msda_forward_fused(value, spatial_shapes, level_start_index, reference_points,
                       sampling_offsets, attention_logits, out=None, stream=None):
    """reference_points [B, Nq, R, 2]; offsets [B, Nq, H, L, P, 2] (level
    pixels); logits [B, Nq, H, L, P] -> out [B, Nq, H*32] fp32."""
    torch = _torch()
    _contig(value, reference_points, sampling_offsets, attention_logits, out)
    B, Nv, H, _ = value.shape
    _, Nq, _, L, P, _ = sampling_offsets.shape
    R = reference_points.shape[2]
    shapes, starts = _levels(spatial_shapes, level_start_index)
    if out is None:
        out = torch.empty((B, Nq, H * HEAD_DIM), device=value.device, dtype=torch.float32)
    d = Dims(B, 1, Nq, Nv, H, L, P, R)
    _check(lib().msda_forward_fused(_ptr(value), _vdt(value), shapes.ctypes.data_as(_i64p),
                                    starts.ctypes.data_as(_i64p), _ptr(reference_points),
                                    _ptr(sampling_offsets), _ptr(attention_logits), d, _ptr(out),
                                    _stream(stream)),
           "msda_forward_fused")
    return out


def tsa_reference_points(ego_motion, bev_h, bev_w, grid_length=(0.512, 0.512), out=None,
                         stream=None):
    """ego_motion [B, T, 3] fp32 (dx m, dy m, yaw degrees) on the device ->
    reference points [B, T, bev_h * bev_w, 2] fp32; grid_length = (gy, gx)."""
    torch = _torch()
    _contig(ego_motion, out)
    B, T, _ = ego_motion.shape
    if out is None:
        out = torch.empty((B, T, bev_h * bev_w, 2), device=ego_motion.device,
                          dtype=torch.float32)
    gy, gx = grid_length
    _check(lib().tsa_reference_points(_ptr(ego_motion), B, T, bev_h, bev_w, float(gy), float(gx),
                                      _ptr(out), _stream(stream)),
           "tsa_reference_points")
    return out


def tsa_forward(value, spatial_shapes, level_start_index, reference_points, sampling_offsets,
                attention_logits, num_queues, out=None, stream=None):
    """value [B*T, Nv, H, 32] (item b*T + t = queue t of sample b);
    reference_points [B*T, Nq, R, 2]; offsets [B*T, Nq, H, L, P, 2];
    logits [B*T, Nq, H, L, P] -> out [B, Nq, H*32] fp32, the mean over the
    T = num_queues queues of the fused MSDA."""
    torch = _torch()
    _contig(value, reference_points, sampling_offsets, attention_logits, out)
    BT, Nv, H, _ = value.shape
    T = int(num_queues)
    if T < 1 or BT % T:
        raise MsdaError("tsa_forward: the value batch is not a multiple of num_queues")
    _, Nq, _, L, P, _ = sampling_offsets.shape
    R = reference_points.shape[2]
    shapes, starts = _levels(spatial_shapes, level_start_index)
    if out is None:
        out = torch.empty((BT // T, Nq, H * HEAD_DIM), device=value.device, dtype=torch.float32)
    d = Dims(BT // T, 1, Nq, Nv, H, L, P, R)
    _check(lib().tsa_forward(_ptr(value), _vdt(value), shapes.ctypes.data_as(_i64p),
                             starts.ctypes.data_as(_i64p), _ptr(reference_points),
                             _ptr(sampling_offsets), _ptr(attention_logits), T, d, _ptr(out),
                             _stream(stream)),
           "tsa_forward")
    return out


def tsa_backward(value, spatial_shapes, level_start_index, reference_points, sampling_offsets,
                 attention_logits, num_queues, grad_out, workspace=None, stream=None, out=None):
    """-> (grad_value [B*T, Nv, H, 32], grad_sampling_offsets [B*T, Nq, H, L, P, 2],
    grad_attention_logits [B*T, Nq, H, L, P], grad_reference_points [B*T, Nq, R, 2])."""
    torch = _torch()
    _contig(value, reference_points, sampling_offsets, attention_logits, grad_out)
    BT, Nv, H, _ = value.shape
    T = int(num_queues)
    if T < 1 or BT % T:
        raise MsdaError("tsa_backward: the value batch is not a multiple of num_queues")
    _, Nq, _, L, P, _ = sampling_offsets.shape
    R = reference_points.shape[2]
    shapes, starts = _levels(spatial_shapes, level_start_index)
    d = Dims(BT // T, 1, Nq, Nv, H, L, P, R)
    dev = value.device
    if out is not None:
        gv, g_off, g_lg, g_ref = out
        _contig(gv, g_off, g_lg, g_ref)
    else:
        gv = torch.empty(value.shape, device=dev, dtype=torch.float32)
        g_off = torch.empty(sampling_offsets.shape, device=dev, dtype=torch.float32)
        g_lg = torch.empty(attention_logits.shape, device=dev, dtype=torch.float32)
        g_ref = torch.empty(reference_points.shape, device=dev, dtype=torch.float32)
    workspace = _workspace(int(lib().tsa_backward_workspace_size(d, T)), dev, workspace)
    _check(lib().tsa_backward(_ptr(value), _vdt(value), shapes.ctypes.data_as(_i64p),
                              starts.ctypes.data_as(_i64p), _ptr(reference_points),
                              _ptr(sampling_offsets), _ptr(attention_logits), T, _ptr(grad_out),
                              d, _ptr(workspace), workspace.numel(), _ptr(gv), _ptr(g_off),
                              _ptr(g_lg), _ptr(g_ref), _stream(stream)),
           "tsa_backward")
    return gv, g_off, g_lg, g_ref


def msda_backward(value, spatial_shapes, level_start_index, sampling_locations,
                  attention_weights, grad_out, grad_value=None, grad_sampling_locations=None,
                  grad_attention_weights=None, stream=None, deterministic=False, workspace=None):
    """-> (grad_value [B, Nv, H, 32] fp32, grad_sampling_locations,
    grad_attention_weights).  deterministic=True accumulates grad_value in
    fixed point (bitwise reproducible; needs a workspace, allocated here when
    not given)."""
    torch = _torch()
    _contig(value, sampling_locations, attention_weights, grad_out)
    B, Nv, H, _ = value.shape
    _, Nq, _, L, P, _ = sampling_locations.shape
    shapes, starts = _levels(spatial_shapes, level_start_index)
    dev = value.device
    if grad_value is None:
        grad_value = torch.empty(value.shape, device=dev, dtype=torch.float32)
    if grad_sampling_locations is None:
        grad_sampling_locations = torch.empty(sampling_locations.shape, device=dev,
                                              dtype=torch.float32)
    if grad_attention_weights is None:
        grad_attention_weights = torch.empty(attention_weights.shape, device=dev,
                                             dtype=torch.float32)
    d = Dims(B, 1, Nq, Nv, H, L, P, 1)
    args = (_ptr(value), _vdt(value), shapes.ctypes.data_as(_i64p), starts.ctypes.data_as(_i64p),
            _ptr(sampling_locations), _ptr(attention_weights), _ptr(grad_out), d)
    outs = (_ptr(grad_value), _ptr(grad_sampling_locations), _ptr(grad_attention_weights),
            _stream(stream))
    if deterministic:
        workspace = _workspace(int(lib().msda_backward_deterministic_workspace_size(d)), dev,
                               workspace)
        _check(lib().msda_backward_deterministic(*args, _ptr(workspace), workspace.numel(),
                                                 *outs), "msda_backward_deterministic")
    else:
        _check(lib().msda_backward(*args, *outs), "msda_backward")
    return grad_value, grad_sampling_locations, grad_attention_weights


def _sca_dims(value, sampling_offsets, reference_points_cam):
    B, Ncam, Nv, H, _ = value.shape
    _, Nq, _, L, P, _ = sampling_offsets.shape
    R = reference_points_cam.shape[3]
    return Dims(B, Ncam, Nq, Nv, H, L, P, R)


def msda_workspace_size(dims):
    return int(lib().msda_workspace_size(dims))


def sca_compact_workspace_size(dims):
    return int(lib().sca_compact_workspace_size(dims))


def _workspace(nbytes, device, workspace):
    torch = _torch()
    if workspace is None:
        workspace = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=device)
    return workspace


def sca_compact(bev_mask, workspace=None, stream=None, out=None):
    """bev_mask [Ncam, B, Nq, R] (uint8 / bool) -> (idx [B, Ncam, Nq],
    count [B, Ncam], pos [B, Ncam, Nq], hits [B, Nq]), int32; `out` may
    supply the four tensors."""
    torch = _torch()
    _contig(bev_mask)
    if bev_mask.dtype == torch.bool:
        bev_mask = bev_mask.view(torch.uint8)
    Ncam, B, Nq, R = bev_mask.shape
    dev = bev_mask.device
    if out is not None:
        idx, count, pos, hits = out
        _contig(idx, count, pos, hits)
    else:
        idx = torch.empty((B, Ncam, Nq), dtype=torch.int32, device=dev)
        count = torch.empty((B, Ncam), dtype=torch.int32, device=dev)
        pos = torch.empty((B, Ncam, Nq), dtype=torch.int32, device=dev)
        hits = torch.empty((B, Nq), dtype=torch.int32, device=dev)
    d = Dims(B, Ncam, Nq, 1, 1, 1, 1, R)
    nbytes = sca_compact_workspace_size(d)
    workspace = _workspace(nbytes, dev, workspace)
    _check(lib().sca_compact(_ptr(bev_mask), d, _ptr(workspace), workspace.numel(), _ptr(idx),
                             _ptr(count), _ptr(pos), _ptr(hits), _stream(stream)),
           "sca_compact")
    return idx, count, pos, hits


def sca_forward(value, spatial_shapes, level_start_index, reference_points_cam, bev_mask,
                sampling_offsets, attention_logits, out=None, workspace=None, stream=None):
    """value [B, Ncam, Nv, H, 32]; reference_points_cam [Ncam, B, Nq, R, 2];
    bev_mask [Ncam, B, Nq, R]; offsets [B, Nq, H, L, P, 2]; logits
    [B, Nq, H, L, P] -> out [B, Nq, H*32] fp32."""
    torch = _torch()
    _contig(value, reference_points_cam, bev_mask, sampling_offsets, attention_logits, out)
    if bev_mask.dtype == torch.bool:
        bev_mask = bev_mask.view(torch.uint8)
    d = _sca_dims(value, sampling_offsets, reference_points_cam)
    shapes, starts = _levels(spatial_shapes, level_start_index)
    if out is None:
        out = torch.empty((d.B, d.Nq, d.H * HEAD_DIM), device=value.device, dtype=torch.float32)
    workspace = _workspace(msda_workspace_size(d), value.device, workspace)
    _check(lib().sca_forward(_ptr(value), _vdt(value), shapes.ctypes.data_as(_i64p),
                             starts.ctypes.data_as(_i64p), _ptr(reference_points_cam),
                             _ptr(bev_mask), _ptr(sampling_offsets), _ptr(attention_logits), d,
                             _ptr(workspace), workspace.numel(), _ptr(out), _stream(stream)),
           "sca_forward")
    return out


def sca_forward_query_major(value, spatial_shapes, level_start_index, reference_points_cam,
                            bev_mask, sampling_offsets, attention_logits, out=None, stream=None):
    """sca_forward's result from one query-major kernel, without workspace."""
    torch = _torch()
    _contig(value, reference_points_cam, bev_mask, sampling_offsets, attention_logits, out)
    if bev_mask.dtype == torch.bool:
        bev_mask = bev_mask.view(torch.uint8)
    d = _sca_dims(value, sampling_offsets, reference_points_cam)
    shapes, starts = _levels(spatial_shapes, level_start_index)
    if out is None:
        out = torch.empty((d.B, d.Nq, d.H * HEAD_DIM), device=value.device, dtype=torch.float32)
    _check(lib().sca_forward_query_major(_ptr(value), _vdt(value), shapes.ctypes.data_as(_i64p),
                                         starts.ctypes.data_as(_i64p), _ptr(reference_points_cam),
                                         _ptr(bev_mask), _ptr(sampling_offsets),
                                         _ptr(attention_logits), d, _ptr(out), _stream(stream)),
           "sca_forward_query_major")
    return out


def sca_backward(value, spatial_shapes, level_start_index, reference_points_cam, bev_mask,
                 sampling_offsets, attention_logits, grad_out, grad_value=None,
                 grad_sampling_locations_rb=None, grad_attention_weights_rb=None,
                 workspace=None, stream=None, deterministic=False):
    """-> (grad_value [B, Ncam, Nv, H, 32], grad_sampling_locations_rb
    [B, Ncam, Nq, H, L, P, 2], grad_attention_weights_rb [B, Ncam, Nq, H, L, P]).
    deterministic=True accumulates grad_value in fixed point (bitwise
    reproducible; the workspace then also holds the fixed-point copy)."""
    torch = _torch()
    _contig(value, reference_points_cam, bev_mask, sampling_offsets, attention_logits, grad_out)
    if bev_mask.dtype == torch.bool:
        bev_mask = bev_mask.view(torch.uint8)
    d = _sca_dims(value, sampling_offsets, reference_points_cam)
    shapes, starts = _levels(spatial_shapes, level_start_index)
    dev = value.device
    if grad_value is None:
        grad_value = torch.empty(value.shape, device=dev, dtype=torch.float32)
    if grad_sampling_locations_rb is None:
        grad_sampling_locations_rb = torch.empty((d.B, d.Ncam, d.Nq, d.H, d.L, d.P, 2),
                                                 device=dev, dtype=torch.float32)
    if grad_attention_weights_rb is None:
        grad_attention_weights_rb = torch.empty((d.B, d.Ncam, d.Nq, d.H, d.L, d.P), device=dev,
                                                dtype=torch.float32)
    fn = lib().sca_backward_deterministic if deterministic else lib().sca_backward
    need = (int(lib().sca_backward_deterministic_workspace_size(d)) if deterministic
            else msda_workspace_size(d))
    workspace = _workspace(need, dev, workspace)
    _check(fn(_ptr(value), _vdt(value), shapes.ctypes.data_as(_i64p),
              starts.ctypes.data_as(_i64p), _ptr(reference_points_cam), _ptr(bev_mask),
              _ptr(sampling_offsets), _ptr(attention_logits), _ptr(grad_out), d, _ptr(workspace),
              workspace.numel(), _ptr(grad_value), _ptr(grad_sampling_locations_rb),
              _ptr(grad_attention_weights_rb), _stream(stream)),
           "sca_backward_deterministic" if deterministic else "sca_backward")
    return grad_value, grad_sampling_locations_rb, grad_attention_weights_rb


def sca_backward_full(value, spatial_shapes, level_start_index, reference_points_cam, bev_mask,
                      sampling_offsets, attention_logits, grad_out, out=None, workspace=None,
                      stream=None):
    """The SCA backward down to its inputs -> (grad_value [B, Ncam, Nv, H, 32],
    grad_sampling_offsets [B, Nq, H, L, P, 2], grad_attention_logits
    [B, Nq, H, L, P], grad_reference_points_cam [Ncam, B, Nq, R, 2]); `out`
    may supply the four tensors."""
    torch = _torch()
    _contig(value, reference_points_cam, bev_mask, sampling_offsets, attention_logits, grad_out)
    if bev_mask.dtype == torch.bool:
        bev_mask = bev_mask.view(torch.uint8)
    d = _sca_dims(value, sampling_offsets, reference_points_cam)
    shapes, starts = _levels(spatial_shapes, level_start_index)
    dev = value.device
    if out is not None:
        gv, g_off, g_lg, g_ref = out
        _contig(gv, g_off, g_lg, g_ref)
    else:
        gv = torch.empty(value.shape, device=dev, dtype=torch.float32)
        g_off = torch.empty(sampling_offsets.shape, device=dev, dtype=torch.float32)
        g_lg = torch.empty(attention_logits.shape, device=dev, dtype=torch.float32)
        g_ref = torch.empty(reference_points_cam.shape, device=dev, dtype=torch.float32)
    workspace = _workspace(int(lib().sca_backward_full_workspace_size(d)), dev, workspace)
    _check(lib().sca_backward_full(_ptr(value), _vdt(value), shapes.ctypes.data_as(_i64p),
                                   starts.ctypes.data_as(_i64p), _ptr(reference_points_cam),
                                   _ptr(bev_mask), _ptr(sampling_offsets), _ptr(attention_logits),
                                   _ptr(grad_out), d, _ptr(workspace), workspace.numel(),
                                   _ptr(gv), _ptr(g_off), _ptr(g_lg), _ptr(g_ref),
                                   _stream(stream)),
           "sca_backward_full")
    return gv, g_off, g_lg, g_ref


def sca_rebatched_forward(value, spatial_shapes, level_start_index, reference_points_cam,
                          sampling_offsets, attention_logits, idx, count, out_rb=None,
                          stream=None):
    """Fused MSDA of every camera's seeing queries (idx, count from
    sca_compact) -> out_rb [B, Ncam, Nq, H*32]; rows >= count untouched."""
    torch = _torch()
    _contig(value, reference_points_cam, sampling_offsets, attention_logits, idx, count, out_rb)
    d = _sca_dims(value, sampling_offsets, reference_points_cam)
    shapes, starts = _levels(spatial_shapes, level_start_index)
    if out_rb is None:
        out_rb = torch.empty((d.B, d.Ncam, d.Nq, d.H * HEAD_DIM), device=value.device,
                             dtype=torch.float32)
    _check(lib().sca_rebatched_forward(_ptr(value), _vdt(value), shapes.ctypes.data_as(_i64p),
                                       starts.ctypes.data_as(_i64p), _ptr(reference_points_cam),
                                       _ptr(sampling_offsets), _ptr(attention_logits), _ptr(idx),
                                       _ptr(count), d, _ptr(out_rb), _stream(stream)),
           "sca_rebatched_forward")
    return out_rb


def sca_camera_average(out_rb, pos, hits, out=None, stream=None):
    """out[b, q] = sum over seeing cameras of out_rb rows / max(1, hits)."""
    torch = _torch()
    _contig(out_rb, pos, hits, out)
    B, Ncam, Nq, C = out_rb.shape
    if out is None:
        out = torch.empty((B, Nq, C), device=out_rb.device, dtype=torch.float32)
    d = Dims(B, Ncam, Nq, 1, C // HEAD_DIM, 1, 1, 1)
    _check(lib().sca_camera_average(_ptr(out_rb), _ptr(pos), _ptr(hits), d, _ptr(out),
                                    _stream(stream)),
           "sca_camera_average")
    return out


def sca_camera_average_linear(out_rb, pos, hits, w, bias=None, residual=None, out=None,
                              out_dtype=None, stream=None, dropout_p=0.0, dropout_seed=0):
    """y = residual + dropout(bf16(camera average of out_rb) w^T + bias), the
    average formed inside the tensor-core projection.  out_rb [B, Ncam, Nq, C]
    fp32; pos, hits from sca_compact; w [N, C] bf16; bias [N] fp32; residual
    [B * Nq, N] fp32 -> y [B * Nq, N] (fp32, or bf16 when out_dtype / out is
    bfloat16)."""
    torch = _torch()
    _contig(out_rb, pos, hits, w, bias, residual, out)
    if w.dtype != torch.bfloat16:
        raise MsdaError("sca_camera_average_linear takes a bfloat16 w")
    B, Ncam, Nq, C = out_rb.shape
    N = w.shape[0]
    if out is None:
        out = torch.empty((B * Nq, N), device=out_rb.device, dtype=out_dtype or torch.float32)
    ydt = MSDA_BF16 if out.dtype == torch.bfloat16 else MSDA_F32
    d = Dims(B, Ncam, Nq, 1, C // HEAD_DIM, 1, 1, 1)
    _check(lib().sca_camera_average_linear(_ptr(out_rb), _ptr(pos), _ptr(hits), d, _ptr(w),
                                           _ptr(bias), _ptr(residual), N, ydt, _ptr(out),
                                           float(dropout_p), int(dropout_seed), _stream(stream)),
           "sca_camera_average_linear")
    return out


def sca_rebatched_backward(value, spatial_shapes, level_start_index, reference_points_cam,
                           sampling_offsets, attention_logits, grad_out, idx, count, hits,
                           grad_value=None, grad_sampling_locations_rb=None,
                           grad_attention_weights_rb=None, stream=None):
    """Backward of sca_rebatched_forward + sca_camera_average on a given
    compaction -> (grad_value, grad_sampling_locations_rb, grad_attention_weights_rb)."""
    torch = _torch()
    _contig(value, reference_points_cam, sampling_offsets, attention_logits, grad_out, idx, count,
            hits)
    d = _sca_dims(value, sampling_offsets, reference_points_cam)
    shapes, starts = _levels(spatial_shapes, level_start_index)
    dev = value.device
    if grad_value is None:
        grad_value = torch.empty(value.shape, device=dev, dtype=torch.float32)
    if grad_sampling_locations_rb is None:
        grad_sampling_locations_rb = torch.empty((d.B, d.Ncam, d.Nq, d.H, d.L, d.P, 2),
                                                 device=dev, dtype=torch.float32)
    if grad_attention_weights_rb is None:
        grad_attention_weights_rb = torch.empty((d.B, d.Ncam, d.Nq, d.H, d.L, d.P), device=dev,
                                                dtype=torch.float32)
    _check(lib().sca_rebatched_backward(_ptr(value), _vdt(value), shapes.ctypes.data_as(_i64p),
                                        starts.ctypes.data_as(_i64p), _ptr(reference_points_cam),
                                        _ptr(sampling_offsets), _ptr(attention_logits),
                                        _ptr(grad_out), _ptr(idx), _ptr(count), _ptr(hits), d,
                                        _ptr(grad_value), _ptr(grad_sampling_locations_rb),
                                        _ptr(grad_attention_weights_rb), _stream(stream)),
           "sca_rebatched_backward")
    return grad_value, grad_sampling_locations_rb, grad_attention_weights_rb


def msda_linear(x, w, bias=None, residual=None, out=None, out_dtype=None, stream=None,
                dropout_p=0.0, dropout_seed=0):
    """y = x w^T (+ bias) (+ residual) on the tensor cores.  x [M, K] bf16,
    w [N, K] bf16, bias [N] fp32, residual [M, N] fp32 -> y [M, N] (fp32, or
    bf16 when out_dtype / out is bfloat16).  dropout_p > 0 applies
    training-time dropout to x w^T + bias before the residual."""
    torch = _torch()
    _contig(x, w, bias, residual, out)
    if x.dtype != torch.bfloat16 or w.dtype != torch.bfloat16:
        raise MsdaError("msda_linear takes bfloat16 x and w")
    M, K = x.shape
    N = w.shape[0]
    if out is None:
        out = torch.empty((M, N), device=x.device, dtype=out_dtype or torch.float32)
    ydt = MSDA_BF16 if out.dtype == torch.bfloat16 else MSDA_F32
    _check(lib().msda_linear_dropout(_ptr(x), _ptr(w), _ptr(bias), _ptr(residual), M, N, K,
                                     ydt, _ptr(out), float(dropout_p), int(dropout_seed),
                                     _stream(stream)),
           "msda_linear")
    return out


def sca_module_forward(query, query_pos, features, w_value, b_value, w_offsets, b_offsets,
                       w_weights, b_weights, w_output, b_output, reference_points_cam, bev_mask,
                       spatial_shapes, level_start_index, num_levels, num_points,
                       value_dtype=None, out=None, workspace=None, stream=None, dropout_p=0.0,
                       dropout_seed=0, camera_embeds=None, level_embeds=None):
    """The SCA module forward: q_hat = q + output_proj(SCA(value_proj(F~),
    offsets(q + pos), weights(q + pos))).  query, query_pos [B, Nq, C] fp32;
    features [B, Ncam, Nv, C] bf16; weights bf16 [out, in]; biases fp32;
    reference_points_cam [Ncam, B, Nq, R, 2]; bev_mask [Ncam, B, Nq, R]
    -> q_hat [B, Nq, C] fp32."""
    torch = _torch()
    _contig(query, query_pos, features, w_value, w_offsets, w_weights, w_output,
            reference_points_cam, bev_mask, camera_embeds, level_embeds)
    if bev_mask.dtype == torch.bool:
        bev_mask = bev_mask.view(torch.uint8)
    B, Nq, C = query.shape
    _, Ncam, Nv, _ = features.shape
    H = C // HEAD_DIM
    R = reference_points_cam.shape[3]
    vdt = MSDA_BF16 if value_dtype == torch.bfloat16 else MSDA_F32
    d = Dims(B, Ncam, Nq, Nv, H, num_levels, num_points, R)
    shapes, starts = _levels(spatial_shapes, level_start_index)
    if out is None:
        out = torch.empty((B, Nq, C), device=query.device, dtype=torch.float32)
    nbytes = int(lib().sca_module_workspace_size(d, vdt))
    if workspace is None:
        workspace = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=query.device)
    prm = ScaModuleParams(*[_ptr(t) for t in (query, query_pos, features, w_value, b_value,
                                              w_offsets, b_offsets, w_weights, b_weights,
                                              w_output, b_output, reference_points_cam,
                                              bev_mask)], vdt, float(dropout_p),
                           int(dropout_seed), _ptr(camera_embeds), _ptr(level_embeds))
    _check(lib().sca_module_forward(ctypes.byref(prm), shapes.ctypes.data_as(_i64p),
                                    starts.ctypes.data_as(_i64p), d, _ptr(workspace),
                                    workspace.numel(), _ptr(out), _stream(stream)),
           "sca_module_forward")
    return out


def sca_backward_inputs(spatial_shapes, level_start_index, attention_logits, pos,
                        grad_sampling_locations_rb, grad_attention_weights_rb, num_cameras,
                        num_anchors, out=None, stream=None):
    """-> (grad_sampling_offsets [B, Nq, H, L, P, 2], grad_attention_logits
    [B, Nq, H, L, P], grad_reference_points_cam [Ncam, B, Nq, R, 2]); `out`
    may supply the three tensors."""
    torch = _torch()
    _contig(attention_logits, pos, grad_sampling_locations_rb, grad_attention_weights_rb)
    B, Nq, H, L, P = attention_logits.shape
    Ncam, R = num_cameras, num_anchors
    shapes, starts = _levels(spatial_shapes, level_start_index)
    nv = int(np.max(starts + shapes[:, 0] * shapes[:, 1]))  # value rows the levels span
    d = Dims(B, Ncam, Nq, nv, H, L, P, R)
    dev = attention_logits.device
    if out is not None:
        g_off, g_lg, g_ref = out
        _contig(g_off, g_lg, g_ref)
    else:
        g_off = torch.empty((B, Nq, H, L, P, 2), device=dev, dtype=torch.float32)
        g_lg = torch.empty((B, Nq, H, L, P), device=dev, dtype=torch.float32)
        g_ref = torch.empty((Ncam, B, Nq, R, 2), device=dev, dtype=torch.float32)
    _check(lib().sca_backward_inputs(shapes.ctypes.data_as(_i64p), starts.ctypes.data_as(_i64p),
                                     _ptr(attention_logits), _ptr(pos),
                                     _ptr(grad_sampling_locations_rb),
                                     _ptr(grad_attention_weights_rb), d, _ptr(g_off), _ptr(g_lg),
                                     _ptr(g_ref), _stream(stream)),
           "sca_backward_inputs")
    return g_off, g_lg, g_ref
