"""Out-of-bounds writes, checked with canary bands (in place of a memory
checker): every output and workspace of every entry point is placed inside a
larger device buffer whose 4 KiB before and after are filled with a canary
byte; after the call (and a synchronisation) the bands must be unchanged, byte
for byte.  Small problems with ragged sizes, on each entry point through the
C ABI.  Also: inconsistent compaction lists (counts above Nq, indices out of
range) read and write nothing outside the rebatched blocks.
"""
import ctypes

import numpy as np
import pytest
import torch

import scale_deformable_attention_03_b200 as msda
from scale_deformable_attention_03_b200 import inputs

from .gpu_util import dev, softmax_weights

pytestmark = pytest.mark.gpu

MARGIN = 4096
CANARY = 0xA5


class Guards:
    """Device tensors carved from canary-filled buffers."""

    def __init__(self):
        self.bufs = []

    def tensor(self, shape, dtype, fill=None):
        elem = torch.empty((), dtype=dtype).element_size()
        n = int(np.prod(shape)) * elem
        buf = torch.full((MARGIN + ((n + 255) // 256) * 256 + MARGIN,), CANARY,
                         dtype=torch.uint8, device="cuda")
        view = buf[MARGIN:MARGIN + n].view(dtype).view(shape)
        if fill is not None:
            view.fill_(fill)
        self.bufs.append((buf, n))
        return view

    def bytes(self, n):
        return self.tensor((max(int(n), 16),), torch.uint8)

    def check(self, what):
        torch.cuda.synchronize()
        for i, (buf, n) in enumerate(self.bufs):
            h = buf.cpu().numpy()
            before, after = h[:MARGIN], h[MARGIN + n:]
            assert np.all(before == CANARY), f"{what}: buffer {i} written before its start"
            assert np.all(after == CANARY), f"{what}: buffer {i} written past its end"


def _sca_problem(seed=61, B=2, Ncam=3, bev=(5, 7), shapes=((9, 13), (4, 7)), H=2, P=4, R=2):
    return inputs.workload3(seed=seed, B=B, Ncam=Ncam, bev_h=bev[0], bev_w=bev[1],
                            shapes=list(shapes), H=H, P=P, R=R, rho="uniform", same_mask=False,
                            with_grad=True)


def _sca_tensors(w):
    return (dev(w.value), w.spatial_shapes, w.level_start_index, dev(w.reference_points),
            dev(w.bev_mask), dev(w.sampling_offsets), dev(w.attention_logits))


@pytest.mark.parametrize("H,P", [(2, 4), (8, 4), (3, 12)])
def test_msda_forward_and_backward(H, P):
    rng = np.random.Generator(np.random.PCG64(62 + H))
    s, starts, Nv = inputs.level_table([(7, 9), (3, 5)])
    B, Nq, L = 2, 37, 2
    value = dev(rng.standard_normal((B, Nv, H, 32)).astype(np.float32))
    loc = dev(rng.uniform(-0.2, 1.2, (B, Nq, H, L, P, 2)).astype(np.float32))
    wts = dev(softmax_weights(rng.standard_normal((B, Nq, H, L, P)), L * P))
    ref = dev(rng.uniform(-0.1, 1.1, (B, Nq, 1, 2)).astype(np.float32))
    off = dev(rng.standard_normal((B, Nq, H, L, P, 2)).astype(np.float32))
    lg = dev(rng.standard_normal((B, Nq, H, L, P)).astype(np.float32))
    gout = dev(rng.standard_normal((B, Nq, H * 32)).astype(np.float32))
    g = Guards()
    out = g.tensor((B, Nq, H * 32), torch.float32)
    msda.msda_forward(value, s, starts, loc, wts, out=out)
    msda.msda_forward_fused(value, s, starts, ref, off, lg, out=out)
    gv = g.tensor(tuple(value.shape), torch.float32)
    gl = g.tensor(tuple(loc.shape), torch.float32)
    gw = g.tensor(tuple(wts.shape), torch.float32)
    msda.msda_backward(value, s, starts, loc, wts, gout, gv, gl, gw)
    ws = g.bytes(msda.lib().msda_backward_deterministic_workspace_size(
        msda.Dims(B, 1, Nq, Nv, H, L, P, 1)))
    msda.msda_backward(value, s, starts, loc, wts, gout, gv, gl, gw, deterministic=True,
                       workspace=ws)
    g.check("msda forward / backward")


def test_sca_entry_points():
    w = _sca_problem()
    value, s, starts, ref, mask, off, lg = _sca_tensors(w)
    gout = dev(w.grad_out)
    B, Ncam, Nq, H, L, P, R = w.B, w.Ncam, w.Nq, w.H, w.L, w.P, w.R
    d = msda.Dims(B, Ncam, Nq, w.Nv, H, L, P, R)
    g = Guards()
    i32 = torch.int32
    idx, count, pos = g.tensor((B, Ncam, Nq), i32), g.tensor((B, Ncam), i32), \
        g.tensor((B, Ncam, Nq), i32)
    hits = g.tensor((B, Nq), i32)
    msda.sca_compact(mask, workspace=g.bytes(msda.sca_compact_workspace_size(d)),
                     out=(idx, count, pos, hits))
    out_rb = g.tensor((B, Ncam, Nq, H * 32), torch.float32)
    msda.sca_rebatched_forward(value, s, starts, ref, off, lg, idx, count, out_rb=out_rb)
    out = g.tensor((B, Nq, H * 32), torch.float32)
    msda.sca_camera_average(out_rb, pos, hits, out=out)
    msda.sca_forward(value, s, starts, ref, mask, off, lg, out=out,
                     workspace=g.bytes(msda.msda_workspace_size(d)))
    msda.sca_forward_query_major(value, s, starts, ref, mask, off, lg, out=out)
    gv = g.tensor(tuple(value.shape), torch.float32)
    gl = g.tensor((B, Ncam, Nq, H, L, P, 2), torch.float32)
    gw = g.tensor((B, Ncam, Nq, H, L, P), torch.float32)
    msda.sca_rebatched_backward(value, s, starts, ref, off, lg, gout, idx, count, hits, gv, gl,
                                gw)
    msda.sca_backward(value, s, starts, ref, mask, off, lg, gout, gv, gl, gw,
                      workspace=g.bytes(msda.msda_workspace_size(d)))
    msda.sca_backward(value, s, starts, ref, mask, off, lg, gout, gv, gl, gw,
                      workspace=g.bytes(msda.lib().sca_backward_deterministic_workspace_size(d)),
                      deterministic=True)
    g_off = g.tensor(tuple(off.shape), torch.float32)
    g_lg = g.tensor(tuple(lg.shape), torch.float32)
    g_ref = g.tensor(tuple(ref.shape), torch.float32)
    msda.sca_backward_inputs(s, starts, lg, pos, gl, gw, Ncam, R, out=(g_off, g_lg, g_ref))
    msda.sca_backward_full(value, s, starts, ref, mask, off, lg, gout,
                           out=(gv, g_off, g_lg, g_ref),
                           workspace=g.bytes(msda.lib().sca_backward_full_workspace_size(d)))
    g.check("sca entry points")


def test_sca_no_alloc_compaction():
    w = _sca_problem(seed=63)
    mask = dev(w.bev_mask)
    B, Ncam, Nq, R = w.B, w.Ncam, w.Nq, w.R
    g = Guards()
    i32 = torch.int32
    idx, count, pos = g.tensor((B, Ncam, Nq), i32), g.tensor((B, Ncam), i32), \
        g.tensor((B, Ncam, Nq), i32)
    hits = g.tensor((B, Nq), i32)
    f = msda.lib().sca_compact_no_alloc
    f.argtypes = [ctypes.c_void_p, msda.Dims] + [ctypes.c_void_p] * 5
    f.restype = ctypes.c_int
    p = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731
    st = f(p(mask), msda.Dims(B, Ncam, Nq, 1, 1, 1, 1, R), p(idx), p(count), p(pos), p(hits),
           ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0
    g.check("sca_compact_no_alloc")


def test_tsa_entry_points():
    rng = np.random.Generator(np.random.PCG64(64))
    bh, bw, T, H, P = 6, 7, 2, 8, 4
    s, starts, Nv = inputs.level_table([(bh, bw)])
    Nq = bh * bw
    value = dev(rng.standard_normal((T, Nv, H, 32)).astype(np.float32))
    off = dev(rng.standard_normal((T, Nq, H, 1, P, 2)).astype(np.float32))
    lg = dev(rng.standard_normal((T, Nq, H, 1, P)).astype(np.float32))
    gout = dev(rng.standard_normal((1, Nq, H * 32)).astype(np.float32))
    ego = dev(np.array([[[0.7, -0.3, 5.0], [0.0, 0.0, 0.0]]], np.float32))
    g = Guards()
    ref = g.tensor((1, T, Nq, 2), torch.float32)
    msda.tsa_reference_points(ego, bh, bw, out=ref)
    refv = ref.view(T, Nq, 1, 2)
    out = g.tensor((1, Nq, H * 32), torch.float32)
    msda.tsa_forward(value, s, starts, refv, off, lg, T, out=out)
    outs = (g.tensor((T, Nv, H, 32), torch.float32), g.tensor((T, Nq, H, 1, P, 2), torch.float32),
            g.tensor((T, Nq, H, 1, P), torch.float32), g.tensor((T, Nq, 1, 2), torch.float32))
    ws = g.bytes(msda.lib().tsa_backward_workspace_size(msda.Dims(1, 1, Nq, Nv, H, 1, P, 1), T))
    msda.tsa_backward(value, s, starts, refv, off, lg, T, gout, workspace=ws, out=outs)
    g.check("tsa entry points")


@pytest.mark.parametrize("M,N,K,out_bf16", [(300, 256, 256, False), (129, 512, 64, True)])
def test_linear(M, N, K, out_bf16):
    gen = torch.Generator(device="cuda").manual_seed(65)
    x = torch.randn((M, K), device="cuda", generator=gen).to(torch.bfloat16)
    wt = torch.randn((N, K), device="cuda", generator=gen).to(torch.bfloat16)
    bias = torch.randn(N, device="cuda", generator=gen)
    res = torch.randn((M, N), device="cuda", generator=gen)
    g = Guards()
    y = g.tensor((M, N), torch.bfloat16 if out_bf16 else torch.float32)
    msda.msda_linear(x, wt, bias, res, out=y)
    msda.msda_linear(x, wt, bias, res, out=y, dropout_p=0.25, dropout_seed=9)
    g.check("msda_linear")


@pytest.mark.parametrize("H,N,out_bf16", [(8, 256, False), (2, 512, True)])
def test_sca_camera_average_linear(H, N, out_bf16):
    rng = np.random.Generator(np.random.PCG64(67 + H))
    B, Ncam, Nq, C = 2, 5, 133, H * 32
    mask = (rng.random((Ncam, B, Nq, 2)) < 0.4).astype(np.uint8)
    g = Guards()
    idx, count, pos, hits = msda.sca_compact(dev(mask))
    rb = g.tensor((B, Ncam, Nq, C), torch.float32)
    rb.copy_(torch.from_numpy(rng.standard_normal((B, Ncam, Nq, C)).astype(np.float32)))
    wt = torch.from_numpy(rng.standard_normal((N, C)).astype(np.float32)).cuda().to(torch.bfloat16)
    bias = torch.from_numpy(rng.standard_normal(N).astype(np.float32)).cuda()
    res = torch.from_numpy(rng.standard_normal((B * Nq, N)).astype(np.float32)).cuda()
    y = g.tensor((B * Nq, N), torch.bfloat16 if out_bf16 else torch.float32)
    msda.sca_camera_average_linear(rb, pos, hits, wt, bias, res, out=y)
    msda.sca_camera_average_linear(rb, pos, hits, wt, bias, res, out=y, dropout_p=0.2,
                                   dropout_seed=5)
    g.check("sca_camera_average_linear")


def test_sca_module_forward():
    # C = 256 and H * L * P = 256: the projections' N (2 * 256, 256) are multiples of 256
    w = _sca_problem(seed=66, B=1, Ncam=2, bev=(4, 6), shapes=((6, 8), (3, 4), (2, 2), (1, 2)),
                     H=8, P=8, R=4)
    C, S = w.H * 32, w.H * w.L * w.P
    gen = torch.Generator(device="cuda").manual_seed(66)
    q = torch.randn((w.B, w.Nq, C), device="cuda", generator=gen)
    feats = torch.randn((w.B, w.Ncam, w.Nv, C), device="cuda", generator=gen).to(torch.bfloat16)

    def lin(n):
        return ((torch.randn((n, C), device="cuda", generator=gen) / 16).to(torch.bfloat16),
                torch.randn(n, device="cuda", generator=gen) * 0.1)

    (wv, bv), (wo, bo), (wa, ba), (wout, bout) = lin(C), lin(2 * S), lin(S), lin(C)
    d = msda.Dims(w.B, w.Ncam, w.Nq, w.Nv, w.H, w.L, w.P, w.R)
    g = Guards()
    out = g.tensor((w.B, w.Nq, C), torch.float32)
    ws = g.bytes(msda.lib().sca_module_workspace_size(d, msda.MSDA_F32))
    msda.sca_module_forward(q, None, feats, wv, bv, wo, bo, wa, ba, wout, bout,
                            dev(w.reference_points), dev(w.bev_mask), w.spatial_shapes,
                            w.level_start_index, w.L, w.P, out=out, workspace=ws,
                            dropout_p=0.1, dropout_seed=3)
    g.check("sca_module_forward")


def test_inconsistent_lists_stay_inside_their_blocks():
    """Counts above Nq (or negative) and indices outside [0, Nq): the
    rebatched kernels clamp every count to Nq and skip bad indices, so
    nothing outside out_rb and the gradients is touched."""
    w = _sca_problem(seed=67)
    value, s, starts, ref, mask, off, lg = _sca_tensors(w)
    B, Ncam, Nq, H, L, P = w.B, w.Ncam, w.Nq, w.H, w.L, w.P
    rng = np.random.Generator(np.random.PCG64(67))
    g = Guards()
    idx = g.tensor((B, Ncam, Nq), torch.int32)
    idx.copy_(torch.from_numpy(rng.integers(-3, Nq + 3, (B, Ncam, Nq)).astype(np.int32)))
    count = g.tensor((B, Ncam), torch.int32)
    count.copy_(torch.tensor([[Nq + 5, -2, Nq], [3, Nq * 4, 0]][:B], dtype=torch.int32)[:, :Ncam])
    hits = g.tensor((B, Nq), torch.int32, fill=1)
    out_rb = g.tensor((B, Ncam, Nq, H * 32), torch.float32)
    msda.sca_rebatched_forward(value, s, starts, ref, off, lg, idx, count, out_rb=out_rb)
    gout = dev(w.grad_out)
    gv = g.tensor(tuple(value.shape), torch.float32)
    gl = g.tensor((B, Ncam, Nq, H, L, P, 2), torch.float32)
    gw = g.tensor((B, Ncam, Nq, H, L, P), torch.float32)
    msda.sca_rebatched_backward(value, s, starts, ref, off, lg, gout, idx, count, hits, gv, gl,
                                gw)
    g.check("inconsistent lists")
