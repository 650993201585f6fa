"""SCA on the GPU against the oracle, through the C ABI: the compaction
bit-exact, the forward element by element at the full BEVFormer-base size
(fp32 and bf16 value, coherent and uniform reference points) and on small
randomised problems with several batch items and cameras."""
import numpy as np
import pytest
import torch

import oracle
import scale_deformable_attention_03_b200 as msda
from scale_deformable_attention_03_b200 import inputs

from .gpu_util import assert_close, dev, value_tensor

pytestmark = pytest.mark.gpu


def _compact_gpu(mask):
    idx, cnt, pos, hits = msda.sca_compact(dev(mask))
    torch.cuda.synchronize()
    return [t.cpu().numpy() for t in (idx, cnt, pos, hits)]


def _assert_compaction_equal(mask):
    got = _compact_gpu(mask)
    want = oracle.sca_compact(mask)
    for name, g, w in zip(("idx", "count", "pos", "hits"), got, want):
        assert g.dtype == np.int32 and g.shape == w.shape, name
        assert np.array_equal(g, w), f"{name} differs at {np.argwhere(g != w)[:5]}"


def test_compaction_workload3_bit_exact():
    w = inputs.workload3()
    _assert_compaction_equal(w.bev_mask)


@pytest.mark.parametrize("shape,p", [
    ((6, 1, 40000, 4), 0.1),
    ((6, 2, 1025, 4), 0.3),     # two chunks, ragged tail of one query
    ((3, 3, 1023, 1), 0.5),
    ((1, 1, 31, 2), 0.5),       # less than a warp
    ((32, 1, 2048, 3), 0.05),   # the camera limit
    ((5, 2, 4097, 8), 0.02),
    ((6, 1, 65536, 2), 0.1),    # 64 chunks: the scatter pass sums the chunk counts itself
    ((6, 1, 65537, 2), 0.1),    # 65 chunks: the separate scan pass
    ((2, 2, 150000, 1), 0.05),  # 147 chunks per (batch, camera)
])
def test_compaction_random_bit_exact(shape, p):
    rng = np.random.Generator(np.random.PCG64(sum(shape)))
    _assert_compaction_equal((rng.random(shape) < p).astype(np.uint8))


@pytest.mark.parametrize("fill", [0, 1])
def test_compaction_all_or_nothing(fill):
    _assert_compaction_equal(np.full((6, 2, 3000, 4), fill, np.uint8))


@pytest.mark.parametrize("R", [1, 2, 4, 8, 3])
def test_compaction_mask_at_odd_address(R):
    """The compaction reads a query's R anchor bytes as one word when R is
    1, 2, 4 or 8 and the mask is aligned to R bytes, byte by byte otherwise:
    a mask one byte past an aligned address (and R = 3) takes the byte path,
    with the same lists."""
    rng = np.random.Generator(np.random.PCG64(60 + R))
    Ncam, B, Nq = 5, 2, 2500
    mask = (rng.random((Ncam, B, Nq, R)) < 0.3).astype(np.uint8)
    mask[:, :, ::7, :] = 0
    buf = torch.zeros(mask.size + 16, dtype=torch.uint8, device="cuda")
    off = buf[1:1 + mask.size].view(mask.shape)
    off.copy_(torch.from_numpy(mask))
    aligned = dev(mask)
    got_off = [t.cpu().numpy() for t in msda.sca_compact(off)]
    got = [t.cpu().numpy() for t in msda.sca_compact(aligned)]
    want = oracle.sca_compact(mask)
    for name, a, b, c in zip(("idx", "count", "pos", "hits"), got_off, got, want):
        assert np.array_equal(a, c), f"{name} (odd address)"
        assert np.array_equal(b, c), f"{name} (aligned)"


def test_compaction_non_binary_mask_bytes():
    rng = np.random.Generator(np.random.PCG64(3))
    mask = rng.integers(0, 256, (4, 1, 999, 4)).astype(np.uint8) * (rng.random((4, 1, 999, 4)) < 0.2)
    _assert_compaction_equal(mask.astype(np.uint8))


def _sca(w, bf16):
    out = msda.sca_forward(value_tensor(w, bf16), w.spatial_shapes, w.level_start_index,
                           dev(w.reference_points), dev(w.bev_mask), dev(w.sampling_offsets),
                           dev(w.attention_logits))
    torch.cuda.synchronize()
    ref = oracle.sca_forward(w.value, w.spatial_shapes, w.level_start_index, w.reference_points,
                             w.bev_mask, w.sampling_offsets, w.attention_logits)
    return out, ref


@pytest.mark.parametrize("bf16", [False, True])
def test_workload3_bevformer_base(bf16):
    w = inputs.workload3(value_dtype="bf16" if bf16 else "f32")
    out, ref = _sca(w, bf16)
    assert_close(out, ref, bf16, "workload 3 SCA")


def test_workload3_uniform_reference_points():
    w = inputs.workload3(rho="uniform", bev_h=100, bev_w=200)
    out, ref = _sca(w, False)
    assert_close(out, ref, False, "workload 3 SCA, uniform rho")


@pytest.mark.parametrize("seed,B,Ncam,bev,shapes,H,P,R", [
    (11, 2, 3, (7, 9), [(9, 13), (4, 7)], 2, 4, 2),
    (12, 3, 6, (33, 35), [(16, 20), (8, 10), (4, 5), (2, 3)], 8, 8, 4),
    (13, 1, 1, (1, 3), [(5, 5)], 1, 2, 1),
    (14, 2, 5, (20, 52), [(6, 7)] * 3, 4, 12, 3),   # L*P = 36: two chunks
])
def test_random_sca(seed, B, Ncam, bev, shapes, H, P, R):
    w = inputs.workload3(seed=seed, B=B, Ncam=Ncam, bev_h=bev[0], bev_w=bev[1], shapes=shapes,
                         H=H, P=P, R=R, rho="uniform", same_mask=False)
    # widen the offsets so that many reads leave the maps
    w.sampling_offsets *= 3
    out, ref = _sca(w, False)
    assert_close(out, ref, False, f"random SCA {seed}")


def test_queries_seen_by_no_camera_are_zero():
    w = inputs.workload3(seed=21, bev_h=16, bev_w=16)
    w.bev_mask[:, :, :50, :] = 0
    out, ref = _sca(w, False)
    assert torch.all(out[:, :50] == 0)
    assert_close(out, ref, False, "unseen queries")


def test_empty_mask():
    w = inputs.workload3(seed=22, bev_h=8, bev_w=8)
    w.bev_mask[:] = 0
    out, _ = _sca(w, False)
    assert torch.all(out == 0)


def test_rebatched_bf16_full_size():
    """The staged rebatched path with bf16 value (head-pair gather) at the
    full BEVFormer-base size, against the oracle and bit for bit against
    sca_forward, which runs the same kernels."""
    w = inputs.workload3(value_dtype="bf16")
    v = value_tensor(w, True)
    args = (v, w.spatial_shapes, w.level_start_index, dev(w.reference_points))
    idx, count, pos, hits = msda.sca_compact(dev(w.bev_mask))
    rows = msda.sca_rebatched_forward(*args, dev(w.sampling_offsets), dev(w.attention_logits),
                                      idx, count)
    staged = msda.sca_camera_average(rows, pos, hits)
    whole = msda.sca_forward(*args, dev(w.bev_mask), dev(w.sampling_offsets),
                             dev(w.attention_logits))
    torch.cuda.synchronize()
    ref = oracle.sca_forward(w.value, w.spatial_shapes, w.level_start_index, w.reference_points,
                             w.bev_mask, w.sampling_offsets, w.attention_logits)
    assert_close(staged, ref, True, "staged bf16 SCA")
    assert_close(whole, ref, True, "sca_forward bf16")
    assert torch.equal(staged, whole)


def test_rebatched_rows_into_16_byte_aligned_buffer():
    """The gather writes each lane's eight channels with one 32-byte store
    when out_rb is 32-byte aligned and with two 16-byte stores otherwise:
    the same rows either way."""
    w = inputs.workload3(seed=45, bev_h=20, bev_w=30)
    args = (dev(w.value), w.spatial_shapes, w.level_start_index, dev(w.reference_points),
            dev(w.sampling_offsets), dev(w.attention_logits))
    idx, count, pos, hits = msda.sca_compact(dev(w.bev_mask))
    shape = (w.B, w.Ncam, w.Nq, w.H * 32)
    n = w.B * w.Ncam * w.Nq * w.H * 32
    store = torch.zeros(n + 8, device="cuda")
    assert store.data_ptr() % 32 == 0
    aligned = msda.sca_rebatched_forward(*args, idx, count, out_rb=store[:n].view(shape))
    off16 = msda.sca_rebatched_forward(*args, idx, count,
                                       out_rb=torch.zeros(n + 8, device="cuda")[4:4 + n].view(shape))
    torch.cuda.synchronize()
    assert off16.data_ptr() % 32 == 16
    cnt = count.cpu().numpy().reshape(-1)
    for bc in range(len(cnt)):
        b, c = divmod(bc, w.Ncam)
        assert torch.equal(aligned[b, c, :cnt[bc]], off16[b, c, :cnt[bc]])


def test_sca_forward_in_a_cuda_graph():
    """sca_forward captured once into a CUDA graph (its launches, the
    overlapping ones included, become graph nodes) and replayed on new inputs
    copied into the captured buffers: each replay equals a direct call bit
    for bit."""
    ws = [inputs.workload3(seed=s, bev_h=30, bev_w=40) for s in (46, 47)]
    w0 = ws[0]
    dims = msda.Dims(w0.B, w0.Ncam, w0.Nq, w0.Nv, w0.H, w0.L, w0.P, w0.R)
    workspace = torch.empty(msda.msda_workspace_size(dims), dtype=torch.uint8, device="cuda")
    bufs = [dev(w0.value), dev(w0.reference_points), dev(w0.bev_mask), dev(w0.sampling_offsets),
            dev(w0.attention_logits)]
    out = torch.empty((w0.B, w0.Nq, w0.H * 32), device="cuda")

    def call(stream=None):
        msda.sca_forward(bufs[0], w0.spatial_shapes, w0.level_start_index, bufs[1], bufs[2],
                         bufs[3], bufs[4], out=out, workspace=workspace, stream=stream)

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        call(side)  # warm-up outside the capture
    torch.cuda.current_stream().wait_stream(side)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        call(torch.cuda.current_stream())
    for w in ws + ws[:1]:
        for b, a in zip(bufs, (w.value, w.reference_points, w.bev_mask, w.sampling_offsets,
                               w.attention_logits)):
            b.copy_(torch.from_numpy(np.ascontiguousarray(a)))
        graph.replay()
        direct = msda.sca_forward(dev(w.value), w.spatial_shapes, w.level_start_index,
                                  dev(w.reference_points), dev(w.bev_mask),
                                  dev(w.sampling_offsets), dev(w.attention_logits))
        torch.cuda.synchronize()
        assert torch.equal(out, direct)
    del graph


def test_back_to_back_calls_share_one_workspace():
    """Consecutive calls on one stream with different masks and inputs, one
    workspace and one set of lists, no host synchronisation in between: each
    result must be its own.  The compaction's later passes, the gather and the
    camera average begin while the kernel before them finishes (programmatic
    dependent launches); this checks that a call's lists and rows are never
    read before they are complete, nor overwritten while the call before
    still reads them."""
    ws = [inputs.workload3(seed=s, bev_h=40, bev_w=50, rho=rho, same_mask=False)
          for s, rho in ((41, "coherent"), (42, "uniform"), (43, "coherent"))]
    ws[1].bev_mask[:, :, ::3, :] = 0  # fewer rows than the call before it
    dims = msda.Dims(ws[0].B, ws[0].Ncam, ws[0].Nq, ws[0].Nv, ws[0].H, ws[0].L, ws[0].P,
                     ws[0].R)
    workspace = torch.empty(msda.msda_workspace_size(dims), dtype=torch.uint8, device="cuda")
    dev_args = [(dev(w.value), w.spatial_shapes, w.level_start_index, dev(w.reference_points),
                 dev(w.bev_mask), dev(w.sampling_offsets), dev(w.attention_logits)) for w in ws]
    outs = [msda.sca_forward(*a, workspace=workspace) for a in dev_args + dev_args[:1]]
    lists = msda.sca_compact(dev_args[0][4])
    rows = torch.empty((ws[0].B, ws[0].Ncam, ws[0].Nq, ws[0].H * 32), device="cuda")
    staged = []
    for a in dev_args:
        msda.sca_compact(a[4], out=lists)
        msda.sca_rebatched_forward(*a[:4], a[5], a[6], lists[0], lists[1], out_rb=rows)
        staged.append(msda.sca_camera_average(rows, lists[2], lists[3]))
    torch.cuda.synchronize()
    for k, w in enumerate(ws):
        ref = oracle.sca_forward(w.value, w.spatial_shapes, w.level_start_index,
                                 w.reference_points, w.bev_mask, w.sampling_offsets,
                                 w.attention_logits)
        assert_close(outs[k], ref, False, f"sca_forward call {k}")
        assert torch.equal(staged[k], outs[k]), f"staged call {k}"
    assert torch.equal(outs[3], outs[0])


def test_staged_calls_equal_sca_forward():
    """sca_compact + sca_rebatched_forward + sca_camera_average is sca_forward,
    bit for bit, and the rebatched rows match the oracle's."""
    w = inputs.workload3(seed=23, bev_h=50, bev_w=60)
    args = (dev(w.value), w.spatial_shapes, w.level_start_index, dev(w.reference_points))
    idx, count, pos, hits = msda.sca_compact(dev(w.bev_mask))
    rows = msda.sca_rebatched_forward(*args, dev(w.sampling_offsets), dev(w.attention_logits),
                                      idx, count)
    staged = msda.sca_camera_average(rows, pos, hits)
    whole = msda.sca_forward(*args, dev(w.bev_mask), dev(w.sampling_offsets),
                             dev(w.attention_logits))
    torch.cuda.synchronize()
    assert torch.equal(staged, whole)
    ref, ref_rb = oracle.sca_forward(w.value, w.spatial_shapes, w.level_start_index,
                                     w.reference_points, w.bev_mask, w.sampling_offsets,
                                     w.attention_logits, return_rebatched=True)
    cnt = count.cpu().numpy()
    for c in range(w.Ncam):
        n = cnt[0, c]
        assert_close(rows[0, c, :n], ref_rb[0, c, :n], False, f"rebatched rows, camera {c}")
