"""The query-major SCA forward on the GPU against the oracle, through the C
ABI: the full BEVFormer-base size (fp32 and bf16 value), randomised problems
(odd head counts take the one-head bf16 path; more batch-camera pairs than the
rebatched path accepts), unseen queries, and agreement with sca_forward."""
import numpy as np
import pytest
import torch

import oracle
import scale_deformable_attention_03_b200 as msda
from scale_deformable_attention_03_b200 import inputs

from .gpu_util import assert_close, dev, value_tensor

pytestmark = pytest.mark.gpu


def _qm(w, bf16):
    out = msda.sca_forward_query_major(value_tensor(w, bf16), w.spatial_shapes,
                                       w.level_start_index, dev(w.reference_points),
                                       dev(w.bev_mask), dev(w.sampling_offsets),
                                       dev(w.attention_logits))
    torch.cuda.synchronize()
    ref = oracle.sca_forward(w.value, w.spatial_shapes, w.level_start_index, w.reference_points,
                             w.bev_mask, w.sampling_offsets, w.attention_logits)
    return out, ref


@pytest.mark.parametrize("bf16", [False, True])
def test_workload3_bevformer_base(bf16):
    w = inputs.workload3(value_dtype="bf16" if bf16 else "f32")
    out, ref = _qm(w, bf16)
    assert_close(out, ref, bf16, "query-major SCA, BEVFormer-base")


@pytest.mark.parametrize("seed,B,Ncam,bev,shapes,H,P,R", [
    (111, 2, 3, (7, 9), [(9, 13), (4, 7)], 2, 4, 2),
    (112, 3, 6, (33, 35), [(16, 20), (8, 10), (4, 5), (2, 3)], 8, 8, 4),
    (113, 1, 1, (1, 3), [(5, 5)], 1, 2, 1),
    (114, 2, 5, (20, 52), [(6, 7)] * 3, 4, 12, 3),   # L*P = 36: two chunks
    (115, 1, 32, (6, 10), [(8, 8), (4, 4)], 3, 4, 1),  # 32 cameras, odd H
    (116, 40, 32, (2, 3), [(3, 4)], 2, 2, 2),          # B * Ncam = 1280
])
@pytest.mark.parametrize("bf16", [False, True])
def test_random_sca_query_major(seed, B, Ncam, bev, shapes, H, P, R, bf16):
    w = inputs.workload3(seed=seed, B=B, Ncam=Ncam, bev_h=bev[0], bev_w=bev[1], shapes=shapes,
                         H=H, P=P, R=R, rho="uniform", same_mask=False,
                         value_dtype="bf16" if bf16 else "f32")
    w.sampling_offsets *= 3  # many reads leave the maps
    if Ncam > 2:  # some queries seen by three or more cameras
        w.bev_mask[:3, :, ::5, 0] = 1
    out, ref = _qm(w, bf16)
    assert_close(out, ref, bf16, f"query-major SCA {seed}")


def test_unseen_queries_are_zero():
    w = inputs.workload3(seed=121, bev_h=16, bev_w=16)
    w.bev_mask[:, :, :50, :] = 0
    out, ref = _qm(w, False)
    assert torch.all(out[:, :50] == 0)
    assert_close(out, ref, False, "unseen queries")


def test_agrees_with_the_rebatched_path():
    w = inputs.workload3(seed=122, bev_h=60, bev_w=80)
    args = (dev(w.value), w.spatial_shapes, w.level_start_index, dev(w.reference_points),
            dev(w.bev_mask), dev(w.sampling_offsets), dev(w.attention_logits))
    a = msda.sca_forward_query_major(*args)
    b = msda.sca_forward(*args)
    torch.cuda.synchronize()
    assert_close(a, b.cpu().numpy(), False, "query-major vs rebatched")


def test_empty():
    w = inputs.workload3(seed=123, bev_h=4, bev_w=4)
    z = np.zeros((1, 0) + w.sampling_offsets.shape[2:], np.float32)
    out = msda.sca_forward_query_major(
        dev(w.value), w.spatial_shapes, w.level_start_index,
        dev(np.zeros((w.Ncam, 1, 0, w.R, 2), np.float32)),
        dev(np.zeros((w.Ncam, 1, 0, w.R), np.uint8)), dev(z),
        dev(np.zeros((1, 0) + w.attention_logits.shape[2:], np.float32)))
    assert out.shape == (1, 0, w.H * 32)
