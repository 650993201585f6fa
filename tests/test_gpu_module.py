"""sca_module_forward (the whole SCA module: projections on the tensor
cores, SCA, output projection plus residual) against the oracle's
composition of the same steps, through the C ABI.  Operands are bf16
(query + pos, features, weights, and g before the output projection), so the
bf16 bound applies: |q_hat - oracle| <= 2e-2.  With training-time dropout
both sides draw the mask from Philox4x32-10 on the same element index and
seed, so a mask difference would show as an error of the size of a value."""
import numpy as np
import pytest
import torch

import oracle
import scale_deformable_attention_03_b200 as msda
from scale_deformable_attention_03_b200 import inputs

pytestmark = pytest.mark.gpu


def _bf16_tensor(a):
    return torch.from_numpy(inputs.to_bf16_bits(a).view(np.int16)).cuda().view(torch.bfloat16)


SMALL = dict(bev_h=16, bev_w=20, shapes=[(29, 50), (15, 25), (8, 13), (4, 7)])
FULL = {}  # the BEVFormer-base sizes: 200 x 200 BEV, 6 cameras, 4 levels


@pytest.mark.parametrize("size,value_bf16,dropout_p,embeds", [
    ("small", False, 0.0, False), ("small", True, 0.0, False), ("small", False, 0.1, False),
    ("small", True, 0.3, False), ("small", False, 0.0, True), ("small", True, 0.1, True),
    ("full", False, 0.0, False), ("full", True, 0.1, True),
])
def test_module_matches_oracle(size, value_bf16, dropout_p, embeds):
    timeouts0 = msda.lib().msda_linear_timeouts()
    rng = np.random.Generator(np.random.PCG64(77))
    w = inputs.workload3(seed=78, **(SMALL if size == "small" else FULL))
    B, Ncam, Nq, Nv, H, L, P = w.B, w.Ncam, w.Nq, w.Nv, w.H, w.L, w.P
    C, S = H * 32, H * L * P
    q = rng.standard_normal((B, Nq, C)).astype(np.float32)
    pos = (rng.standard_normal((B, Nq, C)) * 0.1).astype(np.float32)
    feats = inputs.bf16_bits_to_f32(inputs.to_bf16_bits(
        rng.standard_normal((B, Ncam, Nv, C)).astype(np.float32)))

    def weight(n, scale):
        return inputs.bf16_bits_to_f32(inputs.to_bf16_bits(
            (rng.standard_normal((n, C)) * scale).astype(np.float32)))
    wv, wo = weight(C, C ** -0.5), weight(C, C ** -0.5)
    woff, ww = weight(2 * S, 0.1), weight(S, 0.1)
    bv, bo = (rng.standard_normal(C) * 0.1).astype(np.float32), (rng.standard_normal(C) * 0.1).astype(np.float32)
    boff, bw = rng.standard_normal(2 * S).astype(np.float32), rng.standard_normal(S).astype(np.float32)

    e_cam = (rng.standard_normal((Ncam, C)) * 0.5).astype(np.float32) if embeds else None
    e_lvl = (rng.standard_normal((L, C)) * 0.5).astype(np.float32) if embeds else None

    def t(a):
        return None if a is None else torch.from_numpy(np.ascontiguousarray(a)).cuda()
    out = msda.sca_module_forward(
        t(q), t(pos), _bf16_tensor(feats), _bf16_tensor(wv), t(bv), _bf16_tensor(woff), t(boff),
        _bf16_tensor(ww), t(bw), _bf16_tensor(wo), t(bo), t(w.reference_points), t(w.bev_mask),
        w.spatial_shapes, w.level_start_index, L, P,
        value_dtype=torch.bfloat16 if value_bf16 else torch.float32, dropout_p=dropout_p,
        dropout_seed=0x1234_5678_9ABC, camera_embeds=t(e_cam), level_embeds=t(e_lvl))
    torch.cuda.synchronize()
    ref = oracle.sca_module_forward(q, pos, feats, wv, bv, woff, boff, ww, bw, wo, bo,
                                    w.reference_points, w.bev_mask, w.spatial_shapes,
                                    w.level_start_index, L, P, value_bf16=value_bf16,
                                    dropout_p=dropout_p, dropout_seed=0x1234_5678_9ABC,
                                    camera_embeds=e_cam, level_embeds=e_lvl)
    err = np.abs(out.cpu().numpy().astype(np.float64) - ref)
    assert err.max() <= 2e-2, err.max()
    assert msda.lib().msda_linear_timeouts() == timeouts0
