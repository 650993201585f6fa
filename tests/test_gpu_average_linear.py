"""sca_camera_average_linear (the SCA camera average formed inside the
tensor-core output projection) through the C ABI.

Two checks per case:
  - bit for bit against the split path on the GPU (sca_camera_average, a
    bf16 conversion, msda_linear_dropout): the fused kernel must form the
    same bf16 operand (same sum order, division and rounding) and run the
    same projection;
  - element by element against the oracle: its camera average, rounded to
    bf16, through its projection (and its dropout).  The bound follows from
    the arithmetic: the kernel's fp32 average and the oracle's double average
    may round to neighbouring bf16 values (one bf16 ulp, at most 2^-7 |g|),
    and the K products are summed in fp32 (K * 2^-24 of the magnitudes), so
    |y - oracle| <= 1e-6 + (2^-7 + (K + 2) 2^-24) * (|g| |W|^T + |b|) * s + |r| 2^-24
    with s = 1 / (1 - p) under dropout; a bf16 output adds 2^-8 |y|.
"""
import numpy as np
import pytest
import torch

import oracle
import scale_deformable_attention_03_b200 as msda
from scale_deformable_attention_03_b200 import inputs

from .gpu_util import dev

pytestmark = pytest.mark.gpu


def _bf16(a):
    bits = inputs.to_bf16_bits(np.asarray(a, dtype=np.float32))
    return inputs.bf16_bits_to_f32(bits), torch.from_numpy(bits.view(np.int16)).cuda().view(torch.bfloat16)


def _run(mask, rb, N, out_bf16, with_bias, with_res, p, seed):
    rng = np.random.Generator(np.random.PCG64(seed))
    B, Ncam, Nq, C = rb.shape
    _, _, pos, hits = oracle.sca_compact(mask)
    w32, w = _bf16(rng.standard_normal((N, C)) / np.sqrt(C))
    b = rng.standard_normal(N).astype(np.float32) if with_bias else None
    r = rng.standard_normal((B * Nq, N)).astype(np.float32) if with_res else None
    bt = dev(b) if b is not None else None
    rt = dev(r) if r is not None else None
    odt = torch.bfloat16 if out_bf16 else torch.float32
    timeouts0 = msda.lib().msda_linear_timeouts()
    rbt, post, hitst = dev(rb), dev(pos), dev(hits)
    y = msda.sca_camera_average_linear(rbt, post, hitst, w, bt, rt, out_dtype=odt,
                                       dropout_p=p, dropout_seed=seed)
    g = msda.sca_camera_average(rbt, post, hitst).reshape(B * Nq, C).to(torch.bfloat16)
    y_split = msda.msda_linear(g, w, bt, rt, out_dtype=odt, dropout_p=p, dropout_seed=seed)
    torch.cuda.synchronize()
    assert msda.lib().msda_linear_timeouts() == timeouts0
    assert torch.equal(y.view(torch.int16 if out_bf16 else torch.int32),
                       y_split.view(torch.int16 if out_bf16 else torch.int32)), \
        "fused average differs from the split path"

    gb = oracle.round_bf16(oracle.sca_camera_average(rb, pos, hits).reshape(B * Nq, C))
    o = oracle.linear(gb, w32, b)
    mag = oracle.linear(np.abs(gb), np.abs(w32), np.abs(b) if b is not None else None)
    if p > 0:
        o = oracle.dropout(o, p, seed)
        mag = mag / (1.0 - p)
    ref = o + r if r is not None else o
    tol = 1e-6 + (2.0 ** -7 + (C + 2) * 2.0 ** -24) * mag
    if r is not None:
        tol = tol + 2.0 ** -24 * np.abs(r)
    if out_bf16:
        tol = tol + 2.0 ** -8 * np.abs(ref)
    got = y.float().cpu().numpy().astype(np.float64)
    err = np.abs(got - ref)
    worst = np.unravel_index(np.argmax(err - tol), err.shape)
    assert np.all(err <= tol), f"max err {err.max():.3e}; at worst {err[worst]:.3e} > {tol[worst]:.3e}"
    return y


def _mask(rng, Ncam, B, Nq, frac):
    m = (rng.random((Ncam, B, Nq, 1)) < frac).astype(np.uint8)
    m[:, 0, 0, :] = 0   # a query no camera sees
    m[:, 0, 1, :] = 1   # a query every camera sees
    return m


@pytest.mark.parametrize("B,Ncam,Nq,H,N,out_bf16,with_bias,with_res,p", [
    (1, 6, 320, 8, 256, False, True, True, 0.0),     # three tiles, ragged last one
    (2, 6, 930, 8, 512, True, True, False, 0.0),     # two W tiles, bf16 output
    (1, 8, 400, 4, 256, False, False, True, 0.1),    # eight cameras, K = 128, dropout
    (2, 3, 130, 2, 256, False, True, True, 0.3),     # K = 64, a 2-row last tile
    (1, 2, 128 * 148 * 2 + 5, 8, 256, False, True, True, 0.0),  # several tiles per CTA
])
def test_matches_split_path_and_oracle(B, Ncam, Nq, H, N, out_bf16, with_bias, with_res, p):
    rng = np.random.Generator(np.random.PCG64(B * 1000 + Ncam * 10 + H))
    mask = _mask(rng, Ncam, B, Nq, 0.35)
    rb = rng.standard_normal((B, Ncam, Nq, H * 32)).astype(np.float32)
    _run(mask, rb, N, out_bf16, with_bias, with_res, p, seed=Nq + Ncam)


def test_bevformer_base_size():
    """The BEVFormer-base output projection: 200 x 200 queries, six cameras,
    C = 256, camera masks from the workload's generator, bias and residual,
    with and without dropout."""
    rng = np.random.Generator(np.random.PCG64(81))
    B, Ncam, Nq, R, C = 1, 6, 200 * 200, 4, 256
    mask = inputs.sca_mask(rng, Ncam, B, Nq, R)
    rb = rng.standard_normal((B, Ncam, Nq, C)).astype(np.float32)
    _run(mask, rb, C, False, True, True, 0.0, seed=82)
    _run(mask, rb, C, False, True, True, 0.1, seed=83)


def test_unseen_queries_project_the_bias():
    """A query no camera sees averages to zero: its output is bias + residual."""
    rng = np.random.Generator(np.random.PCG64(84))
    B, Ncam, Nq, C = 1, 6, 200, 256
    mask = np.zeros((Ncam, B, Nq, 1), np.uint8)
    rb = rng.standard_normal((B, Ncam, Nq, C)).astype(np.float32)
    _, w = _bf16(rng.standard_normal((C, C)))
    bias = dev(rng.standard_normal(C).astype(np.float32))
    res = dev(rng.standard_normal((Nq, C)).astype(np.float32))
    _, _, pos, hits = oracle.sca_compact(mask)
    y = msda.sca_camera_average_linear(dev(rb), dev(pos), dev(hits), w, bias, res)
    torch.cuda.synchronize()
    assert torch.equal(y, res + bias[None, :])


def test_host_side_errors():
    """Sizes the kernel does not take are refused on the host (nothing is
    launched); an empty batch is a no-op."""
    def z(shape, dtype=torch.float32):
        return torch.zeros(shape, dtype=dtype, device="cuda")

    hits = z((1, 4), torch.int32)
    w = z((256, 256), torch.bfloat16)
    with pytest.raises(msda.MsdaError):   # nine cameras
        msda.sca_camera_average_linear(z((1, 9, 4, 256)), z((1, 9, 4), torch.int32), hits, w)
    pos6 = z((1, 6, 4), torch.int32)
    with pytest.raises(msda.MsdaError):   # H = 1: rows of 32 channels
        msda.sca_camera_average_linear(z((1, 6, 4, 32)), pos6, hits, z((256, 32), torch.bfloat16))
    with pytest.raises(msda.MsdaError):   # N = 128
        msda.sca_camera_average_linear(z((1, 6, 4, 256)), pos6, hits, z((128, 256), torch.bfloat16))
    empty = msda.sca_camera_average_linear(z((1, 6, 0, 256)), z((1, 6, 0), torch.int32),
                                           z((1, 0), torch.int32), w)
    torch.cuda.synchronize()
    assert empty.shape == (0, 256)
