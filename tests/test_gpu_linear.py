"""msda_linear (the value / offset / weight / output projections on tcgen05
tensor cores) against the oracle's plain-loop projection, through the C ABI.

The inputs are bf16 (products exact in fp32) and the accumulation is fp32, so
the bound is derived from the arithmetic: for K products summed in fp32 in
any order, |error| <= K * 2^-24 * sum_k |x_k w_k| (plus the same for bias and
residual); a bf16 output adds half a bf16 ulp, at most 2^-8 |y| (an 8-bit
significand).  Ragged M checks the
zero-filled last tile; no pipeline wait may time out.
"""
import numpy as np
import pytest
import torch

import oracle
import scale_deformable_attention_03_b200 as msda
from scale_deformable_attention_03_b200 import inputs

pytestmark = pytest.mark.gpu


def _bf16(a):
    bits = inputs.to_bf16_bits(a)
    return inputs.bf16_bits_to_f32(bits), torch.from_numpy(bits.view(np.int16)).cuda().view(torch.bfloat16)


@pytest.mark.parametrize("M,N,K", [(1000, 256, 256), (129, 512, 256), (1, 256, 64),
                                   (300, 256, 192), (2048, 512, 128), (128, 256, 256)])
@pytest.mark.parametrize("with_bias,with_res", [(True, True), (False, False)])
@pytest.mark.parametrize("out_bf16", [False, True])
def test_linear_matches_oracle(M, N, K, with_bias, with_res, out_bf16):
    timeouts0 = msda.lib().msda_linear_timeouts()
    rng = np.random.Generator(np.random.PCG64(M * 7 + N + K))
    x32, x = _bf16(rng.standard_normal((M, K)).astype(np.float32))
    w32, w = _bf16((rng.standard_normal((N, K)) / np.sqrt(K)).astype(np.float32))
    b = rng.standard_normal(N).astype(np.float32) if with_bias else None
    r = rng.standard_normal((M, N)).astype(np.float32) if with_res else None
    y = msda.msda_linear(x, w, torch.from_numpy(b).cuda() if b is not None else None,
                         torch.from_numpy(r).cuda() if r is not None else None,
                         out_dtype=torch.bfloat16 if out_bf16 else torch.float32)
    torch.cuda.synchronize()
    ref = oracle.linear(x32, w32, b, r)
    mag = oracle.linear(np.abs(x32), np.abs(w32), np.abs(b) if b is not None else None,
                        np.abs(r) if r is not None else None)
    tol = 1e-6 + (K + 2) * 2.0 ** -24 * mag
    if out_bf16:
        tol = tol + 2.0 ** -8 * np.abs(ref)
    got = y.float().cpu().numpy().astype(np.float64)
    err = np.abs(got - ref)
    assert np.all(err <= tol), f"max err {err.max():.3e} (tol at worst {tol[np.unravel_index(np.argmax(err - tol), err.shape)]:.3e})"
    assert msda.lib().msda_linear_timeouts() == timeouts0


@pytest.mark.parametrize("M,N,K,out_bf16", [
    (148 * 128 * 3 + 77, 256, 256, False),   # several tiles per CTA, ragged last tile
    (40000, 512, 256, True),                 # the offset head: a W-tile switch per CTA
    (9000, 768, 64, False),                  # three W tiles, one K block
])
def test_linear_persistent_tiles(M, N, K, out_bf16):
    """Many tiles per CTA: the X ring and both TMEM accumulators wrap many
    times and the W tile is reloaded when a CTA's tiles move to a new N-tile."""
    timeouts0 = msda.lib().msda_linear_timeouts()
    rng = np.random.Generator(np.random.PCG64(M + N + K))
    x32, x = _bf16(rng.standard_normal((M, K)).astype(np.float32))
    w32, w = _bf16((rng.standard_normal((N, K)) / np.sqrt(K)).astype(np.float32))
    b = rng.standard_normal(N).astype(np.float32)
    r = rng.standard_normal((M, N)).astype(np.float32)
    y = msda.msda_linear(x, w, torch.from_numpy(b).cuda(), torch.from_numpy(r).cuda(),
                         out_dtype=torch.bfloat16 if out_bf16 else torch.float32)
    torch.cuda.synchronize()
    ref = oracle.linear(x32, w32, b, r)
    mag = np.abs(x32) @ np.abs(w32).T + np.abs(b) + np.abs(r)
    tol = 1e-6 + (K + 2) * 2.0 ** -24 * mag
    if out_bf16:
        tol = tol + 2.0 ** -8 * np.abs(ref)
    err = np.abs(y.float().cpu().numpy().astype(np.float64) - ref)
    assert np.all(err <= tol), f"max err {err.max():.3e}"
    assert msda.lib().msda_linear_timeouts() == timeouts0


def test_linear_identity_reproduces_input():
    """W = I (N = K = 256): the projection returns x exactly (fp32 output)."""
    rng = np.random.Generator(np.random.PCG64(5))
    x32, x = _bf16(rng.standard_normal((333, 256)).astype(np.float32))
    _, w = _bf16(np.eye(256, dtype=np.float32))
    y = msda.msda_linear(x, w)
    torch.cuda.synchronize()
    assert np.array_equal(y.cpu().numpy(), x32)


@pytest.mark.parametrize("p,seed,out_bf16", [(0.1, 7, False), (0.5, (3 << 40) | 11, False),
                                             (0.25, 99, True)])
def test_linear_dropout_matches_oracle(p, seed, out_bf16):
    """Training-time dropout in the epilogue: y = r + dropout(x w^T + b).  The
    mask is the same Philox4x32-10 draw on both sides, so any mask difference
    fails by the size of a value; the bound is the fp32 one scaled by
    1 / (1 - p) plus one fp32 rounding of the scaling."""
    M, N, K = 3000, 512, 128
    rng = np.random.Generator(np.random.PCG64(31))
    x32, x = _bf16(rng.standard_normal((M, K)).astype(np.float32))
    w32, w = _bf16((rng.standard_normal((N, K)) / np.sqrt(K)).astype(np.float32))
    b = rng.standard_normal(N).astype(np.float32)
    r = rng.standard_normal((M, N)).astype(np.float32)
    y = msda.msda_linear(x, w, torch.from_numpy(b).cuda(), torch.from_numpy(r).cuda(),
                         out_dtype=torch.bfloat16 if out_bf16 else torch.float32,
                         dropout_p=p, dropout_seed=seed)
    torch.cuda.synchronize()
    o = oracle.linear(x32, w32, b)
    ref = r + oracle.dropout(o, p, seed)
    mag = np.abs(x32) @ np.abs(w32).T + np.abs(b)
    tol = 1e-6 + (K + 2) * 2.0 ** -24 * mag / (1 - p) + 2.0 ** -23 * np.abs(o) / (1 - p)
    if out_bf16:
        tol = tol + 2.0 ** -8 * np.abs(ref)
    err = np.abs(y.float().cpu().numpy().astype(np.float64) - ref)
    assert np.all(err <= tol), f"max err {err.max():.3e}"
    kept = np.count_nonzero(oracle.dropout(np.ones(M * N), p, seed))
    assert abs(kept - M * N * (1 - p)) < 5 * np.sqrt(M * N * p * (1 - p))
