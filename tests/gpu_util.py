"""Helpers shared by the GPU parity tests: device copies of workloads and the
element-wise tolerance checks.

Tolerances: fp32 value |gpu - oracle| <= 1e-5 + 1e-5 |oracle|; bf16 value
(fp32 arithmetic) |gpu - oracle| <= 2e-2, the oracle reading the same
bf16-rounded values.  Integer outputs must be equal.
"""
import numpy as np
import torch

import oracle

F32_ATOL = 1e-5
F32_RTOL = 1e-5
BF16_ATOL = 2e-2


def dev(a, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.to(dtype)
    return t.cuda()


def value_tensor(w, bf16):
    """The workload's value on the device: bf16 bits when asked (the oracle
    then reads w.value, the same values widened to fp32)."""
    if bf16:
        bits = w.value_bf16
        assert bits is not None
        return dev(bits.view(np.int16)).view(torch.bfloat16)
    return dev(w.value)


def assert_close(gpu, ref, bf16=False, what=""):
    g = gpu.detach().cpu().numpy().astype(np.float64) if isinstance(gpu, torch.Tensor) else gpu
    r = np.asarray(ref, dtype=np.float64)
    assert g.shape == r.shape, (what, g.shape, r.shape)
    err = np.abs(g - r)
    tol = BF16_ATOL + 0 * r if bf16 else F32_ATOL + F32_RTOL * np.abs(r)
    bad = ~(err <= tol)
    if bad.any():
        i = np.unravel_index(np.argmax(np.where(bad, err - tol, -np.inf)), r.shape)
        raise AssertionError(
            f"{what}: {int(bad.sum())} of {r.size} elements out of tolerance; worst at {i}: "
            f"gpu={g[i]!r} oracle={r[i]!r} err={err[i]:.3e}; max err {err.max():.3e}")
    return float(err.max()) if err.size else 0.0


def softmax_weights(logits, axis_len):
    """Attention weights for msda_forward: the oracle's softmax, stored fp32."""
    return oracle.softmax(logits, axis_len).reshape(logits.shape).astype(np.float32)
