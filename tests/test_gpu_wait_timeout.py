"""The bounded-wait path of the tensor-core projection (msda_linear), made to
run out on purpose: msda_linear_test_withhold_load makes the next launch hold
back one X-tile load of its first CTA (a barrier that nothing completes), so
that CTA's tensor-core wait gives up after its limit, counts a timeout, stops
its other roles, waits for the copies it did issue and frees its tensor
memory.  The call must return, the counter must rise by one, and the next
normal call must be exact again (the GPU context stays usable)."""
import numpy as np
import pytest
import torch

import oracle
import scale_deformable_attention_03_b200 as msda
from scale_deformable_attention_03_b200 import inputs

pytestmark = pytest.mark.gpu


def _bf16(a):
    bits = inputs.to_bf16_bits(a)
    return (inputs.bf16_bits_to_f32(bits),
            torch.from_numpy(bits.view(np.int16)).cuda().view(torch.bfloat16))


def test_withheld_load_times_out_and_the_next_call_is_exact():
    rng = np.random.Generator(np.random.PCG64(404))
    M, N, K = 1000, 256, 256
    x32, x = _bf16(rng.standard_normal((M, K)).astype(np.float32))
    w32, w = _bf16((rng.standard_normal((N, K)) / np.sqrt(K)).astype(np.float32))
    b = rng.standard_normal(N).astype(np.float32)
    bias = torch.from_numpy(b).cuda()
    L = msda.lib()
    before = L.msda_linear_timeouts()
    assert L.msda_linear_test_withhold_load() == 0
    msda.msda_linear(x, w, bias)          # the launch whose first CTA gives up
    torch.cuda.synchronize()
    assert L.msda_linear_timeouts() == before + 1
    y = msda.msda_linear(x, w, bias)      # a normal call afterwards
    torch.cuda.synchronize()
    assert L.msda_linear_timeouts() == before + 1
    ref = oracle.linear(x32, w32, b)
    mag = oracle.linear(np.abs(x32), np.abs(w32), np.abs(b))
    err = np.abs(y.cpu().numpy().astype(np.float64) - ref)
    assert np.all(err <= 1e-6 + (K + 2) * 2.0 ** -24 * mag), err.max()
