"""sca_compact_no_alloc: the mask compaction for callers that cannot allocate
device memory (their framework owns all device memory and gives this step no
scratch, or their pipeline forbids allocation while it runs).  It keeps its
scratch in a fixed array inside the library and takes no workspace.

The test calls it through the C ABI, twice in a row on the same stream (the
second call finds the first call's counts in the shared array), and checks
each result against sca_compact, bit for bit, the bar every compaction test
here uses.  It also checks that a problem larger than the fixed array is
refused with a message.  This file is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

import scale_deformable_attention_03_b200 as msda
from scale_deformable_attention_03_b200 import inputs

pytestmark = pytest.mark.gpu

UNSUPPORTED = 2


def _entry():
    f = msda.lib().sca_compact_no_alloc
    f.argtypes = [ctypes.c_void_p, msda.Dims] + [ctypes.c_void_p] * 5
    f.restype = ctypes.c_int
    return f


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr())


def _call_no_alloc(mask):
    Ncam, B, Nq, R = mask.shape
    # outputs start as garbage: the call must overwrite all of them
    idx = torch.full((B, Ncam, Nq), 12345, dtype=torch.int32, device="cuda")
    count = torch.full((B, Ncam), -7, dtype=torch.int32, device="cuda")
    pos = torch.full((B, Ncam, Nq), 999, dtype=torch.int32, device="cuda")
    hits = torch.full((B, Nq), 77, dtype=torch.int32, device="cuda")
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    st = _entry()(_ptr(mask), msda.Dims(B, Ncam, Nq, 1, 1, 1, 1, R), _ptr(idx), _ptr(count),
                  _ptr(pos), _ptr(hits), stream)
    assert st == 0, msda.lib().msda_last_error().decode()
    return idx, count, pos, hits


def _masks():
    rng = np.random.Generator(np.random.PCG64(91))
    yield "bevformer-base", inputs.workload3().bev_mask
    yield "random-ragged", (rng.random((5, 2, 4097, 3)) < 0.2).astype(np.uint8)
    yield "tiny", (rng.random((1, 1, 31, 2)) < 0.5).astype(np.uint8)


@pytest.mark.parametrize("name,mask", list(_masks()), ids=[m[0] for m in _masks()])
def test_matches_sca_compact_on_two_calls_in_a_row(name, mask):
    m = torch.from_numpy(np.ascontiguousarray(mask)).cuda()
    want = msda.sca_compact(m)
    torch.cuda.synchronize()
    for _ in range(2):
        got = _call_no_alloc(m)
        torch.cuda.synchronize()
        for label, g, w in zip(("idx", "count", "pos", "hits"), got, want):
            assert torch.equal(g, w), f"{name}: {label} differs from sca_compact"


def test_refuses_problems_beyond_the_fixed_array():
    # B * Ncam * ceil(Nq / 1024) = 8 * 8 * 1025 = 65600 > 65536 count slots;
    # the call must refuse before touching any pointer
    d = msda.Dims(8, 8, 1024 * 1025, 1, 1, 1, 1, 4)
    fake = ctypes.c_void_p(0x7F0000000000)
    st = _entry()(fake, d, fake, fake, fake, fake, None)
    assert st == UNSUPPORTED
    assert b"count slots" in msda.lib().msda_last_error()
