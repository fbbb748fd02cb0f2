"""archead_logits_noalloc: the entry point for callers that cannot allocate device memory
(serving engines that reserve nearly all GPU memory for their own pool, decode loops
that must not enter an allocator).  It must give the same logits as archead_logits while
taking its temporaries from a fixed device array instead of allocating.

This file is collected last so that a run stopping at the first failure has already run
every other test; it also passes on its own in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

import packed_int4_lm_b200 as ah
from packed_int4_lm_b200 import _lib
from workloads import make_channel_scales, make_hidden, random_canonical_head

pytestmark = pytest.mark.gpu

LOGIT_TOL = 1e-2  # max |Y - Y_ref| <= LOGIT_TOL * rms(Y_ref), as in the other parity tests


def _noalloc(H, dh, Y):
    return _lib.lib().archead_logits_noalloc(
        H.data_ptr(), ctypes.byref(dh.struct), Y.data_ptr(), H.shape[0], *dh.shape_args,
        torch.cuda.current_stream().cuda_stream)


def test_noalloc_matches_allocating_entry_point_on_consecutive_calls(cuda_ok):
    dev = torch.device("cuda:0")
    head = random_canonical_head(1000, 512, 8, 8, 64, seed=21, zero_rows=2)
    dh = ah.DeviceHead.from_canonical(head, dev)
    s = make_channel_scales(512, 0.5, 4, 20.0, 22)
    # two calls in a row with different batch sizes: the second reuses the fixed array
    # that the first left filled
    for N in (40, 5):
        H = make_hidden(N, s, 23 + N).to(dev)
        Y_ref = ah.logits(H, dh)
        Y = torch.full((N, head["V"]), float("nan"), device=dev)
        assert _noalloc(H, dh, Y) == 0
        ah.check()
        a, b = Y.double().cpu().numpy(), Y_ref.double().cpu().numpy()
        rms = np.sqrt(np.mean(b ** 2))
        assert np.all(np.isfinite(a))
        assert np.max(np.abs(a - b)) <= LOGIT_TOL * rms


def test_noalloc_rejects_requests_beyond_its_scratch(cuda_ok):
    dev = torch.device("cuda:0")
    head = random_canonical_head(300, 4096, 32, 32, 128, seed=24)
    dh = ah.DeviceHead.from_canonical(head, dev)
    H = torch.zeros(256, 4096, dtype=torch.bfloat16, device=dev)  # FP16 copy alone is 2 MiB
    Y = torch.empty(256, 300, device=dev)
    assert _noalloc(H, dh, Y) == _lib.STATUS_CODE["ARCHEAD_ERR_SHAPE"]
    H = torch.zeros(192, 4096, dtype=torch.bfloat16, device=dev)     # fits
    Y = torch.empty(192, 300, device=dev)
    assert _noalloc(H, dh, Y) == 0
    ah.check()
