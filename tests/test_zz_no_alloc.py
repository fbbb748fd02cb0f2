"""archead_logits_noalloc: the entry point for callers that cannot allocate device memory
(serving engines that reserve nearly all GPU memory for their own pool, decode loops
that must not enter an allocator).  It must give the logits of the ARCHead formula, as
archead_logits does, while taking its temporaries from a fixed device array instead of
allocating.  The reference here is the fp64 CPU oracle, at the tolerance of the other
parity tests; the allocating entry point is compared as well.

This file is collected last so that a run stopping at the first failure has already run
every other test; it also passes on its own in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import packed_int4_lm_b200 as ah
from packed_int4_lm_b200 import _lib
from workloads import bf16_bits, make_channel_scales, make_hidden, random_canonical_head

pytestmark = pytest.mark.gpu

LOGIT_TOL = 1e-2  # max |Y - Y_ref| <= LOGIT_TOL * rms(Y_ref), as in the other parity tests


def _noalloc(H, dh, Y):
    return _lib.lib().archead_logits_noalloc(
        H.data_ptr(), ctypes.byref(dh.struct), Y.data_ptr(), H.shape[0], *dh.shape_args,
        torch.cuda.current_stream().cuda_stream)


def _assert_close(Y, Yref, what):
    Y = np.asarray(Y, dtype=np.float64)
    rms = np.sqrt(np.mean(Yref ** 2))
    assert np.all(np.isfinite(Y)), what
    err = np.max(np.abs(Y - Yref))
    assert err <= LOGIT_TOL * rms, f"{what}: {err:.3e} > {LOGIT_TOL} * {rms:.3e}"


def test_noalloc_matches_oracle_on_consecutive_calls(cuda_ok):
    dev = torch.device("cuda:0")
    head = random_canonical_head(1000, 512, 8, 8, 64, seed=21, zero_rows=2)
    dh = ah.DeviceHead.from_canonical(head, dev)
    s = make_channel_scales(512, 0.5, 4, 20.0, 22)
    # two calls in a row with different batch sizes: the second reuses the fixed array
    # that the first left filled
    for N in (40, 5):
        Hc = make_hidden(N, s, 23 + N)
        H = Hc.to(dev)
        Y = torch.full((N, head["V"]), float("nan"), device=dev)
        assert _noalloc(H, dh, Y) == 0
        ah.check()
        Yref = oracle.logits(head, bf16_bits(Hc))
        _assert_close(Y.cpu().numpy(), Yref, f"noalloc N={N} vs oracle")
        _assert_close(ah.logits(H, dh).cpu().numpy(), Yref, f"logits N={N} vs oracle")


def test_noalloc_allocates_no_device_memory(cuda_ok):
    dev = torch.device("cuda:0")
    head = random_canonical_head(700, 512, 8, 8, 64, seed=25)
    dh = ah.DeviceHead.from_canonical(head, dev)
    H = make_hidden(24, make_channel_scales(512, 0.5, 4, 20.0, 26), 27).to(dev)
    Y = torch.empty(24, head["V"], device=dev)
    assert _noalloc(H, dh, Y) == 0  # warm-up: module loading happens on the first launch
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info(dev)[0]
    for _ in range(3):
        assert _noalloc(H, dh, Y) == 0
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info(dev)[0] == free0
    ah.check()


def test_noalloc_limit_and_beyond(cuda_ok):
    dev = torch.device("cuda:0")
    head = random_canonical_head(300, 4096, 32, 32, 128, seed=24, super_exp_range=(-17, -13),
                                 factor_exp_range=(-13, -10))
    dh = ah.DeviceHead.from_canonical(head, dev)
    H = torch.zeros(256, 4096, dtype=torch.bfloat16, device=dev)  # FP16 copy alone is 2 MiB
    Y = torch.empty(256, 300, device=dev)
    assert _noalloc(H, dh, Y) == _lib.STATUS_CODE["ARCHEAD_ERR_SHAPE"]
    # the largest batch that fits (D = 4096, r_c + r_r = 64): values against the oracle
    Hc = make_hidden(192, make_channel_scales(4096, 0.5, 4, 20.0, 28), 29)
    Y = torch.full((192, 300), float("nan"), device=dev)
    assert _noalloc(Hc.to(dev), dh, Y) == 0
    ah.check()
    _assert_close(Y.cpu().numpy(), oracle.logits(head, bf16_bits(Hc)), "noalloc N=192")
