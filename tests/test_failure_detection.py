"""Failure detection without a GPU fault: a bounded device wait that runs out.

The test build of the library (libarchead_testhooks.so, the same sources compiled with
ARCHEAD_TEST_HOOKS) lets one consumer warp of the decode kernel wait on an mbarrier that no
thread ever arrives on, with a short bound.  The wait gives up, the kernel sets
ARCHEAD_ERR_TIMEOUT in the device error word and finishes (its producer drains every bulk
copy it issued before the CTA exits), archead_check reports the status once, and the next
call on the same context is correct.  No fault, trap or unbounded wait is involved.
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

E = _lib.STATUS_CODE


def test_bounded_wait_timeout_is_reported_and_the_device_stays_usable(cuda_ok):
    T = _lib.testhooks_lib()
    dev = torch.device("cuda:0")
    head = random_canonical_head(1000, 512, 8, 8, 128, seed=31, super_exp_range=(-17, -13),
                                 factor_exp_range=(-13, -10))
    dh = ah.DeviceHead.from_canonical(head, dev)
    Hc = make_hidden(4, make_channel_scales(512, 0.5, 4, 20.0, 32), 33)
    H = Hc.to(dev)
    Y = torch.empty(4, head["V"], device=dev)
    st = torch.cuda.current_stream().cuda_stream

    def call():
        return T.archead_logits(H.data_ptr(), ctypes.byref(dh.struct), Y.data_ptr(), 4,
                                *dh.shape_args, st)

    assert T.archead_test_hooks(0, 0) == E["ARCHEAD_ERR_SHAPE"]
    try:
        # ~2^20 SM cycles (about half a millisecond) per wait; CTA 0's first consumer warp
        # waits on the barrier nothing completes
        assert T.archead_test_hooks(1 << 20, 0) == E["ARCHEAD_OK"]
        assert call() == E["ARCHEAD_OK"]  # the launch itself succeeds
        assert T.archead_check(st) == E["ARCHEAD_ERR_TIMEOUT"]
        assert T.archead_check(st) == E["ARCHEAD_OK"]  # the word was cleared
    finally:
        assert T.archead_test_hooks(1 << 31, -1) == E["ARCHEAD_OK"]
    # the same context, a normal call: correct logits, no error
    assert call() == E["ARCHEAD_OK"]
    assert T.archead_check(st) == E["ARCHEAD_OK"]
    Yref = oracle.logits(head, bf16_bits(Hc))
    err = np.max(np.abs(Y.cpu().double().numpy() - Yref))
    assert err <= 1e-2 * np.sqrt(np.mean(Yref ** 2))
    # and the product library on the same device
    Yp = ah.logits(H, dh)
    assert float((Yp - Y).abs().max()) <= 1e-5 * float(Y.abs().max())
    ah.check()
