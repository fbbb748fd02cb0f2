"""archead_logits_host with the vocabulary in chunks: each chunk's logits go to the host on
a second stream while the next chunks are evaluated.  Every chunk is a head view of its own
(the row arrays advanced by a multiple of 128 rows), so the test covers the views of both
formats, the strided copies into the host matrix, a ragged last chunk and each main kernel
(the decode kernel, the tcgen05 kernel with one split token tile and with several token
tiles, and the warp-MMA kernel of the Row INT8 format).  The host result is checked against
the fp64 oracle (max |Y - Y_ref| <= 1e-2 rms(Y_ref)) and against the device entry point
(1e-4 max |Y|: the kernels split their work by the row count, so the FP32 sums of a chunk and
of the whole head may round differently).
"""
import numpy as np
import pytest
import torch

import oracle
import packed_int4_lm_b200 as ah
from packed_int4_lm_b200 import _lib
from workloads import bf16_bits, make_channel_scales, make_hidden, random_canonical_head

pytestmark = pytest.mark.gpu

LOGIT_TOL = 1e-2


def _chunks(N, V):
    """The chunk count the library uses: about 3 MB of logits per chunk, at most 8 chunks of
    a multiple of 128 rows, none below 2 chunks or for V < 256."""
    c = min(8, (N * V * 4) // (3 << 20))
    if c < 2 or V < 256:
        return 1
    per_chunk = -(-V // c)
    rows = -(-per_chunk // 128) * 128
    return -(-V // rows)


def _row8_head(V, D, seed):
    rng = np.random.default_rng(seed)
    return {"format": "row8", "V": V, "D": D, "r_c": 0, "r_r": 0, "g": 128,
            "q8": rng.integers(-127, 128, size=(V, D)).astype(np.int8),
            "row_scale": (2.0 ** rng.uniform(-13, -11, size=V)).astype(np.float32)}


@pytest.fixture(scope="module")
def dev(cuda_ok):
    return torch.device("cuda:0")


@pytest.fixture(scope="module")
def big_head(dev):
    head = random_canonical_head(100000, 256, 16, 16, 128, seed=5, zero_rows=2,
                                 super_exp_range=(-17, -13), factor_exp_range=(-13, -10))
    return head, ah.DeviceHead.from_canonical(head, dev)


def _check(head, dh, N, seed, dev):
    Hc = make_hidden(N, make_channel_scales(head["D"], 0.5, 4, 20.0, seed), seed + 1)
    Yd = ah.logits(Hc.to(dev), dh)
    ah.check()
    Yh = ah.logits_host(Hc.pin_memory(), dh)
    ah.check()
    n_chunks = _chunks(N, head["V"])
    assert n_chunks >= 2
    assert _lib.lib().archead_last_launches() >= 2 * n_chunks  # a prologue and a main kernel each
    Yref = oracle.logits(head, bf16_bits(Hc))
    Y = Yh.double().numpy()
    rms = np.sqrt(np.mean(Yref ** 2))
    assert np.all(np.isfinite(Y))
    assert np.max(np.abs(Y - Yref)) <= LOGIT_TOL * rms
    Yd = Yd.cpu().double().numpy()
    assert np.max(np.abs(Y - Yd)) <= 1e-4 * np.max(np.abs(Yd))


@pytest.mark.parametrize("N,path", [(16, "decode kernel, 2 chunks"),
                                    (40, "tcgen05 kernel, one split token tile, 5 chunks"),
                                    (200, "tcgen05 kernel, two token tiles, 8 chunks")])
def test_host_chunks_match_oracle(dev, big_head, N, path):
    head, dh = big_head
    _check(head, dh, N, 60 + N, dev)


def test_host_chunks_row8(dev):
    head = _row8_head(40000, 256, seed=9)
    dh = ah.DeviceHead.from_canonical(head, dev)
    _check(head, dh, 64, 70, dev)


def test_host_single_chunk_below_threshold(dev, big_head):
    """Small outputs take one call and one copy (no second stream)."""
    head, dh = big_head
    assert _chunks(4, head["V"]) == 1
    Hc = make_hidden(4, make_channel_scales(256, 0.5, 4, 20.0, 3), 4)
    Yd = ah.logits(Hc.to(dev), dh).cpu()
    per_call = _lib.lib().archead_last_launches()
    Yh = ah.logits_host(Hc.pin_memory(), dh)
    ah.check()
    assert _lib.lib().archead_last_launches() == per_call
    assert torch.equal(Yd, Yh)
