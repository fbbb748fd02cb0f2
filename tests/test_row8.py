"""The Row INT8 baseline head (ARCHead Sec. 5: the storage-matched comparison of Tables 3
and 8, "Row INT8 remains more accurate, but uses approximately twice the head storage") on
the library's warp-MMA kernel, against the fp64 oracle: logits within 1e-2 rms, NLL and
agreement within 1e-3 nats, for arbitrary INT8 bytes and for a head built from a dense W."""
import numpy as np
import pytest
import torch

import oracle
import packed_int4_lm_b200 as ah
from packed_int4_lm_b200 import pack
from workloads import bf16_bits, make_channel_scales, make_hidden, make_targets, make_weight

LOGIT_TOL, NLL_TOL = 1e-2, 1e-3


def _row8_head(V, D, seed):
    rng = np.random.default_rng(seed)
    return {"format": "row8", "V": V, "D": D, "r_c": 0, "r_r": 0, "g": 128,
            "q8": rng.integers(-127, 128, size=(V, D)).astype(np.int8),
            "row_scale": (2.0 ** rng.uniform(-13, -11, size=V)).astype(np.float32)}


def test_row8_storage_is_about_twice_the_packed_head():
    W = make_weight(512, 1024, 16, 0.5, 0.02, seed=1)
    r8 = pack.build_row8_head(W)
    assert abs(pack.storage_ratio(r8) - (0.5 + 2.0 / 1024)) < 1e-12
    assert np.array_equal(r8["q8"].astype(np.int64).clip(-127, 127), r8["q8"].astype(np.int64))
    err = np.abs(oracle.dense_head_rows(r8) - W.double().numpy()).max(axis=1)
    assert np.all(err <= r8["row_scale"].astype(np.float64) / 2 + 1e-12)  # half a step


@pytest.mark.gpu
@pytest.mark.parametrize("N", [1, 9, 40, 130])
def test_row8_logits_and_nll_match_oracle(cuda_ok, N):
    dev = torch.device("cuda:0")
    head = _row8_head(1000, 512, seed=3)
    dh = ah.DeviceHead.from_canonical(head, dev)
    Hc = make_hidden(N, make_channel_scales(512, 0.5, 4, 20.0, 4), 5 + N)
    Y = ah.logits(Hc.to(dev), dh)
    ah.check()
    Yref = oracle.logits(head, bf16_bits(Hc))
    rms = np.sqrt(np.mean(Yref ** 2))
    assert 0.5 < rms < 20  # the logit regime
    assert np.max(np.abs(Y.cpu().double().numpy() - Yref)) <= LOGIT_TOL * rms
    tg = make_targets(N, 1000, 6 + N)
    nl = ah.nll(Hc.to(dev), dh, tg.to(dev))
    ah.check()
    assert np.max(np.abs(nl.cpu().double().numpy() - oracle.nll_from_logits(Yref, tg.numpy()))) <= NLL_TOL


@pytest.mark.gpu
def test_row8_built_head_and_agreement(cuda_ok):
    dev = torch.device("cuda:0")
    W = make_weight(700, 1024, 32, 0.5, 0.02, seed=7)
    head = pack.build_row8_head(W)
    dh = ah.DeviceHead.from_canonical(head, dev)
    Hc = make_hidden(12, make_channel_scales(1024, 0.5, 4, 20.0, 8), 9)
    Yref = oracle.logits(head, bf16_bits(Hc))
    Y = ah.logits(Hc.to(dev), dh)
    ah.check()
    assert np.max(np.abs(Y.cpu().double().numpy() - Yref)) <= LOGIT_TOL * np.sqrt(np.mean(Yref ** 2))
    yd = (Hc.double() @ W.double().t()).float().numpy()  # the dense head's own logits
    got = ah.agreement(Hc.to(dev), dh, torch.from_numpy(yd).to(dev), 5)
    ah.check()
    ref = oracle.agreement(head, bf16_bits(Hc), yd, 5)
    assert np.array_equal(got["top1_dense"].cpu().numpy(), ref["top1_dense"])
    assert np.max(np.abs(got["kl"].cpu().numpy() - ref["kl"])) <= NLL_TOL
    # the dequant hook reads the packed layout only
    with pytest.raises(ah.ArcheadError):
        ah.dequant(dh)
