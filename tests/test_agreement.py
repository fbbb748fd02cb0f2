"""Agreement of the packed head with a dense reference head (ARCHead Sec. 5, Table 8 and
the paragraph on it: the dense top-1 token kept among the packed head's top k, and the
KL divergence), through archead_agreement, against the fp64 oracle.

What is unique is compared exactly: the dense argmax (from the same float32 dense logits
on both sides).  KL and the packed log-sum-exp are compared within 1e-3 nats in the logit
regime.  The packed top-k ids depend on packed logits that the GPU evaluates within its
own rounding, so near-ties may order differently: every GPU id must be a valid choice,
i.e. its oracle logit lies within 2 e of the oracle's value at that rank, where e is the
largest |Y_gpu - Y_oracle| of the same call, and ids are unique; without near-ties the
lists must be equal.
"""
import numpy as np
import pytest
import torch

import oracle
import packed_int4_lm_b200 as ah
from workloads import bf16_bits, make_channel_scales, make_hidden, random_canonical_head

pytestmark = pytest.mark.gpu

TOL = 1e-3  # nats


def _head(V, D, g, seed):
    return random_canonical_head(V, D, 8, 8, g, seed=seed, zero_rows=3, zero_groups=20,
                                 super_exp_range=(-17, -13), factor_exp_range=(-13, -10))


def _check(head, dh, Hc, yd, k, dev):
    H = Hc.to(dev)
    got = ah.agreement(H, dh, torch.from_numpy(yd).to(dev), k)
    ah.check()
    got = {x: v.cpu().numpy() for x, v in got.items()}
    ref = oracle.agreement(head, bf16_bits(Hc), yd.astype(np.float64), k)
    Yg = ah.logits(H, dh).cpu().double().numpy()
    e = float(np.max(np.abs(Yg - ref["y_packed"])))
    assert np.array_equal(got["top1_dense"], ref["top1_dense"])
    assert np.max(np.abs(got["kl"] - ref["kl"])) <= TOL
    assert np.max(np.abs(got["lse"] - ref["lse"])) <= TOL
    yp = ref["y_packed"]
    for n in range(yp.shape[0]):
        ids, rid = got["topk"][n], ref["topk"][n]
        valid = rid >= 0
        assert np.array_equal(ids[~valid], rid[~valid])          # -1 past V
        ids, rid = ids[valid], rid[valid]
        assert len(set(ids.tolist())) == len(ids)                 # unique
        assert np.all((ids >= 0) & (ids < head["V"]))
        # each GPU pick is a valid choice at its rank
        assert np.all(np.abs(yp[n, ids] - yp[n, rid]) <= 2 * e + 1e-9), (n, ids, rid)
        s = np.sort(yp[n])[::-1]
        gaps = np.diff(s[:len(rid) + 1]) if len(s) > len(rid) else np.diff(s)
        if len(gaps) and np.all(np.abs(gaps) > 2 * e + 1e-9):
            assert np.array_equal(ids, rid)
    return got, ref


@pytest.mark.parametrize("N,k", [(1, 10), (7, 5), (40, 16), (130, 1)])
def test_agreement_matches_oracle(cuda_ok, N, k):
    dev = torch.device("cuda:0")
    head = _head(1000, 512, 64, seed=90)
    dh = ah.DeviceHead.from_canonical(head, dev)
    Hc = make_hidden(N, make_channel_scales(512, 0.5, 4, 20.0, 91), 92 + N)
    # a dense reference close to the packed head: its fp64 logits plus noise, in float32
    rng = np.random.default_rng(N)
    yd = (oracle.logits(head, bf16_bits(Hc)) + rng.normal(scale=0.2, size=(N, 1000))).astype(np.float32)
    got, ref = _check(head, dh, Hc, yd, k, dev)
    assert np.all(got["kl"] > -TOL)  # FP32 cancellation may round a tiny KL to 0


def test_agreement_g128_and_short_vocabulary(cuda_ok):
    """g = 128 (one code per 128 columns) and a vocabulary shorter than k: ids -1 past V."""
    dev = torch.device("cuda:0")
    for V, k in ((300, 10), (10, 16)):
        head = _head(V, 1024, 128, seed=V)
        dh = ah.DeviceHead.from_canonical(head, dev)
        Hc = make_hidden(9, make_channel_scales(1024, 0.5, 4, 20.0, 5), 6)
        yd = (oracle.logits(head, bf16_bits(Hc)) * 1.1).astype(np.float32)
        _check(head, dh, Hc, yd, k, dev)


def test_agreement_ties_take_the_smaller_id(cuda_ok):
    """An all-zero head gives equal packed logits everywhere: the top-k is 0..k-1, the dense
    argmax of equal values is 0, and KL against equal dense logits is 0."""
    dev = torch.device("cuda:0")
    head = random_canonical_head(500, 256, 0, 0, 64, seed=7)
    head["r_super"][:] = 0
    dh = ah.DeviceHead.from_canonical(head, dev)
    H = make_hidden(5, make_channel_scales(256, 0.5, 4, 20.0, 8), 9).to(dev)
    got = ah.agreement(H, dh, torch.zeros(5, 500, device=dev), 12)
    ah.check()
    assert torch.equal(got["topk"].cpu(), torch.arange(12, dtype=torch.int32).repeat(5, 1))
    assert torch.equal(got["top1_dense"].cpu(), torch.zeros(5, dtype=torch.int32))
    assert float(got["kl"].abs().max()) <= 1e-6
    assert torch.allclose(got["lse"].cpu(), torch.full((5,), float(np.log(500))), atol=1e-5)
