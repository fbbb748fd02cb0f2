"""Vocabulary-parallel NLL: every GPU holds a row shard of the head, reduces it to
(max, sum exp, target logit) per token, one all-gather exchanges those triples and each rank
merges them (ARCHead Sec. 5 cross-entropy, split over the vocabulary).

CPU: the row-shard helper against the oracle, and the two-rank protocol on gloo with the
two library calls replaced by fp64 test doubles.  GPU: the shard partials and the merge
through the library against the oracle on the whole head, and two gloo ranks (processes
sharing the GPU, host all-gather) running the real library calls."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
import packed_int4_lm_b200 as ah
from packed_int4_lm_b200.pack import shard_rows
from workloads import bf16_bits, make_channel_scales, make_hidden, make_targets, random_canonical_head

NLL_TOL = 1e-3  # nats
SHARDS = ((0, 300), (300, 700), (700, 1000))


def _head():
    # logit regime (rms of a few units), where a bound in nats is meaningful
    return random_canonical_head(1000, 512, 8, 8, 64, seed=21, zero_rows=3,
                                 super_exp_range=(-17, -13), factor_exp_range=(-13, -10))


def _H(N, seed):
    return make_hidden(N, make_channel_scales(512, 0.5, 4, 20.0, seed), seed + 1)


def test_shard_rows_logits_are_column_slices():
    head = _head()
    H = bf16_bits(_H(6, 3))
    Y = oracle.logits(head, H)
    for v0, v1 in SHARDS:
        sh = shard_rows(head, v0, v1)
        assert sh["V"] == v1 - v0
        # the same fp64 dot products (BLAS may sum in another order for another shape)
        assert np.allclose(oracle.logits(sh, H), Y[:, v0:v1], rtol=1e-12, atol=1e-12)
    with pytest.raises(ValueError):
        shard_rows(head, 500, 500)


class _ShardDouble:
    """Test double of a device head: the canonical shard, evaluated by the fp64 oracle."""

    def __init__(self, head):
        self.head = head


def _partials_double(H, dh, targets, v_begin, v_total):
    Y = oracle.logits(dh.head, bf16_bits(H))
    m = Y.max(axis=1)
    s = np.exp(Y - m[:, None]).sum(axis=1)
    t = targets.numpy().astype(np.int64) - v_begin
    own = (t >= 0) & (t < Y.shape[1])
    y = np.where(own, Y[np.arange(len(t)), np.clip(t, 0, Y.shape[1] - 1)], 0.0)
    return torch.from_numpy(np.stack([m, s, y], axis=1))


def _merge_double(partials):
    p = partials.numpy()
    M = p[:, :, 0].max(axis=0)
    S = (p[:, :, 1] * np.exp(p[:, :, 0] - M[None, :])).sum(axis=0)
    return torch.from_numpy(M + np.log(S) - p[:, :, 2].sum(axis=0))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ah.nll_partials = _partials_double
        ah.nll_merge = _merge_double
        head = _head()
        bounds = ((0, 450), (450, 1000))
        v0, v1 = bounds[rank]
        H = _H(9, 5)
        tg = make_targets(9, 1000, 6)
        nll = ah.vocab_parallel_nll(H, _ShardDouble(shard_rows(head, v0, v1)), tg, v0, 1000)
        out[rank] = nll.numpy().tolist()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_vocab_parallel_nll():
    world, port = 2, _free_port()
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        mp.spawn(_rank, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    head = _head()
    ref = oracle.nll(head, bf16_bits(_H(9, 5)), make_targets(9, 1000, 6).numpy())
    for r in range(world):
        assert np.allclose(res[r], ref, rtol=0, atol=1e-9)


@pytest.mark.gpu
@pytest.mark.parametrize("N", [5, 40, 130])
def test_shard_partials_and_merge_match_oracle(cuda_ok, N):
    dev = torch.device("cuda:0")
    head = _head()
    H = _H(N, 7 + N)
    tg = make_targets(N, 1000, 8 + N)
    Hd, tgd = H.to(dev), tg.to(dev)
    parts = []
    for v0, v1 in SHARDS:
        dh = ah.DeviceHead.from_canonical(shard_rows(head, v0, v1), dev)
        parts.append(ah.nll_partials(Hd, dh, tgd, v0, 1000))
        ah.check()
    nll = ah.nll_merge(torch.stack(parts))
    ah.check()
    ref = oracle.nll(head, bf16_bits(H), tg.numpy())
    err = np.max(np.abs(nll.cpu().double().numpy() - ref))
    assert err <= NLL_TOL, err
    # the target logit comes from exactly one shard
    owned = torch.stack(parts)[:, :, 2].ne(0).sum(dim=0)
    assert int(owned.max()) <= 1


def _rank_lib(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        dev = torch.device("cuda:0")
        head = _head()
        v0, v1 = ((0, 450), (450, 1000))[rank]
        dh = ah.DeviceHead.from_canonical(shard_rows(head, v0, v1), dev)
        H = _H(9, 5).to(dev)
        tg = make_targets(9, 1000, 6).to(dev)
        nll = ah.vocab_parallel_nll(H, dh, tg, v0, 1000)
        ah.check()
        out[rank] = nll.cpu().double().numpy().tolist()
    finally:
        dist.destroy_process_group()


@pytest.mark.gpu
def test_two_gloo_ranks_with_library_partials(cuda_ok):
    """The exchange of vocab_parallel_nll with the library's own partials and merge: two
    ranks (processes on the same GPU, gloo all-gather through host memory) each hold half
    of the rows; both must return the whole head's NLL, identical on the two ranks."""
    world, port = 2, _free_port()
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        mp.spawn(_rank_lib, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    ref = oracle.nll(_head(), bf16_bits(_H(9, 5)), make_targets(9, 1000, 6).numpy())
    assert res[0] == res[1]
    assert np.max(np.abs(np.asarray(res[0]) - ref)) <= NLL_TOL
