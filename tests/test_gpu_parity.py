"""GPU parity: the CUDA path through the C ABI against the fp64 CPU oracle.

Acceptance (the logit path's stated tolerances):
  * dequantised components bit-exact;
  * logits: max |Y - Y_ref| <= 1e-2 * rms(Y_ref);
  * per-token NLL: |nll - nll_ref| <= 1e-3 nats.
Shapes span several 128-row vocabulary blocks with a ragged tail, token counts on both
sides of every token-block size (8, 16, 32, 64) and a multi-block prefill, and all
supported group sizes.  The five synthetic heads run at full size on sampled tokens.
"""
import numpy as np
import pytest
import torch

import oracle
import packed_int4_lm_b200 as ah
from workloads import (WORKLOADS, bf16_bits, make_channel_scales, make_hidden,
                       make_targets, make_weight, random_canonical_head)

pytestmark = pytest.mark.gpu

LOGIT_TOL = 1e-2   # relative to rms(Y_ref)
NLL_TOL = 1e-3     # nats


def _rand_H(N, D, seed, sigma_s=0.5, n_out=4, mult=20.0):
    s = make_channel_scales(D, sigma_s, n_out, mult, seed)
    return make_hidden(N, s, seed + 1)


def _assert_logits(Y, Yref, what=""):
    Y = np.asarray(Y, dtype=np.float64)
    rms = np.sqrt(np.mean(Yref ** 2))
    err = np.max(np.abs(Y - Yref))
    assert np.all(np.isfinite(Y)), what
    assert err <= LOGIT_TOL * rms, f"{what}: max err {err:.3e} > {LOGIT_TOL} * rms {rms:.3e}"
    return err / rms


@pytest.fixture(scope="module")
def dev(cuda_ok):
    return torch.device("cuda:0")


# ----------------------------------------------------------------------------------------
# bit-exact dequantisation (repack + device layout + dequant hook)
# ----------------------------------------------------------------------------------------
@pytest.mark.parametrize("g", [32, 64, 128, 256])
def test_dequant_bit_exact(dev, g):
    head = random_canonical_head(300, 512, 5, 3, g, seed=g, zero_rows=4, zero_groups=20)
    dh = ah.DeviceHead.from_canonical(head, dev)
    out = ah.dequant(dh)
    torch.cuda.synchronize()
    assert np.array_equal(out["R"].cpu().double().numpy(), oracle.unpack_residual(head))
    assert np.array_equal(out["Ac"].cpu().double().numpy(),
                          oracle.dequant_int8_rowwise(head["Ac"], head["sAc"]))
    assert np.array_equal(out["Aw"].cpu().double().numpy(),
                          oracle.dequant_int8_rowwise(head["Aw"], head["sAw"]))
    assert np.array_equal(out["Bc"].cpu().double().numpy(),
                          oracle.dequant_int8_groupwise(head["Bc"], head["sBc"], g))
    assert np.array_equal(out["Bw"].cpu().double().numpy(),
                          oracle.dequant_int8_groupwise(head["Bw"], head["sBw"], g))
    part = ah.dequant(dh, 17, 40)
    assert np.array_equal(part["R"].cpu().double().numpy(),
                          oracle.unpack_residual(head, slice(17, 57)))


# ----------------------------------------------------------------------------------------
# logits and NLL on arbitrary packed bytes
# ----------------------------------------------------------------------------------------
@pytest.fixture(scope="module")
def rhead(dev):
    head = random_canonical_head(1000, 512, 8, 8, 64, seed=11, zero_rows=3, zero_groups=50)
    return head, ah.DeviceHead.from_canonical(head, dev)


@pytest.mark.parametrize("N", [1, 3, 8, 9, 16, 17, 31, 33, 64, 65, 130, 200])
def test_logits_random_head(dev, rhead, N):
    head, dh = rhead
    H = _rand_H(N, 512, 100 + N)
    Y = ah.logits(H.to(dev), dh)
    ah.check()
    Yref = oracle.logits(head, bf16_bits(H))
    _assert_logits(Y.cpu().numpy(), Yref, f"N={N}")


@pytest.mark.parametrize("g,r_c,r_r,V,D", [(32, 3, 0, 257, 256), (64, 0, 0, 129, 128),
                                           (128, 16, 16, 515, 1024), (256, 1, 7, 300, 512),
                                           (128, 0, 32, 700, 640), (128, 80, 80, 300, 256)])
def test_logits_shapes_groups_ranks(dev, g, r_c, r_r, V, D):
    head = random_canonical_head(V, D, r_c, r_r, g, seed=V + D)
    dh = ah.DeviceHead.from_canonical(head, dev)
    for N in (5, 40, 150):
        H = _rand_H(N, D, N + g)
        Y = ah.logits(H.to(dev), dh)
        ah.check()
        _assert_logits(Y.cpu().numpy(), oracle.logits(head, bf16_bits(H)), f"{g} {N}")


@pytest.mark.parametrize("sup_exp,fac_exp", [((-40, -30), (-5, -3)), ((-4, -2), (-30, -25)),
                                             ((-20, -20), (-9, -9))])
def test_logits_extreme_scale_ratios(dev, sup_exp, fac_exp):
    """Factor scales far above the residual super-scale (the per-row accumulator exponent
    at its upper clamp, the residual below FP16 resolution there), far below it (lower
    clamp, factor pieces subnormal in FP16), and one fixed ratio, on both paths."""
    head = random_canonical_head(515, 512, 12, 20, 64, seed=77, zero_rows=5,
                                 super_exp_range=sup_exp, factor_exp_range=fac_exp)
    dh = ah.DeviceHead.from_canonical(head, dev)
    for N in (3, 40, 130):
        H = _rand_H(N, 512, 500 + N)
        Y = ah.logits(H.to(dev), dh)
        ah.check()
        _assert_logits(Y.cpu().numpy(), oracle.logits(head, bf16_bits(H)), f"{sup_exp} {N}")


@pytest.mark.parametrize("g,N,launches", [(128, 3, 3), (128, 12, 3), (128, 100, 3), (32, 12, 3)])
def test_fallback_kernels_for_wide_rows(dev, g, N, launches):
    """D = 16384: the decode kernel's resident H does not fit shared memory, so N <= 8 runs
    on the token-block warp-MMA kernel; with g = 32 the tcgen05 kernel's code ring does not
    fit either and N = 12 also takes the warp-MMA kernel (three launches each path)."""
    V, D = 300, 16384
    head = random_canonical_head(V, D, 8, 8, g, seed=N + g, zero_rows=2)
    dh = ah.DeviceHead.from_canonical(head, dev)
    H = _rand_H(N, D, 900 + N)
    Y = ah.logits(H.to(dev), dh)
    ah.check()
    assert ah.last_launches() == launches
    _assert_logits(Y.cpu().numpy(), oracle.logits(head, bf16_bits(H)), f"D={D} g={g} N={N}")


@pytest.fixture(scope="module")
def nhead(dev):
    """Random packed bytes scaled so that rms(Y) is a few units, the regime of language-model
    logits.  The absolute NLL error of any FP32 evaluation grows with the logit magnitude
    (rounding of sums of size |Y|), so an absolute bound in nats is meaningful only there."""
    head = random_canonical_head(1000, 512, 8, 8, 64, seed=12, zero_rows=3, zero_groups=50,
                                 super_exp_range=(-17, -13), factor_exp_range=(-13, -10))
    return head, ah.DeviceHead.from_canonical(head, dev)


def test_nll_head_is_in_logit_regime(nhead):
    head, _ = nhead
    Y = oracle.logits(head, bf16_bits(_rand_H(8, 512, 1)))
    rms = np.sqrt(np.mean(Y ** 2))
    assert 0.5 < rms < 20, rms


@pytest.mark.parametrize("N", [1, 7, 8, 9, 64, 100, 130, 300])
def test_nll_random_head(dev, nhead, N):
    head, dh = nhead
    H = _rand_H(N, 512, 300 + N)
    tg = make_targets(N, head["V"], 7 + N)
    out = ah.nll(H.to(dev), dh, tg.to(dev))
    ah.check()
    ref = oracle.nll(head, bf16_bits(H), tg.numpy())
    err = np.max(np.abs(out.cpu().double().numpy() - ref))
    assert err <= NLL_TOL, err


_WIDE_GROUP_HEADS = {}


def _wide_group_head(dev, g, r_c, r_r):
    """A logit-regime head with one group code per 128 columns or fewer (g >= 128): the
    decode kernel's raw-nibble path (H / 16 on half of the columns, the per-block offset
    taken off through the chain's start value, the code applied to the FP32 block sum)."""
    key = (g, r_c, r_r)
    if key not in _WIDE_GROUP_HEADS:
        head = random_canonical_head(1000, 1024, r_c, r_r, g, seed=60 + g + r_c, zero_rows=3,
                                     zero_groups=20, super_exp_range=(-17, -13),
                                     factor_exp_range=(-13, -10))
        _WIDE_GROUP_HEADS[key] = (head, ah.DeviceHead.from_canonical(head, dev))
    return _WIDE_GROUP_HEADS[key]


@pytest.mark.parametrize("g,r_c,r_r", [(128, 16, 16), (256, 16, 16), (128, 5, 3)])
@pytest.mark.parametrize("N", [1, 4, 8, 9, 16])
def test_nll_decode_kernel_one_code_per_block(dev, g, r_c, r_r, N):
    """Fused NLL on the decode kernel (N <= 16) with g >= 128, element by element against
    the oracle at 1e-3 nats; rank terms on warp MMAs (ranks multiples of 16) and in FP32
    (5 and 3).  The logits of the same calls are checked too."""
    head, dh = _wide_group_head(dev, g, r_c, r_r)
    H = _rand_H(N, 1024, 700 + N + g)
    Yref = oracle.logits(head, bf16_bits(H))
    rms = np.sqrt(np.mean(Yref ** 2))
    assert 0.5 < rms < 20, rms  # the language-model logit regime
    tg = make_targets(N, head["V"], 800 + N)
    out = ah.nll(H.to(dev), dh, tg.to(dev))
    ah.check()
    ref = oracle.nll_from_logits(Yref, tg.numpy())
    err = np.max(np.abs(out.cpu().double().numpy() - ref))
    assert err <= NLL_TOL, (g, N, err)
    Y = ah.logits(H.to(dev), dh)
    ah.check()
    _assert_logits(Y.cpu().numpy(), Yref, f"g={g} N={N}")


def test_many_items_per_cta_consistent(dev):
    """A vocabulary large enough that every persistent CTA of the tensor-memory kernel runs
    several 128-row tiles, repeated: the first 16 tokens of N = 64 and N = 32 calls must
    match the N = 16 call tile for tile, and sampled rows must match the oracle.  Races
    between the producer's bulk copies and the consumers' reads of a ring stage show up
    here as a few corrupted tiles."""
    V, D = 151936, 4096
    head = random_canonical_head(V, D, 32, 32, 128, seed=40, super_exp_range=(-17, -13),
                                 factor_exp_range=(-13, -10))
    dh = ah.DeviceHead.from_canonical(head, dev)
    H = _rand_H(64, D, 41)
    Hd = H.to(dev)
    Y16 = ah.logits(Hd[:16].contiguous(), dh)
    ah.check()
    rows = np.arange(0, V, 97)
    Yref = oracle.logits(head, bf16_bits(H[:16]), rows=rows)
    _assert_logits(Y16.cpu().numpy()[:, rows], Yref, "N=16 sampled rows")
    tol = 1e-4 * float(Y16.abs().max())
    for rep in range(4):
        for N in (64, 32):
            Yn = ah.logits(Hd[:N].contiguous(), dh)
            ah.check()
            diff = float((Yn[:16] - Y16).abs().max())
            assert diff <= tol, (rep, N, diff, tol)


@pytest.mark.parametrize("N", [20, 64])
def test_split_tiles_match_oracle(dev, N):
    """One token tile over more 128-row tiles than resident CTAs: the (tile, K block) units
    are split evenly, so the tiles at the edges of the CTAs' ranges are computed in two
    parts (raw accumulators through scratch, finished by the part that arrives second).
    Every row of the logits and the NLL must match the oracle, and repeated calls must be
    bit-identical (the two parts are added in an order-independent way)."""
    V, D = 40000, 256
    # scaled into the logit regime (rms of a few units), where an NLL bound in nats means
    # something (as the NLL head above)
    head = random_canonical_head(V, D, 16, 16, 64, seed=50, zero_rows=5,
                                 super_exp_range=(-17, -13), factor_exp_range=(-13, -10))
    dh = ah.DeviceHead.from_canonical(head, dev)
    H = _rand_H(N, D, 51 + N)
    Hd = H.to(dev)
    Y = ah.logits(Hd, dh)
    ah.check()
    _assert_logits(Y.cpu().numpy(), oracle.logits(head, bf16_bits(H)), f"split N={N}")
    for _ in range(3):
        assert torch.equal(ah.logits(Hd, dh), Y)
    tg = make_targets(N, V, 52 + N)
    out = ah.nll(Hd, dh, tg.to(dev))
    ah.check()
    ref = oracle.nll(head, bf16_bits(H), tg.numpy())
    err = np.max(np.abs(out.cpu().double().numpy() - ref))
    assert err <= NLL_TOL, err


def test_host_entry_points_match_device(dev, rhead):
    head, dh = rhead
    H = _rand_H(20, 512, 5)
    Yd = ah.logits(H.to(dev), dh).cpu()
    Yh = ah.logits_host(H.pin_memory(), dh)
    assert torch.equal(Yd, Yh)
    tg = make_targets(20, head["V"], 3)
    nd = ah.nll(H.to(dev), dh, tg.to(dev)).cpu()
    nh = ah.nll_host(H, dh, tg)
    assert torch.equal(nd, nh)


def test_launch_counts(dev, rhead):
    """Kernels per call.  N <= 16 (decode kernel): one prologue (H image, corrections and t)
    and the contraction, plus the combine for NLL.  Larger N (tcgen05 kernel): blocked H,
    the rank pieces of t, the contraction."""
    head, dh = rhead
    H = _rand_H(4, 512, 1).to(dev)
    ah.logits(H, dh)
    assert ah.last_launches() == 2
    ah.logits(_rand_H(40, 512, 2).to(dev), dh)
    assert ah.last_launches() == 3
    ah.nll(H, dh, make_targets(4, head["V"], 1).to(dev))
    assert ah.last_launches() == 3
    ah.nll(_rand_H(40, 512, 3).to(dev), dh, make_targets(40, head["V"], 2).to(dev))
    assert ah.last_launches() == 4
    torch.cuda.synchronize()


def test_empty_batch_is_noop(dev, rhead):
    _, dh = rhead
    H = torch.empty(0, 512, dtype=torch.bfloat16, device=dev)
    Y = ah.logits(H, dh)
    assert Y.shape == (0, 1000)
    ah.check()


def test_h_beyond_fp16_is_scaled_and_non_finite_h_is_reported(dev, rhead):
    """An entry beyond the FP16 range is taken (its token is scaled by a power of two,
    see test_token_scaling.py); a NaN entry is reported and its token's logits are NaN."""
    head, dh = rhead
    H = _rand_H(3, 512, 9)
    H[1, 17] = 1.0e5
    Y = ah.logits(H.to(dev), dh)
    ah.check()
    _assert_logits(Y.cpu().numpy()[1], oracle.logits(head, bf16_bits(H))[1], "token scaled")
    H[1, 17] = float("nan")
    Y = ah.logits(H.to(dev), dh)
    with pytest.raises(ah.ArcheadError) as ei:
        ah.check()
    assert ei.value.status == -4
    assert not torch.isfinite(Y[1]).all()
    ah.check()  # the error word was cleared


def test_bad_target_is_reported(dev, rhead):
    head, dh = rhead
    H = _rand_H(4, 512, 10).to(dev)
    tg = torch.tensor([0, head["V"], 5, -1], dtype=torch.int32, device=dev)
    out = ah.nll(H, dh, tg)
    with pytest.raises(ah.ArcheadError) as ei:
        ah.check()
    assert ei.value.status == -5
    o = out.cpu()
    assert torch.isnan(o[1]) and torch.isnan(o[3]) and torch.isfinite(o[0]) and torch.isfinite(o[2])


def test_shape_mismatch_rejected(dev, rhead):
    _, dh = rhead
    H = _rand_H(2, 512, 11).to(dev)
    Y = torch.empty(2, 1000, device=dev)
    import ctypes
    rc = ah._lib.lib().archead_logits(H.data_ptr(), ctypes.byref(dh.struct), Y.data_ptr(), 2,
                                      999, 512, 8, 8, 64, None)
    assert rc == -3


# ----------------------------------------------------------------------------------------
# the five synthetic heads (full size; oracle on sampled tokens where N is large)
# ----------------------------------------------------------------------------------------
def _build(w, device):
    W = make_weight(w.V, w.D, w.rank, w.sigma0, w.noise, w.seed_w, device=device)
    s = make_channel_scales(w.D, w.sigma_s, w.n_outliers, w.outlier_mult, w.seed_scales)
    Hc = make_hidden(w.n_cal, s, w.seed_hcal)
    head = ah.pack.build_head(W, Hc.to(device), w.r_c, w.r_r, w.g, w.p, w.lam,
                              seed=w.seed_rsvd)
    del W
    torch.cuda.empty_cache()
    return head, s


_HEADS = {}


def _workload_head(name, dev):
    w = WORKLOADS[name]
    key = (w.index,)
    if key not in _HEADS:
        head, s = _build(w, dev)
        _HEADS[key] = (head, s, ah.DeviceHead.from_canonical(head, dev))
    return w, _HEADS[key]


def test_workload_tiny(dev):
    w, (head, s, dh) = _workload_head("tiny", dev)
    N = w.Ns[0]
    H = make_hidden(N, s, w.seed_heval)
    Y = ah.logits(H.to(dev), dh)
    ah.check()
    Yref = oracle.logits(head, bf16_bits(H))
    _assert_logits(Y.cpu().numpy(), Yref, "tiny")
    tg = make_targets(N, w.V, w.seed_targets)
    n = ah.nll(H.to(dev), dh, tg.to(dev))
    ah.check()
    assert np.max(np.abs(n.cpu().double().numpy() - oracle.nll_from_logits(Yref, tg.numpy()))) <= NLL_TOL


@pytest.mark.slow
def test_workload_qwen_decode_and_prefill(dev):
    w, (head, s, dh) = _workload_head("qwen_decode", dev)
    Hfull = make_hidden(4096, s, w.seed_heval)           # prefill batch; decode uses its prefix
    sample = np.array([0, 1, 2, 3, 15, 63, 64, 1000, 2047, 4095])
    Yref = oracle.logits(head, bf16_bits(Hfull[sample]))
    tg = make_targets(4096, w.V, w.seed_targets)
    for N in w.Ns:
        Y = ah.logits(Hfull[:N].to(dev), dh)
        ah.check()
        rows = [i for i, r in enumerate(sample) if r < N]
        _assert_logits(Y.cpu().numpy()[sample[rows]], Yref[rows], f"decode N={N}")
        # fused NLL of the same batch (N <= 16: the decode kernel's g = 128 raw-nibble
        # path), at the sampled tokens
        out = ah.nll(Hfull[:N].to(dev), dh, tg[:N].to(dev))
        ah.check()
        ref = oracle.nll_from_logits(Yref[rows], tg.numpy()[sample[rows]])
        err = np.max(np.abs(out.cpu().double().numpy()[sample[rows]] - ref))
        assert err <= NLL_TOL, (N, err)
    Y = ah.logits(Hfull.to(dev), dh)
    ah.check()
    _assert_logits(Y[torch.from_numpy(sample).to(dev)].cpu().numpy(), Yref, "prefill N=4096")


@pytest.mark.slow
def test_workload_llama_batched(dev):
    w, (head, s, dh) = _workload_head("llama_batched", dev)
    H = make_hidden(max(w.Ns), s, w.seed_heval)
    sample = np.array([0, 5, 31, 32, 100, 127, 128, 255])
    Yref = oracle.logits(head, bf16_bits(H[sample]))
    for N in w.Ns:
        Y = ah.logits(H[:N].to(dev), dh)
        ah.check()
        rows = [i for i, r in enumerate(sample) if r < N]
        _assert_logits(Y.cpu().numpy()[sample[rows]], Yref[rows], f"llama N={N}")


@pytest.mark.slow
def test_workload_wide_nll(dev):
    w, (head, s, dh) = _workload_head("wide_nll", dev)
    N = w.Ns[0]
    H = make_hidden(N, s, w.seed_heval)
    tg = make_targets(N, w.V, w.seed_targets)
    out = ah.nll(H.to(dev), dh, tg.to(dev))
    ah.check()
    sample = np.array([0, 1, 511, 4096, 8191])
    ref = oracle.nll(head, bf16_bits(H[sample]), tg.numpy()[sample])
    got = out.cpu().double().numpy()[sample]
    assert np.max(np.abs(got - ref)) <= NLL_TOL, (got, ref)
    assert np.all(np.isfinite(out.cpu().numpy()))


_GUARD = 4096          # floats before and after the output
_CANARY = 0x7FC0DEAD   # a NaN bit pattern no kernel writes


def _guarded(n, dev):
    buf = torch.empty(2 * _GUARD + n, dtype=torch.float32, device=dev)
    buf.view(torch.int32).fill_(_CANARY)
    return buf, buf[_GUARD:_GUARD + n]


def _guards_intact(buf):
    iv = buf.view(torch.int32)
    return bool((iv[:_GUARD] == _CANARY).all()) and bool((iv[-_GUARD:] == _CANARY).all())


@pytest.mark.parametrize("V,D,N,g,path", [(1000, 512, 4, 128, "decode"),
                                          (515, 1024, 12, 64, "decode, two token blocks"),
                                          (1000, 512, 40, 64, "tcgen05"),
                                          (40000, 256, 20, 64, "tcgen05, split tiles"),
                                          (300, 16384, 8, 128, "warp-MMA fallback"),
                                          (1000, 512, 300, 128, "tcgen05, several token tiles")])
def test_outputs_stay_inside_their_rows(dev, V, D, N, g, path):
    """Canary bands of a NaN pattern before and after Y (N x V, ragged V) and the NLL output
    stay untouched on every kernel path, including the split tiles that go through scratch
    and the ragged last vocabulary tile."""
    head = random_canonical_head(V, D, 8, 8, g, seed=V + N, zero_rows=2,
                                 super_exp_range=(-17, -13), factor_exp_range=(-13, -10))
    dh = ah.DeviceHead.from_canonical(head, dev)
    Hc = _rand_H(N, D, 1000 + N)
    H = Hc.to(dev)
    buf, flat = _guarded(N * V, dev)
    Y = flat.view(N, V)
    ah.logits(H, dh, out=Y)
    ah.check()
    assert _guards_intact(buf), path
    rows = np.arange(0, V, max(1, V // 997))
    _assert_logits(Y.cpu().numpy()[:, rows], oracle.logits(head, bf16_bits(Hc), rows=rows), path)
    nbuf, nflat = _guarded(N, dev)
    tg = make_targets(N, V, 2000 + N)
    ah.nll(H, dh, tg.to(dev), out=nflat)
    ah.check()
    assert _guards_intact(nbuf), path
    assert torch.isfinite(nflat).all()
