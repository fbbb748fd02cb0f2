"""Token scaling: any finite BF16 H is accepted.  The kernels take FP16 operands, so each
token row is scaled by the power of two that brings its largest |h| below 2^15 (exact) and
its logits are multiplied back.  Rows far outside the FP16 range (|h| up to about 2^107)
and ordinary rows share each call, on every kernel path, and are compared with the fp64
oracle token by token: max |Y[n] - Y_ref[n]| <= 1e-2 rms(Y_ref[n]), the parity tolerance
applied per row because the rows' logits differ by up to 2^100.  A non-finite entry still
raises ARCHEAD_ERR_RANGE_H.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import packed_int4_lm_b200 as ah
from packed_int4_lm_b200 import _lib
from workloads import bf16_bits, make_channel_scales, make_hidden, make_targets, random_canonical_head

pytestmark = pytest.mark.gpu

LOGIT_TOL = 1e-2


def _head(V, D, r, g, seed):
    # factor scales small enough that the scaled rank products stay inside FP16
    return random_canonical_head(V, D, r, r, g, seed=seed, zero_rows=2,
                                 super_exp_range=(-17, -13), factor_exp_range=(-13, -10))


def _scaled_H(N, D, seed, exps):
    """BF16 rows with row n multiplied by 2^exps[n] (exact on BF16 values)."""
    H = make_hidden(N, make_channel_scales(D, 0.5, 4, 20.0, seed), seed + 1).float()
    for n, k in exps.items():
        H[n] *= 2.0 ** k
    H = H.to(torch.bfloat16)
    assert torch.isfinite(H.float()).all()
    return H


def _assert_per_token(Y, Yref, what):
    Y = np.asarray(Y, dtype=np.float64)
    assert np.all(np.isfinite(Y)), what
    for n in range(Yref.shape[0]):
        rms = np.sqrt(np.mean(Yref[n] ** 2))
        err = np.max(np.abs(Y[n] - Yref[n]))
        assert err <= LOGIT_TOL * rms, f"{what} token {n}: {err:.3e} > {LOGIT_TOL} * {rms:.3e}"


@pytest.fixture(scope="module")
def dev(cuda_ok):
    return torch.device("cuda:0")


# (V, D, rank, g, N): the decode kernel with raw nibble reads (g = 128) and with exact
# dequantisation (g = 64), one and two token blocks; the tcgen05 kernel with one split
# token tile and with several 128-token tiles
CASES = [(700, 1024, 32, 128, 5, "decode, g = 128"),
         (700, 1024, 16, 64, 12, "decode, g = 64, two token blocks"),
         (900, 1024, 32, 128, 40, "tcgen05, one token tile"),
         (600, 512, 32, 128, 300, "tcgen05, several token tiles")]


@pytest.mark.parametrize("V,D,r,g,N,path", CASES)
def test_scaled_tokens_logits(dev, V, D, r, g, N, path):
    head = _head(V, D, r, g, seed=V + N)
    dh = ah.DeviceHead.from_canonical(head, dev)
    exps = {0: 20, 1: 100, N - 1: 60}
    if N > 3:
        exps[3] = 17  # just above the FP16 range
    Hc = _scaled_H(N, D, 31 + N, exps)
    Y = ah.logits(Hc.to(dev), dh).cpu().numpy()
    ah.check()
    _assert_per_token(Y, oracle.logits(head, bf16_bits(Hc)), path)


@pytest.mark.parametrize("V,D,r,g,N,path", [CASES[0], CASES[2]])
def test_scaled_tokens_nll(dev, V, D, r, g, N, path):
    """The fused NLL sees the true logits: per token within 1e-3 nats plus 1e-4 of the
    token's rms logit.  The NLL of a token whose logits are of size L is a difference of
    numbers of size L, and FP32 logits carry about 17 significant bits on the decode
    kernel's raw-nibble path (its per-block offset takes about 7 of the 24), so its error is
    about 2e-5 L; the 1e-3 nats of the parity tests is this bound for L of a few units."""
    head = _head(V, D, r, g, seed=V + N + 1)
    dh = ah.DeviceHead.from_canonical(head, dev)
    Hc = _scaled_H(N, D, 41 + N, {0: 16, 2: 24})
    tg = make_targets(N, V, 43)
    nll = ah.nll(Hc.to(dev), dh, tg.to(dev)).cpu().double().numpy()
    ah.check()
    Hb = bf16_bits(Hc)
    ref = oracle.nll(head, Hb, tg.numpy())
    Yref = oracle.logits(head, Hb)
    for n in range(N):
        tol = 1e-3 + 1e-4 * np.sqrt(np.mean(Yref[n] ** 2))
        assert abs(nll[n] - ref[n]) <= tol, (path, n, nll[n], ref[n], tol)


def test_scaled_tokens_warp_mma_noalloc_and_agreement(dev):
    """The token-block warp-MMA kernel (via the no-allocation entry point) and the agreement
    epilogue on the same kernel."""
    head = _head(500, 512, 8, 64, seed=77)
    dh = ah.DeviceHead.from_canonical(head, dev)
    N = 20
    Hc = _scaled_H(N, 512, 78, {0: 30, 7: 90, 19: 18})
    H = Hc.to(dev)
    Yref = oracle.logits(head, bf16_bits(Hc))
    Y = torch.full((N, 500), float("nan"), device=dev)
    rc = _lib.lib().archead_logits_noalloc(H.data_ptr(), ctypes.byref(dh.struct), Y.data_ptr(),
                                           N, *dh.shape_args, torch.cuda.current_stream().cuda_stream)
    assert rc == 0
    ah.check()
    _assert_per_token(Y.cpu().numpy(), Yref, "warp-MMA (no-allocation entry point)")
    # agreement against the oracle's own logits as the dense head: its top-1 must be the
    # packed top-1 wherever the top two oracle logits are apart by more than the tolerance
    a = ah.agreement(H, dh, torch.from_numpy(Yref.astype(np.float32)).to(dev), 3)
    ah.check()
    top = a["topk"].cpu().numpy()
    srt = np.sort(Yref, axis=1)[:, ::-1]
    for n in range(N):
        gap = srt[n, 0] - srt[n, 1]
        if gap > 2 * LOGIT_TOL * np.sqrt(np.mean(Yref[n] ** 2)):
            assert top[n, 0] == int(np.argmax(Yref[n])), n


@pytest.mark.parametrize("N", [4, 40])
def test_non_finite_h_raises(dev, N):
    head = _head(300, 512, 16, 128, seed=N)
    dh = ah.DeviceHead.from_canonical(head, dev)
    Hc = _scaled_H(N, 512, 90, {})
    Hc[1, 37] = float("inf")
    with pytest.raises(_lib.ArcheadError) as ei:
        ah.logits(Hc.to(dev), dh)
        ah.check()
    assert ei.value.status == _lib.STATUS_CODE["ARCHEAD_ERR_RANGE_H"]
    ah.check()  # the error word was cleared
