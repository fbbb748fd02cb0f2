"""The construction (ARCHead Sec. 3 and Algorithm 1) run on the GPU, as the benchmark runs
it: the same invariants as the CPU tests on GPU tensors (the p = 1/2 metric identity, the
conditional optimum of the correction), and agreement with the CPU construction on the same
inputs with exact SVDs.  Randomness: the exact-SVD path draws nothing, so both devices
compute the same quantities and may differ only by floating-point order."""
import numpy as np
import pytest
import torch

import oracle
from packed_int4_lm_b200 import pack
from workloads import make_channel_scales, make_hidden, make_weight

pytestmark = pytest.mark.gpu


def _inputs(V=300, D=128):
    W = make_weight(V, D, rank=16, sigma0=0.5, noise=0.02, seed=40)
    H = make_hidden(600, make_channel_scales(D, 0.5, 4, 20.0, 41), 42)
    return W, H


def test_metric_identity_and_conditional_optimum_on_gpu(cuda_ok):
    dev = torch.device("cuda:0")
    W, H = _inputs()
    lam = 0.05
    T, Tinv, _, _ = pack.metric_transform(H.to(dev), lam, 0.5)
    Hd = H.to(dev).double()
    N = Hd.shape[0]
    cbar = torch.diagonal(Hd.t() @ Hd / N).mean()
    Delta = torch.randn(20, W.shape[1], dtype=torch.float64, device=dev,
                        generator=torch.Generator(device=dev).manual_seed(3))
    lhs = (Delta @ T).pow(2).sum()
    rhs = (Hd @ Delta.t()).pow(2).sum() / N + lam * cbar * Delta.pow(2).sum()
    assert abs(float(lhs - rhs)) <= 1e-9 * float(rhs)
    head, it = pack.build_head(W.to(dev), H.to(dev), 4, 4, 32, 0.75, 0.01, seed=5,
                               exact_svd=True, return_intermediates=True)
    T, E = it["T"], it["E"]
    ours = float(((E - it["Aw_f"] @ it["Bw_f"]) @ T).pow(2).sum())
    sv = torch.linalg.svdvals(E @ T)
    assert abs(ours - float(sv[4:].pow(2).sum())) <= 1e-8 * ours
    U, S, Vt = torch.linalg.svd(E, full_matrices=False)
    assert float(((E - (U[:, :4] * S[:4]) @ Vt[:4]) @ T).pow(2).sum()) >= ours * (1 - 1e-12)


def test_gpu_construction_agrees_with_cpu(cuda_ok):
    """Exact SVDs on both devices: every stored array agrees except where a value lies on a
    rounding boundary of its quantizer (a handful of nibbles and codes); the dequantised
    heads' metric errors agree to 1e-6."""
    dev = torch.device("cuda:0")
    W, H = _inputs()
    args = (4, 4, 32, 0.75, 0.01)
    hc, itc = pack.build_head(W, H, *args, seed=5, exact_svd=True, return_intermediates=True)
    hg, itg = pack.build_head(W.to(dev), H.to(dev), *args, seed=5, exact_svd=True,
                              return_intermediates=True)
    qc = oracle.decode_int4_bytes(hc["r_nib"])
    qg = oracle.decode_int4_bytes(hg["r_nib"])
    assert np.mean(qc == qg) > 0.999
    assert np.mean(hc["r_code"] == hg["r_code"]) > 0.999
    assert np.array_equal(hc["r_super"], hg["r_super"]) or np.mean(hc["r_super"] == hg["r_super"]) > 0.99
    T = itc["T"]
    ec = float(((W.double() - torch.from_numpy(oracle.dense_head_rows(hc))) @ T).pow(2).sum())
    eg = float(((W.double() - torch.from_numpy(oracle.dense_head_rows(hg))) @ T).pow(2).sum())
    assert abs(ec - eg) <= 1e-6 * ec
