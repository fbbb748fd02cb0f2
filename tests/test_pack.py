"""Construction (Algorithm 1) invariants: the quantizers' error bounds, the metric identity
at p = 1/2, the Frobenius special case and the conditional optimum of the correction.

Citations are to the ARCHead paper (arXiv 2608.02703 HTML), Sec. 3.
"""
import numpy as np
import pytest
import torch

import oracle
from packed_int4_lm_b200 import pack
from workloads import WORKLOADS, bf16_bits, make_channel_scales, make_hidden, make_weight


def test_q8_groupwise_bounds():
    rng = np.random.default_rng(0)
    X = torch.from_numpy(rng.standard_normal((9, 256)) * 3)
    q, s, dq = pack.q8_groupwise(X, 64)
    assert q.dtype == torch.int8 and s.shape == (9, 4)
    assert int(q.abs().max()) == 127
    step = s.double().repeat_interleave(64, dim=1)
    assert torch.all((X - dq).abs() <= step / 2 * (1 + 1e-6) + 1e-12)


def test_q8_zero_group():
    X = torch.zeros(2, 128, dtype=torch.float64)
    X[1, 70] = 2.0
    q, s, dq = pack.q8_groupwise(X, 64)
    assert s[0, 0] == 0 and s[0, 1] == 0 and s[1, 0] == 0
    assert torch.all(q[0] == 0) and q[1, 70] == 127 and dq[1, 70] == 2.0


def test_sc4_bounds_and_codes():
    """SC4: |R - q c S| <= c S / 2 wherever the nibble is not clamped; codes in [1, 255]
    for nonzero groups, 0 for zero groups; the super-scale is a BF16 value."""
    rng = np.random.default_rng(1)
    R = torch.from_numpy(rng.standard_normal((13, 512)) * rng.uniform(0.01, 1, (13, 1)))
    R[3, 64:128] = 0
    q, c, S, dq = pack.sc4(R, 64)
    assert int(q.min()) >= -8 and int(q.max()) <= 7
    assert c[3, 1] == 0 and torch.all(c[torch.arange(13) != 3] >= 1)
    step = (c.double() * S.double()[:, None]).repeat_interleave(64, dim=1)
    unclamped = (q > -8) & (q < 7)
    err = (R - dq).abs()
    assert torch.all(err[unclamped] <= step[unclamped] / 2 * (1 + 1e-9))
    # max-amplitude group uses (almost) the full code range
    assert int(c.max()) >= 250


def test_pack_nibbles_roundtrip_with_oracle_decoder():
    rng = np.random.default_rng(2)
    q = torch.from_numpy(rng.integers(-8, 8, size=(7, 64)).astype(np.int8))
    packed = pack.pack_nibbles(q).numpy()
    assert packed.shape == (7, 32) and packed.dtype == np.uint8
    assert np.array_equal(oracle.decode_int4_bytes(packed), q.numpy())


def _rand_H(N, D, seed):
    s = make_channel_scales(D, 0.5, 4, 20.0, seed)
    return make_hidden(N, s, seed + 1)


def test_metric_half_power_identity():
    """Sec. 3.1: at p = 1/2, ||Delta T_p||_F^2 = ||H Delta^T||_F^2 / N + lam c_bar ||Delta||_F^2."""
    D, N, lam = 48, 300, 0.05
    H = _rand_H(N, D, 10)
    T, Tinv, C, C_lam = pack.metric_transform(H, lam, 0.5)
    Hd = H.double()
    cbar = torch.diagonal(Hd.t() @ Hd / N).mean()
    rng = np.random.default_rng(3)
    Delta = torch.from_numpy(rng.standard_normal((20, D)))
    lhs = (Delta @ T).pow(2).sum()
    rhs = (Hd @ Delta.t()).pow(2).sum() / N + lam * cbar * Delta.pow(2).sum()
    assert abs(float(lhs - rhs)) <= 1e-10 * float(rhs)
    assert torch.allclose(T @ Tinv, torch.eye(D, dtype=torch.float64), atol=1e-9)


def test_metric_zero_power_is_frobenius():
    """p = 0 gives T = I: the objective is the Frobenius special case C = I (Sec. 3.1)."""
    T, Tinv, _, _ = pack.metric_transform(_rand_H(100, 16, 20), 0.01, 0.0)
    assert torch.allclose(T, torch.eye(16, dtype=torch.float64), atol=1e-12)
    assert torch.allclose(Tinv, torch.eye(16, dtype=torch.float64), atol=1e-12)


def _small_head(r_c=4, r_r=4, p=0.75, exact=True, V=200, D=64, g=16):
    W = make_weight(V, D, rank=16, sigma0=0.5, noise=0.02, seed=30)
    H = _rand_H(400, D, 31)
    return W, H, pack.build_head(W, H, r_c, r_r, g, p, 0.01, seed=5, exact_svd=exact,
                                 return_intermediates=True)


def test_conditional_optimum_of_correction():
    """Sec. 3.2 / 5: among rank-r_r corrections to the fixed core, the truncated SVD of E T_p
    mapped back through T_p^-1 has the lowest metric error, equal to the discarded
    singular-value energy; Frobenius-SVD and random corrections are not better."""
    W, H, (head, it) = _small_head()
    T, E = it["T"], it["E"]
    r = 4
    err = lambda corr: float(((E - corr) @ T).pow(2).sum())
    ours = err(it["Aw_f"] @ it["Bw_f"])
    sv = torch.linalg.svdvals(E @ T)
    assert abs(ours - float(sv[r:].pow(2).sum())) <= 1e-9 * ours
    U, S, Vt = torch.linalg.svd(E, full_matrices=False)
    assert err((U[:, :r] * S[:r]) @ Vt[:r]) >= ours * (1 - 1e-12)
    gen = torch.Generator().manual_seed(0)
    for _ in range(5):
        a = torch.randn(E.shape[0], r, generator=gen, dtype=torch.float64)
        b = torch.randn(r, E.shape[1], generator=gen, dtype=torch.float64) * 1e-3
        assert err(a @ b) >= ours


def test_randomized_svd_matches_exact_on_low_rank():
    gen = torch.Generator().manual_seed(1)
    A = torch.randn(300, 8, generator=gen, dtype=torch.float64) @ torch.randn(8, 50, generator=gen, dtype=torch.float64)
    U, S, Vt = pack.randomized_svd(A, 8, seed=3)
    assert torch.allclose((U * S) @ Vt, A, atol=1e-9)


def test_correction_reduces_metric_error_and_core_alone_when_r_r_zero():
    W, H, (head, it) = _small_head()
    T = it["T"]
    What = torch.from_numpy(oracle.dense_head_rows(head))
    core_err = float(((W.double() - it["W_d"]) @ T).pow(2).sum())
    full_err = float(((W.double() - What) @ T).pow(2).sum())
    assert full_err < core_err
    _, _, (head0, it0) = _small_head(r_r=0)
    W0 = torch.from_numpy(oracle.dense_head_rows(head0))
    assert torch.equal(W0, it0["W_d"])


def test_head_layout_and_no_dense_matrix():
    """Sec. 3: the packed module registers the SC4 residual and scales, the quantized
    factors and shape metadata; no V x D 16-bit (or wider) array."""
    _, _, (head, _) = _small_head()
    V, D = head["V"], head["D"]
    assert head["r_nib"].shape == (V, D // 2) and head["r_nib"].dtype == np.uint8
    assert head["r_code"].dtype == np.uint8 and head["r_super"].dtype == np.uint16
    for k, a in head.items():
        if isinstance(a, np.ndarray) and a.ndim == 2 and a.shape == (V, D):
            pytest.fail(f"dense V x D array {k} in packed head")
    assert pack.storage_ratio(head) == oracle.packed_nbytes(head) / (2 * V * D)


def test_tiny_workload_quality_and_storage():
    w = WORKLOADS["tiny"]
    W = make_weight(w.V, w.D, w.rank, w.sigma0, w.noise, w.seed_w)
    s = make_channel_scales(w.D, w.sigma_s, w.n_outliers, w.outlier_mult, w.seed_scales)
    Hc = make_hidden(w.n_cal, s, w.seed_hcal)
    head = pack.build_head(W, Hc, w.r_c, w.r_r, w.g, w.p, w.lam, seed=w.seed_rsvd)
    ratio = pack.storage_ratio(head)
    assert 0.29 < ratio < 0.32
    What = oracle.dense_head_rows(head)
    rel = np.linalg.norm(What - W.double().numpy()) / np.linalg.norm(W.double().numpy())
    assert rel < 0.15   # INT4 residual error on a noise-dominated head


def test_storage_matched_baselines_on_tiny_head():
    """The pages' comparison against storage-matched heads on the same kernels, on the tiny
    synthetic workload: plain group INT4 (r_c = r_r = 0, SC4 of W itself, g = 32 so its
    bytes come close to the packed head's) and the core without the correction (r_r = 0).
    On held-out activations the full construction must have clearly the smallest logit
    error (measured: 0.044 against 0.098 and 0.106, storage ratios 0.303 / 0.275 / 0.285)."""
    w = WORKLOADS["tiny"]
    W = make_weight(w.V, w.D, w.rank, w.sigma0, w.noise, w.seed_w)
    s = make_channel_scales(w.D, w.sigma_s, w.n_outliers, w.outlier_mult, w.seed_scales)
    Hc = make_hidden(w.n_cal, s, w.seed_hcal)
    Hb = bf16_bits(make_hidden(128, s, 99))
    Yref = oracle.bf16_bits_to_f64(Hb) @ W.double().numpy().T

    def rel_err(head):
        Y = oracle.logits(head, Hb)
        return np.linalg.norm(Y - Yref) / np.linalg.norm(Yref)

    full = pack.build_head(W, Hc, w.r_c, w.r_r, w.g, w.p, w.lam, seed=w.seed_rsvd)
    naive = pack.build_head(W, Hc, 0, 0, 32, w.p, w.lam, seed=w.seed_rsvd)
    core = pack.build_head(W, Hc, w.r_c, 0, w.g, w.p, w.lam, seed=w.seed_rsvd)
    assert pack.storage_ratio(naive) < pack.storage_ratio(full) < 1.15 * pack.storage_ratio(naive)
    e_full, e_naive, e_core = rel_err(full), rel_err(naive), rel_err(core)
    assert e_full < 0.6 * e_naive, (e_full, e_naive)
    assert e_full < 0.6 * e_core, (e_full, e_core)


def test_agreement_with_the_dense_head_on_tiny_head():
    """Top-k agreement and KL(dense || packed) of the next-token distributions on held-out
    activations of the tiny synthetic head, the pages' agreement measures, for the full
    construction and the two storage-matched baselines (fp64 oracle logits).  Measured:
    KL 0.0018 / 0.0074 / 0.0096 nats, top-5 agreement 0.91 / 0.85 / 0.84."""
    w = WORKLOADS["tiny"]
    W = make_weight(w.V, w.D, w.rank, w.sigma0, w.noise, w.seed_w)
    s = make_channel_scales(w.D, w.sigma_s, w.n_outliers, w.outlier_mult, w.seed_scales)
    Hc = make_hidden(w.n_cal, s, w.seed_hcal)
    Hb = bf16_bits(make_hidden(128, s, 99))
    Yd = oracle.bf16_bits_to_f64(Hb) @ W.double().numpy().T

    def log_softmax(Z):
        Z = Z - Z.max(axis=1, keepdims=True)
        return Z - np.log(np.exp(Z).sum(axis=1, keepdims=True))

    def measures(head):
        Y = oracle.logits(head, Hb)
        pd, pp = log_softmax(Yd), log_softmax(Y)
        kl = float(np.mean((np.exp(pd) * (pd - pp)).sum(axis=1)))
        a, b = np.argsort(-Y, axis=1)[:, :5], np.argsort(-Yd, axis=1)[:, :5]
        top5 = float(np.mean([len(set(a[i]) & set(b[i])) / 5 for i in range(len(a))]))
        return kl, top5

    kl_f, t5_f = measures(pack.build_head(W, Hc, w.r_c, w.r_r, w.g, w.p, w.lam, seed=w.seed_rsvd))
    kl_n, t5_n = measures(pack.build_head(W, Hc, 0, 0, 32, w.p, w.lam, seed=w.seed_rsvd))
    kl_c, t5_c = measures(pack.build_head(W, Hc, w.r_c, 0, w.g, w.p, w.lam, seed=w.seed_rsvd))
    assert kl_f < 0.5 * kl_n and kl_f < 0.5 * kl_c, (kl_f, kl_n, kl_c)
    assert t5_f > t5_n and t5_f > t5_c, (t5_f, t5_n, t5_c)


def test_serialized_module_round_trip_is_bit_identical(tmp_path):
    """Sec. 3 measures storage over the serialised module: the packed head written to a
    file and read back has the same bytes in every array, the same shape metadata, and a
    file size equal to the arrays' bytes plus a small header."""
    from workloads import random_canonical_head
    from packed_int4_lm_b200 import pack
    for (V, D, r_c, r_r, g) in [(300, 512, 5, 3, 64), (129, 256, 0, 0, 128), (64, 128, 16, 0, 32)]:
        head = random_canonical_head(V, D, r_c, r_r, g, seed=V + D, zero_rows=2)
        path = tmp_path / f"h{V}.archead"
        size = pack.save_head(head, str(path))
        assert size == path.stat().st_size == pack.serialized_nbytes(head)
        back = pack.load_head(str(path))
        for k in ("V", "D", "r_c", "r_r", "g"):
            assert back[k] == head[k]
        for k in ("r_nib", "r_code", "r_super", "Ac", "sAc", "Bc", "sBc", "Aw", "sAw", "Bw", "sBw"):
            a, b = np.ascontiguousarray(head[k]), back[k]
            assert a.dtype == b.dtype and a.shape == b.shape, k
            assert a.tobytes() == b.tobytes(), k
        payload = sum(np.asarray(head[k]).nbytes for k in head if isinstance(head[k], np.ndarray))
        assert payload <= size <= payload + 11 * 16 + 1024
        Hb = bf16_bits(make_hidden(3, make_channel_scales(D, 0.5, 4, 20.0, 1), 2))
        assert np.array_equal(oracle.logits(back, Hb), oracle.logits(head, Hb))
    bad = tmp_path / "bad.archead"
    bad.write_bytes(b"NOTAHEAD" + b"\0" * 32)
    with pytest.raises(ValueError):
        pack.load_head(str(bad))
