"""Pins for the CPU oracle: facts that do not come from the oracle's own formulas.

Each test names the passage of the ARCHead paper (arXiv 2608.02703 HTML) it follows.
A plausible slip in the oracle -- swapped nibble order, wrong group index, a transposed
factor, a dropped term, a wrong scale -- makes at least one of these fail.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from workloads import random_canonical_head


def _empty_head(V, D, r_c, r_r, g):
    G = D // g
    return {
        "V": V, "D": D, "r_c": r_c, "r_r": r_r, "g": g,
        "r_nib": np.zeros((V, D // 2), np.uint8),
        "r_code": np.zeros((V, G), np.uint8),
        "r_super": np.zeros(V, np.uint16),
        "Ac": np.zeros((V, r_c), np.int8), "sAc": np.zeros(V, np.float32),
        "Bc": np.zeros((r_c, D), np.int8), "sBc": np.zeros((r_c, G), np.float32),
        "Aw": np.zeros((V, r_r), np.int8), "sAw": np.zeros(V, np.float32),
        "Bw": np.zeros((r_r, D), np.int8), "sBw": np.zeros((r_r, G), np.float32),
    }


def _bf16_bits_of(x):
    """BF16 bit patterns of values exactly representable in BF16 (torch does the rounding)."""
    t = torch.tensor(np.asarray(x, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def _identity_H(D):
    return _bf16_bits_of(np.eye(D, dtype=np.float32))


def test_bf16_decoding_matches_torch_on_all_patterns():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ours = oracle.bf16_bits_to_f64(bits)
    ref = torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16).to(torch.float64).numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], ref[~nan])


def test_int4_decoding_all_bytes():
    """Sec. 3 'packed signed-INT4': each byte splits into two values in [-8, 7] whose
    4-bit two's-complement patterns reassemble the byte (low nibble = even column)."""
    b = np.arange(256, dtype=np.uint8)
    vals = oracle.decode_int4_bytes(b[:, None])
    assert vals.shape == (256, 2)
    lo, hi = vals[:, 0].astype(np.int64), vals[:, 1].astype(np.int64)
    assert lo.min() == -8 and lo.max() == 7 and hi.min() == -8 and hi.max() == 7
    assert np.array_equal(((lo & 0xF) | ((hi & 0xF) << 4)).astype(np.uint8), b)


def _pack_test(q):
    """Inverse of the canonical nibble layout, written from its definition."""
    q = np.asarray(q, np.int64)
    return ((q[:, 0::2] & 0xF) | ((q[:, 1::2] & 0xF) << 4)).astype(np.uint8)


def test_unit_scale_head_is_exact_integer_matmul():
    """r_c = r_r = 0 with codes 1 and super-scale 1 leaves a plain INT4 matrix Q, so the
    logits are H Q^T: an exact integer product (Sec. 3 final formula with empty factors)."""
    rng = np.random.default_rng(1)
    V, D, g, N = 37, 256, 64, 5
    Q = rng.integers(-8, 8, size=(V, D))
    head = _empty_head(V, D, 0, 0, g)
    head["r_nib"] = _pack_test(Q)
    head["r_code"][:] = 1
    head["r_super"][:] = _bf16_bits_of(np.ones(V))
    Hi = rng.integers(-100, 101, size=(N, D))
    Y = oracle.logits(head, _bf16_bits_of(Hi))
    assert np.array_equal(Y, (Hi @ Q.T).astype(np.float64))


@pytest.mark.parametrize("v,d,qv", [(3, 137, -5), (0, 0, 7), (4, 255, -8), (2, 64, 1)])
def test_single_residual_entry(v, d, qv):
    """One nonzero nibble: W_hat has exactly one entry q * code[v, d // g] * S_v."""
    V, D, g = 5, 256, 64
    rng = np.random.default_rng(v * 1000 + d)
    head = _empty_head(V, D, 0, 0, g)
    Q = np.zeros((V, D), np.int64)
    Q[v, d] = qv
    head["r_nib"] = _pack_test(Q)
    head["r_code"] = rng.integers(1, 256, size=(V, D // g)).astype(np.uint8)
    head["r_super"][:] = _bf16_bits_of(np.full(V, 0.375))
    Y = oracle.logits(head, _identity_H(D))  # row n of Y = column n of W_hat^T
    expect = np.zeros((D, V))
    expect[d, v] = qv * int(head["r_code"][v, d // g]) * 0.375
    assert np.array_equal(Y, expect)


def test_group_code_mapping():
    """Every nibble = 1, super-scale 1: W_hat[v, d] = code[v, d // g] (group index pin)."""
    V, D, g = 6, 256, 32
    rng = np.random.default_rng(7)
    head = _empty_head(V, D, 0, 0, g)
    head["r_nib"] = _pack_test(np.ones((V, D), np.int64))
    head["r_code"] = rng.integers(0, 256, size=(V, D // g)).astype(np.uint8)
    head["r_super"][:] = _bf16_bits_of(np.ones(V))
    Y = oracle.logits(head, _identity_H(D))
    for vv in range(V):
        for dd in range(D):
            assert Y[dd, vv] == head["r_code"][vv, dd // g]


def test_single_factor_entries():
    """Core and correction factors each with one entry: W_hat[v, d] = (a s_A)(b s_B[group]).
    Fixes the row-wise scale of A, the group-wise scale of B and both orientations."""
    V, D, g = 4, 128, 64
    head = _empty_head(V, D, 2, 3, g)
    head["Ac"][2, 1] = 7
    head["sAc"][:] = [1.0, 2.0, 0.5, 4.0]
    head["Bc"][1, 70] = -3
    head["sBc"][1] = [0.125, 0.25]          # column 70 is in group 1
    head["Aw"][1, 2] = -11
    head["sAw"][:] = [0.75, 0.0625, 1.5, 3.0]
    head["Bw"][2, 5] = 9
    head["sBw"][2] = [0.5, 8.0]             # column 5 is in group 0
    W = oracle.dense_head_rows(head)
    expect = np.zeros((V, D))
    expect[2, 70] = (7 * 0.5) * (-3 * 0.25)
    expect[1, 5] = (-11 * 0.0625) * (9 * 0.5)
    assert np.array_equal(W, expect)
    Y = oracle.logits(head, _identity_H(D))
    assert np.array_equal(Y, expect.T)


def test_factored_equals_dense():
    """Sec. 3: Y = H W_d^T + (H B_w^T) A_w^T equals H (W_d + A_w B_w)^T."""
    head = random_canonical_head(96, 256, 8, 8, 64, seed=3)
    rng = np.random.default_rng(4)
    H = _bf16_bits_of(rng.standard_normal((7, 256)).astype(np.float32))
    Y1 = oracle.logits(head, H)
    Y2 = oracle.logits_factored(head, H)
    assert np.max(np.abs(Y1 - Y2)) <= 1e-10 * np.max(np.abs(Y1))


def test_vocab_subsets_and_chunks_agree():
    head = random_canonical_head(100, 128, 4, 4, 64, seed=5, zero_rows=3)
    rng = np.random.default_rng(6)
    H = _bf16_bits_of(rng.standard_normal((3, 128)).astype(np.float32))
    Y = oracle.logits(head, H)
    Yc = oracle.logits(head, H, chunk=7)
    tol = 1e-12 * np.max(np.abs(Y))   # BLAS may sum in another order per slice shape
    assert np.max(np.abs(Y - Yc)) <= tol
    rows = np.array([99, 0, 17, 42])
    assert np.max(np.abs(oracle.logits(head, H, rows=rows) - Y[:, rows])) <= tol


def test_zero_super_scale_row_has_no_residual():
    head = random_canonical_head(16, 128, 2, 2, 64, seed=8)
    head["r_super"][5] = 0
    W = oracle.unpack_residual(head)
    assert np.all(W[5] == 0) and np.any(W[4] != 0)


def test_residual_entries_exact_in_single_precision():
    """q * c * S has at most 4 + 8 + 8 significant bits, so it is exact in IEEE single."""
    head = random_canonical_head(64, 256, 0, 0, 64, seed=9)
    R = oracle.unpack_residual(head)
    assert np.array_equal(R.astype(np.float32).astype(np.float64), R)


def test_nll_constant_logits_is_log_vocab():
    Y = np.full((3, 1000), 2.5)
    out = oracle.nll_from_logits(Y, np.array([0, 999, 500]))
    assert np.allclose(out, math.log(1000), rtol=0, atol=1e-12)


def test_nll_shift_invariance_and_dominant_logit():
    rng = np.random.default_rng(10)
    Y = rng.standard_normal((4, 50))
    t = np.array([3, 7, 0, 49])
    a = oracle.nll_from_logits(Y, t)
    b = oracle.nll_from_logits(Y + 123.0, t)
    assert np.allclose(a, b, atol=1e-12)
    Y2 = Y.copy()
    Y2[np.arange(4), t] = 1e3
    assert np.all(oracle.nll_from_logits(Y2, t) < 1e-300 + 1e-12)


def test_nll_matches_library_cross_entropy():
    rng = np.random.default_rng(11)
    Y = rng.standard_normal((6, 333)) * 4
    t = rng.integers(0, 333, size=6)
    ref = torch.nn.functional.cross_entropy(torch.from_numpy(Y), torch.from_numpy(t),
                                            reduction="none").numpy()
    assert np.allclose(oracle.nll_from_logits(Y, t), ref, rtol=0, atol=1e-12)


def test_int8_dequant_is_single_precision_product():
    """The dequantised INT8 factor is the IEEE-single product of value and FP32 scale,
    the same single multiply a GPU performs with round-to-nearest-even."""
    q = np.array([[127, -127, 3]], np.int8)
    s = np.array([0.1], np.float32)
    out = oracle.dequant_int8_rowwise(q, s)
    ref = torch.tensor(q, dtype=torch.float32) * torch.tensor(s)[:, None]
    assert np.array_equal(out, ref.double().numpy())
    assert out[0, 0] != 127 * 0.1  # not the exact real product


def test_brute_force_loops_on_a_tiny_head():
    """The oracle against explicit scalar loops over the canonical bytes (V=8, D=128, g=64,
    N=3, r_c=r_r=2): each logit is sum_d h_d (q c S + sum_j Ac Bc + sum_j Aw Bw), every
    factor entry the single-precision product of its INT8 value and scale (ARCHead Sec. 3,
    the packed head and the logit formula)."""
    import struct

    V, D, g, N, rc, rr = 8, 128, 64, 3, 2, 2
    head = random_canonical_head(V, D, rc, rr, g, seed=99, zero_rows=1, zero_groups=1)
    rng = np.random.default_rng(7)
    Hf = rng.standard_normal((N, D)).astype(np.float32)
    Hb = (Hf.view(np.uint32) >> 16).astype(np.uint16)  # truncate to BF16 bit patterns

    def bf16(b):
        return struct.unpack("<f", struct.pack("<I", int(b) << 16))[0]

    def f32(x):
        return struct.unpack("<f", struct.pack("<f", x))[0]

    def int4(v, d):
        byte = int(head["r_nib"][v, d // 2])
        nib = (byte >> (4 * (d % 2))) & 0xF
        return nib - 16 if nib >= 8 else nib

    def factor(a, s):  # one IEEE-single product
        return f32(float(a) * float(s))

    Y = np.zeros((N, V))
    for n in range(N):
        for v in range(V):
            acc = 0.0
            for d in range(D):
                w = float(int4(v, d)) * float(head["r_code"][v, d // g]) * bf16(head["r_super"][v])
                for j in range(rc):
                    w += factor(head["Ac"][v, j], head["sAc"][v]) * \
                        factor(head["Bc"][j, d], head["sBc"][j, d // g])
                for j in range(rr):
                    w += factor(head["Aw"][v, j], head["sAw"][v]) * \
                        factor(head["Bw"][j, d], head["sBw"][j, d // g])
                acc += bf16(Hb[n, d]) * w
            Y[n, v] = acc
    Yo = oracle.logits(head, Hb)
    assert np.max(np.abs(Yo - Y)) <= 1e-12 * max(1.0, np.max(np.abs(Y)))


@pytest.mark.parametrize("V,D,r_c,r_r,g", [(1000, 512, 8, 8, 64), (300, 1024, 0, 0, 128),
                                           (257, 256, 3, 0, 32), (129, 512, 1, 7, 256)])
def test_packed_nbytes_closed_form(V, D, r_c, r_r, g):
    """Sec. 3 storage: the serialised module holds the INT4 residual (half a byte per
    entry), one UINT8 code per g entries, one BF16 super-scale per row, the INT8 factors
    (V + D)(r_c + r_r) bytes, an FP32 scale per factor row of A and per g entries of a row
    of B -- and no dense head."""
    head = random_canonical_head(V, D, r_c, r_r, g, seed=V)
    closed = (V * D // 2 + V * D // g + 2 * V + (V + D) * (r_c + r_r)
              + 4 * (2 * V + (r_c + r_r) * D // g))
    assert oracle.packed_nbytes(head) == closed
    # against the dense BF16 head: INT4 plus its code and super-scale overheads
    assert oracle.packed_nbytes(head) < 2 * V * D


# ---------------------------------------------------------------------------------------
# agreement with a dense head (Sec. 5, Table 8: top-1 / top-k agreement and KL)
# ---------------------------------------------------------------------------------------
def test_topk_ids_order_and_ties():
    y = np.array([[1.0, 3.0, 3.0, -2.0, 3.0, 0.5],
                  [0.0, 0.0, 0.0, 0.0, 0.0, 0.0]])
    assert oracle.topk_ids(y, 4).tolist() == [[1, 2, 4, 0], [0, 1, 2, 3]]
    assert oracle.topk_ids(y[:, :2], 4).tolist() == [[1, 0, -1, -1], [0, 1, -1, -1]]


def test_kl_matches_torch_and_its_special_cases():
    rng = np.random.default_rng(3)
    yd = rng.normal(size=(5, 50)) * 3
    yp = yd + rng.normal(size=(5, 50)) * 0.3
    ours = oracle.kl_dense_packed(yd, yp)
    ref = torch.nn.functional.kl_div(torch.log_softmax(torch.tensor(yp), 1),
                                     torch.log_softmax(torch.tensor(yd), 1), log_target=True,
                                     reduction="none").sum(1).numpy()
    assert np.allclose(ours, ref, rtol=1e-10, atol=1e-12)
    assert np.all(ours > 0)
    assert np.allclose(oracle.kl_dense_packed(yd, yd), 0.0, atol=1e-12)
    # a constant added to either row changes neither distribution
    assert np.allclose(oracle.kl_dense_packed(yd + 7.0, yp - 3.0), ours, atol=1e-12)
    # two logits: closed form p log(p / q) + (1 - p) log((1 - p) / (1 - q))
    d = np.array([[0.0, math.log(3.0)]])  # p = (1/4, 3/4)
    q = np.array([[0.0, 0.0]])            # q = (1/2, 1/2)
    closed = 0.25 * math.log(0.5) + 0.75 * math.log(1.5)
    assert abs(oracle.kl_dense_packed(d, q)[0] - closed) < 1e-14


def test_agreement_of_a_head_with_its_own_logits():
    head = random_canonical_head(70, 128, 2, 2, 64, seed=4)
    Hb = np.asarray(torch.randn(3, 128).to(torch.bfloat16).view(torch.int16).numpy()).view(np.uint16)
    yp = oracle.logits(head, Hb)
    a = oracle.agreement(head, Hb, yp, 5)
    assert np.array_equal(a["top1_dense"], a["topk"][:, 0])
    assert np.allclose(a["kl"], 0.0, atol=1e-12)
    from scipy.special import logsumexp
    assert np.allclose(a["lse"], logsumexp(yp, axis=1), rtol=1e-12)


def test_row8_head_single_entries_and_integer_matmul():
    """The Row INT8 baseline (Sec. 5): W[v, d] = q8[v, d] * s[v].  A single nonzero entry
    lands at its row and column with its row's scale; unit scales reduce the logits to an
    exact integer matmul."""
    V, D = 5, 128
    q8 = np.zeros((V, D), np.int8)
    q8[3, 77] = -100
    s = np.array([1.0, 2.0, 0.5, 0.25, 4.0], np.float32)
    head = {"format": "row8", "V": V, "D": D, "r_c": 0, "r_r": 0, "g": 128, "q8": q8, "row_scale": s}
    W = oracle.dense_head_rows(head)
    expect = np.zeros((V, D))
    expect[3, 77] = -25.0
    assert np.array_equal(W, expect)
    Hb = _identity_H(D)
    assert np.array_equal(oracle.logits(head, Hb), expect.T)
    rng = np.random.default_rng(0)
    q8 = rng.integers(-127, 128, size=(40, 256)).astype(np.int8)
    head = {"format": "row8", "V": 40, "D": 256, "r_c": 0, "r_r": 0, "g": 128, "q8": q8,
            "row_scale": np.ones(40, np.float32)}
    hi = rng.integers(-20, 21, size=(3, 256))
    Hb = _bf16_bits_of(hi.astype(np.float32))
    assert np.array_equal(oracle.logits(head, Hb), (hi @ q8.astype(np.int64).T).astype(np.float64))
