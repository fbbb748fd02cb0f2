"""CPU oracle for the ARCHead packed LM-head logit path.  TEST INFRASTRUCTURE ONLY.

Only the tests, the package's smoke check and the benchmark's CPU-baseline / reference
leg may import this module.  The GPU library never calls it and shares no code with it:
this file decodes the canonical bytes with its own plain NumPy code.

What it computes (ARCHead, arXiv 2608.02703 HTML, Sec. 3, "final approximation and
logits" and the inference statement closing Sec. 3 / Algorithm 1):

    W_d   = Q8(A_c) Q8(B_c) + SC4(R)                 (quantized core, Sec. 3 Eq. 3)
    W_hat = W_d + A_w B_w                             (final approximation)
    Y     = H W_hat^T  =  H W_d^T + (H B_w^T) A_w^T   (logits)
    nll_n = logsumexp_v Y[n, v] - Y[n, target_n]      (cross-entropy in nats, Sec. 5)
    agreement with a dense head (Sec. 5, Table 8): the packed top-k ids, the dense top-1
    id and KL(P_dense || P_packed), P = softmax of the logits

Everything is evaluated in fp64 from the exact decoded values:

* SC4 residual entry (v, d): q * c * S with q the signed INT4 nibble, c the UINT8 code of
  group d // g of row v and S the row's BF16 super-scale.  The product is an exact real
  number that also fits an IEEE single exactly (<= 20 significant bits).
* INT8 factor entry: the IEEE-single product fl32(q8 * s) of the INT8 value and its FP32
  scale (one round-to-nearest-even multiply) -- the dequantised factor in the precision
  of its stored scale.  A_c, A_w carry one scale per row; B_c, B_w one per group of g
  columns along D.
* H: the exact values of its BF16 bit patterns.

Parity pins (tests/test_oracle_pins.py): all-byte nibble decoding, single-entry heads
that fix every index and scale mapping, the r_c = r_r = 0 unit-scale case against an
exact integer matmul, the BF16 decoding against torch over all 65536 patterns, the
factored-vs-dense associativity identity, and the NLL special cases (constant logits,
shift invariance, a library cross-entropy), and for the agreement measures a library KL
divergence, exact zeros, shift invariance and hand-checked orders of tied logits.
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "bf16_bits_to_f64",
    "decode_int4_bytes",
    "unpack_residual",
    "dequant_int8_rowwise",
    "dequant_int8_groupwise",
    "dense_head_rows",
    "logits",
    "logits_factored",
    "nll_from_logits",
    "nll",
    "topk_ids",
    "kl_dense_packed",
    "agreement",
    "packed_nbytes",
]


def bf16_bits_to_f64(bits) -> np.ndarray:
    """Exact value of BF16 bit patterns: the upper half of an IEEE single."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    with np.errstate(invalid="ignore"):
        return b.view(np.float32).astype(np.float64)


def decode_int4_bytes(packed: np.ndarray) -> np.ndarray:
    """Expand packed bytes (..., K) to signed INT4 values (..., 2K), as int8.

    Byte b holds column 2b in bits 0-3 and column 2b+1 in bits 4-7; each nibble is a
    two's-complement 4-bit integer in [-8, 7].
    """
    packed = np.asarray(packed, dtype=np.uint8)
    lo = (packed & 0x0F).astype(np.int16)
    hi = (packed >> 4).astype(np.int16)
    lo = np.where(lo >= 8, lo - 16, lo)
    hi = np.where(hi >= 8, hi - 16, hi)
    out = np.empty(packed.shape[:-1] + (2 * packed.shape[-1],), dtype=np.int8)
    out[..., 0::2] = lo
    out[..., 1::2] = hi
    return out


def unpack_residual(head: dict, rows=None) -> np.ndarray:
    """SC4(R) rows as fp64: entry (v, d) = q[v, d] * code[v, d // g] * S_v."""
    g = int(head["g"])
    sl = slice(None) if rows is None else rows
    q = decode_int4_bytes(head["r_nib"][sl]).astype(np.float64)
    code = head["r_code"][sl].astype(np.float64)
    S = bf16_bits_to_f64(head["r_super"][sl])
    code_per_col = np.repeat(code, g, axis=1)
    return q * code_per_col * S[:, None]


def dequant_int8_rowwise(q8: np.ndarray, s: np.ndarray) -> np.ndarray:
    """Row-wise INT8 factor: fl32(q8[i, j] * s[i]), returned as fp64."""
    q = np.asarray(q8, dtype=np.int8).astype(np.float32)
    sc = np.asarray(s, dtype=np.float32)
    return (q * sc[:, None]).astype(np.float64)


def dequant_int8_groupwise(q8: np.ndarray, s: np.ndarray, g: int) -> np.ndarray:
    """Group-wise INT8 factor: fl32(q8[i, d] * s[i, d // g]), returned as fp64."""
    q = np.asarray(q8, dtype=np.int8).astype(np.float32)
    sc = np.repeat(np.asarray(s, dtype=np.float32), g, axis=1)
    return (q * sc).astype(np.float64)


def _factors(head: dict):
    g = int(head["g"])
    Ac = dequant_int8_rowwise(head["Ac"], head["sAc"])
    Bc = dequant_int8_groupwise(head["Bc"], head["sBc"], g)
    Aw = dequant_int8_rowwise(head["Aw"], head["sAw"])
    Bw = dequant_int8_groupwise(head["Bw"], head["sBw"], g)
    return Ac, Bc, Aw, Bw


def dense_head_rows(head: dict, rows=None) -> np.ndarray:
    """W_hat = Q8(A_c) Q8(B_c) + SC4(R) + Q8(A_w) Q8(B_w) for the given vocab rows, fp64.
    A Row INT8 head (format "row8", the paper's storage-matched baseline) gives
    W = q8 * row_scale, the product of the INT8 value and its row's FP32 scale, exact."""
    g = int(head["g"])
    sl = slice(None) if rows is None else rows
    if head.get("format") == "row8":
        q = np.asarray(head["q8"], dtype=np.int8)[sl].astype(np.float64)
        return q * np.asarray(head["row_scale"], dtype=np.float32)[sl].astype(np.float64)[:, None]
    W = unpack_residual(head, rows)
    if int(head["r_c"]) > 0:
        Ac = dequant_int8_rowwise(head["Ac"][sl], head["sAc"][sl])
        Bc = dequant_int8_groupwise(head["Bc"], head["sBc"], g)
        W = W + Ac @ Bc
    if int(head["r_r"]) > 0:
        Aw = dequant_int8_rowwise(head["Aw"][sl], head["sAw"][sl])
        Bw = dequant_int8_groupwise(head["Bw"], head["sBw"], g)
        W = W + Aw @ Bw
    return W


def logits(head: dict, H_bits: np.ndarray, rows=None, chunk: int = 16384) -> np.ndarray:
    """Y = H W_hat^T in fp64 (N x V, or N x len(rows)).

    H_bits: N x D BF16 bit patterns.  The vocabulary is visited in slices of `chunk` rows
    only to bound the memory of the dense W_hat; each logit is one full-length dot product.
    """
    H = bf16_bits_to_f64(H_bits)
    if rows is not None:
        return H @ dense_head_rows(head, rows).T
    V = int(head["V"])
    Y = np.empty((H.shape[0], V), dtype=np.float64)
    for v0 in range(0, V, chunk):
        v1 = min(V, v0 + chunk)
        Y[:, v0:v1] = H @ dense_head_rows(head, slice(v0, v1)).T
    return Y


def logits_factored(head: dict, H_bits: np.ndarray) -> np.ndarray:
    """The factored evaluation order H W_d^T + (H B_w^T) A_w^T (fp64), for the identity check."""
    H = bf16_bits_to_f64(H_bits)
    Ac, Bc, Aw, Bw = _factors(head)
    R = unpack_residual(head)
    return H @ R.T + (H @ Bc.T) @ Ac.T + (H @ Bw.T) @ Aw.T


def nll_from_logits(Y: np.ndarray, targets: np.ndarray) -> np.ndarray:
    """Per-token negative log-likelihood in nats: m + ln sum exp(Y - m) - Y[target]."""
    Y = np.asarray(Y, dtype=np.float64)
    t = np.asarray(targets, dtype=np.int64)
    m = Y.max(axis=1)
    lse = m + np.log(np.exp(Y - m[:, None]).sum(axis=1))
    return lse - Y[np.arange(Y.shape[0]), t]


def nll(head: dict, H_bits: np.ndarray, targets: np.ndarray) -> np.ndarray:
    return nll_from_logits(logits(head, H_bits), targets)


def topk_ids(y: np.ndarray, k: int) -> np.ndarray:
    """Ids of the k largest entries of each row, largest first; equal values in increasing
    id order; -1 past the row length."""
    y = np.asarray(y, dtype=np.float64)
    N, V = y.shape
    out = -np.ones((N, k), dtype=np.int64)
    for n in range(N):
        # sort by (-value, id): a stable sort of -y keeps equal values in id order
        order = np.argsort(-y[n], kind="stable")
        m = min(k, V)
        out[n, :m] = order[:m]
    return out


def kl_dense_packed(y_dense: np.ndarray, y_packed: np.ndarray) -> np.ndarray:
    """KL(P_dense || P_packed) per row in nats, P = softmax of the row's logits:
    sum_v p_d (log p_d - log p_p)."""
    yd = np.asarray(y_dense, dtype=np.float64)
    yp = np.asarray(y_packed, dtype=np.float64)
    ld = yd - (yd.max(axis=1, keepdims=True)
               + np.log(np.exp(yd - yd.max(axis=1, keepdims=True)).sum(axis=1, keepdims=True)))
    lp = yp - (yp.max(axis=1, keepdims=True)
               + np.log(np.exp(yp - yp.max(axis=1, keepdims=True)).sum(axis=1, keepdims=True)))
    return (np.exp(ld) * (ld - lp)).sum(axis=1)


def agreement(head: dict, H_bits: np.ndarray, y_dense: np.ndarray, k: int) -> dict:
    """Agreement of the packed head with dense reference logits on the same tokens (Sec. 5,
    Table 8): the packed head's top-k ids, the dense top-1 id (ties: smaller id), KL(dense
    || packed) and the packed log-sum-exp, all from the fp64 packed logits."""
    yp = logits(head, H_bits)
    yd = np.asarray(y_dense, dtype=np.float64)
    m = yp.max(axis=1)
    return {"topk": topk_ids(yp, k), "top1_dense": np.argmax(yd, axis=1),
            "kl": kl_dense_packed(yd, yp),
            "lse": m + np.log(np.exp(yp - m[:, None]).sum(axis=1)), "y_packed": yp}


def packed_nbytes(head: dict) -> int:
    """Persistent bytes: the sum of the stored arrays' sizes (no dense head among them)."""
    return int(sum(np.asarray(head[k]).nbytes for k in
                   ("r_nib", "r_code", "r_super", "Ac", "sAc", "Bc", "sBc",
                    "Aw", "sAw", "Bw", "sBw")))
