"""ARCHead construction: dense head + calibration activations -> canonical packed head.

Offline step (ARCHead, arXiv 2608.02703 HTML, Sec. 3 and Algorithm 1): it runs once per
head, before inference, and is not part of the logit path.  It is written with torch
tensor ops so that it runs on the CPU (small heads, tests) or on a GPU (full-size heads),
in fp64 by default.

Steps, in the order Algorithm 1 gives them:

 1. C = H^T H / N, c_bar = mean diag(C), C_lam = C + lam * c_bar * I      (Sec. 3.1)
 2. quantized core: rank-r_c truncated SVD of W -> A_c = U S, B_c = V^T;
    Q8 both (A_c one scale per row, B_c one per group of g along D);
    R = W - Q8(A_c) Q8(B_c); SC4(R); W_d = Q8(A_c) Q8(B_c) + SC4(R)        (Sec. 3, Eq. 3)
 3. E = W - W_d
 4. C_lam = Q Lam Q^T; T_p = Q Lam^p Q^T and T_p^-1 = Q Lam^-p Q^T         (Sec. 3.1, Eq. 2)
 5. E~ = E T_p; rank-r_r randomized truncated SVD E~ ~ U S V^T
 6. map back: A_w = U S, B_w = V^T T_p^-1
 7. Q8: A_w row-wise, B_w group-wise (g along D)                           (Sec. 3)

Quantizers (the pages name them, their formulas were lost; plainest reading):

 * Q8 group: s = max|x| / 127 over the group, stored FP32; q = clamp(rne(x / s), -127, 127);
   an all-zero group has s = 0 and q = 0.
 * SC4 residual (signed INT4 with quantized group scales): per row, group amplitude
   a_k = max|R| over group k; BF16 super-scale S = bf16_rne(max_k a_k / (7 * 255)); UINT8
   code c_k = clamp(rne(a_k / (7 S)), 1, 255) (0 when a_k = 0); nibble
   q = clamp(rne(R / (c_k S)), -8, 7).  Dequantised entry: q * c_k * S.

Canonical layout: see `workloads.random_canonical_head` (same keys, same byte order).
"""
from __future__ import annotations

from typing import Optional

import numpy as np
import torch

__all__ = ["build_head", "q8_rowwise", "q8_groupwise", "sc4", "pack_nibbles",
           "metric_transform", "randomized_svd", "dequant_head_torch", "storage_ratio",
           "save_head", "load_head", "serialized_nbytes", "shard_rows", "build_row8_head"]


def _rne(x: torch.Tensor) -> torch.Tensor:
    # torch.round rounds half to even
    return torch.round(x)


def q8_rowwise(X: torch.Tensor):
    """Symmetric INT8 with one FP32 scale per row.  Returns (q int8, s fp32, deq)."""
    amax = X.abs().amax(dim=1)
    s32 = (amax / 127.0).to(torch.float32)
    s = s32.to(X.dtype)
    safe = torch.where(s > 0, s, torch.ones_like(s))
    q = torch.clamp(_rne(X / safe[:, None]), -127, 127)
    q = torch.where(s[:, None] > 0, q, torch.zeros_like(q))
    q8 = q.to(torch.int8)
    deq = (q8.to(torch.float32) * s32[:, None]).to(X.dtype)
    return q8, s32, deq


def q8_groupwise(X: torch.Tensor, g: int):
    """Symmetric INT8 with one FP32 scale per group of g columns.  Returns (q, s, deq)."""
    rows, D = X.shape
    Xg = X.reshape(rows, D // g, g)
    amax = Xg.abs().amax(dim=2)
    s32 = (amax / 127.0).to(torch.float32)
    s = s32.to(X.dtype)
    safe = torch.where(s > 0, s, torch.ones_like(s))
    q = torch.clamp(_rne(Xg / safe[..., None]), -127, 127)
    q = torch.where(s[..., None] > 0, q, torch.zeros_like(q))
    q8 = q.to(torch.int8).reshape(rows, D)
    deq = (q8.reshape(rows, D // g, g).to(torch.float32) * s32[..., None]).reshape(rows, D)
    return q8, s32, deq.to(X.dtype)


def sc4(R: torch.Tensor, g: int):
    """SC4 residual quantizer.  Returns (q int8 in [-8, 7], code uint8, super bf16, deq)."""
    V, D = R.shape
    G = D // g
    Rg = R.reshape(V, G, g)
    a = Rg.abs().amax(dim=2)                                   # V x G
    S_bf = (a.amax(dim=1) / (7.0 * 255.0)).to(torch.bfloat16)  # RNE cast
    S = S_bf.to(R.dtype)
    S_safe = torch.where(S > 0, S, torch.ones_like(S))
    c = torch.clamp(_rne(a / (7.0 * S_safe[:, None])), 1, 255)
    c = torch.where((a > 0) & (S[:, None] > 0), c, torch.zeros_like(c))
    step = c * S[:, None]                                      # V x G
    step_safe = torch.where(step > 0, step, torch.ones_like(step))
    q = torch.clamp(_rne(Rg / step_safe[..., None]), -8, 7)
    q = torch.where(step[..., None] > 0, q, torch.zeros_like(q))
    deq = (q * step[..., None]).reshape(V, D)
    return q.to(torch.int8).reshape(V, D), c.to(torch.uint8), S_bf, deq


def pack_nibbles(q: torch.Tensor) -> torch.Tensor:
    """Signed INT4 (V x D, int8 in [-8, 7]) -> bytes (V x D/2): even column in the low nibble."""
    u = (q.to(torch.int16) & 0xF).to(torch.uint8)
    return u[:, 0::2] | (u[:, 1::2] << 4)


def metric_transform(H_cal: torch.Tensor, lam: float, p: float, dtype=torch.float64):
    """T_p = Q Lam^p Q^T and its inverse for C_lam = H^T H / N + lam * mean(diag C) * I."""
    Hc = H_cal.to(dtype)
    N = Hc.shape[0]
    C = Hc.t() @ Hc / N
    cbar = torch.diagonal(C).mean()
    C_lam = C + lam * cbar * torch.eye(C.shape[0], dtype=dtype, device=C.device)
    evals, Q = torch.linalg.eigh(C_lam)
    evals = torch.clamp(evals, min=torch.finfo(dtype).tiny)
    T = (Q * evals.pow(p)) @ Q.t()
    Tinv = (Q * evals.pow(-p)) @ Q.t()
    return T, Tinv, C, C_lam


def randomized_svd(A: torch.Tensor, r: int, seed: int, oversample: int = 10,
                   power_iters: int = 4):
    """Halko-style randomized truncated SVD with QR re-orthonormalisation between passes."""
    m, n = A.shape
    k = min(r + oversample, m, n)
    gen = torch.Generator(device=A.device)
    gen.manual_seed(int(seed))
    Om = torch.randn(n, k, generator=gen, device=A.device, dtype=A.dtype)
    Qm, _ = torch.linalg.qr(A @ Om)
    for _ in range(power_iters):
        Z, _ = torch.linalg.qr(A.t() @ Qm)
        Qm, _ = torch.linalg.qr(A @ Z)
    Bs = Qm.t() @ A
    Ub, S, Vt = torch.linalg.svd(Bs, full_matrices=False)
    U = Qm @ Ub
    return U[:, :r], S[:r], Vt[:r]


def _truncated_svd(A: torch.Tensor, r: int, seed: int, exact: bool):
    if exact:
        U, S, Vt = torch.linalg.svd(A, full_matrices=False)
        return U[:, :r], S[:r], Vt[:r]
    return randomized_svd(A, r, seed)


def build_head(W: torch.Tensor, H_cal: torch.Tensor, r_c: int, r_r: int, g: int,
               p: float, lam: float, seed: int = 0, exact_svd: bool = False,
               dtype=torch.float64, return_intermediates: bool = False):
    """Algorithm 1.  Returns the canonical head (dict of numpy arrays + shape metadata).

    W: V x D dense head (any float dtype, any device); H_cal: N_cal x D activations.
    With return_intermediates=True also returns a dict of the unquantized stages
    (T, Tinv, W_d, E, Aw_f, Bw_f) for the construction's invariant tests.
    """
    V, D = W.shape
    if D % g:
        raise ValueError(f"D={D} is not a multiple of g={g}")
    dev = W.device
    Wd = W.to(dtype)
    # quantized core
    if r_c > 0:
        U, S, Vt = _truncated_svd(Wd, r_c, seed, exact_svd)
        Ac_q, sAc, Ac_dq = q8_rowwise(U * S)
        Bc_q, sBc, Bc_dq = q8_groupwise(Vt.contiguous(), g)
        core = Ac_dq @ Bc_dq
        del U, S, Vt
    else:
        Ac_q = torch.zeros(V, 0, dtype=torch.int8, device=dev)
        sAc = torch.zeros(V, dtype=torch.float32, device=dev)
        Bc_q = torch.zeros(0, D, dtype=torch.int8, device=dev)
        sBc = torch.zeros(0, D // g, dtype=torch.float32, device=dev)
        core = torch.zeros_like(Wd)
    R = Wd - core
    q4, code, sup, r_dq = sc4(R, g)
    del R
    W_d = core
    W_d += r_dq
    del r_dq
    E = Wd - W_d
    # activation-metric correction
    T, Tinv, _, _ = metric_transform(H_cal.to(dev), lam, p, dtype)
    if r_r > 0:
        Et = E @ T
        U, S, Vt = _truncated_svd(Et, r_r, seed + 1, exact_svd)
        del Et
        Aw_f = U * S
        Bw_f = Vt @ Tinv
        Aw_q, sAw, _ = q8_rowwise(Aw_f)
        Bw_q, sBw, _ = q8_groupwise(Bw_f.contiguous(), g)
    else:
        Aw_f = torch.zeros(V, 0, dtype=dtype, device=dev)
        Bw_f = torch.zeros(0, D, dtype=dtype, device=dev)
        Aw_q = torch.zeros(V, 0, dtype=torch.int8, device=dev)
        sAw = torch.zeros(V, dtype=torch.float32, device=dev)
        Bw_q = torch.zeros(0, D, dtype=torch.int8, device=dev)
        sBw = torch.zeros(0, D // g, dtype=torch.float32, device=dev)

    def np_(t):
        return t.detach().to("cpu").contiguous().numpy()

    head = {
        "V": int(V), "D": int(D), "r_c": int(r_c), "r_r": int(r_r), "g": int(g),
        "r_nib": np_(pack_nibbles(q4)),
        "r_code": np_(code),
        "r_super": np_(sup.view(torch.int16)).view(np.uint16),
        "Ac": np_(Ac_q), "sAc": np_(sAc), "Bc": np_(Bc_q), "sBc": np_(sBc),
        "Aw": np_(Aw_q), "sAw": np_(sAw), "Bw": np_(Bw_q), "sBw": np_(sBw),
    }
    if return_intermediates:
        inter = {"T": T, "Tinv": Tinv, "W_d": W_d, "E": E, "Aw_f": Aw_f, "Bw_f": Bw_f,
                 "q4": q4, "code": code, "super": sup}
        return head, inter
    return head


def build_row8_head(W: torch.Tensor, g: int = 128) -> dict:
    """The Row INT8 baseline head the paper compares with (Sec. 5, Tables 3 and 8): every
    row of W quantized to INT8 with its own FP32 scale (the row-wise Q8 above: absmax / 127,
    round to nearest even, clamp to +-127), no core and no correction.  `g` is recorded only
    as the nominal group size the library's argument checks expect."""
    V, D = W.shape
    q, s, _ = q8_rowwise(W.to(torch.float64))
    return {"format": "row8", "V": int(V), "D": int(D), "r_c": 0, "r_r": 0, "g": int(g),
            "q8": q.detach().cpu().contiguous().numpy(),
            "row_scale": s.detach().cpu().contiguous().numpy()}


def dequant_head_torch(head: dict, device="cpu", dtype=torch.float64) -> torch.Tensor:
    """Dense W_hat from a canonical head with torch ops (construction-side diagnostics)."""
    g = head["g"]
    nib = torch.from_numpy(head["r_nib"]).to(device)
    lo = (nib & 0xF).to(torch.int16)
    hi = (nib >> 4).to(torch.int16)
    lo = torch.where(lo >= 8, lo - 16, lo)
    hi = torch.where(hi >= 8, hi - 16, hi)
    q = torch.stack([lo, hi], dim=2).reshape(nib.shape[0], -1).to(dtype)
    code = torch.from_numpy(head["r_code"]).to(device).to(dtype)
    S = torch.from_numpy(head["r_super"].view(np.int16)).to(device).view(torch.bfloat16)
    W = q * code.repeat_interleave(g, dim=1) * S.to(dtype)[:, None]

    def rowq(a, s):
        return (torch.from_numpy(a).to(device).float() * torch.from_numpy(s).to(device)[:, None]).to(dtype)

    def grpq(b, s):
        b = torch.from_numpy(b).to(device).float()
        s = torch.from_numpy(s).to(device).repeat_interleave(g, dim=1)
        return (b * s).to(dtype)

    if head["r_c"]:
        W += rowq(head["Ac"], head["sAc"]) @ grpq(head["Bc"], head["sBc"])
    if head["r_r"]:
        W += rowq(head["Aw"], head["sAw"]) @ grpq(head["Bw"], head["sBw"])
    return W


def storage_ratio(head: dict) -> float:
    """Persistent bytes over the BF16 dense head's bytes."""
    keys = (("q8", "row_scale") if head.get("format") == "row8" else
            ("r_nib", "r_code", "r_super", "Ac", "sAc", "Bc", "sBc", "Aw", "sAw", "Bw", "sBw"))
    nb = sum(np.asarray(head[k]).nbytes for k in keys)
    return nb / (2.0 * head["V"] * head["D"])


# V-indexed arrays of the canonical head (rows of the vocabulary); the B factors and their
# scales are indexed by factor and column and are shared by every row.
_ROW_KEYS = ("r_nib", "r_code", "r_super", "Ac", "sAc", "Aw", "sAw")


def shard_rows(head: dict, v0: int, v1: int) -> dict:
    """Rows [v0, v1) of a canonical packed head: the vocabulary shard one GPU holds when
    the logits or the NLL are evaluated vocabulary-parallel.  The row-indexed arrays are
    sliced and the B factors shared; the result is a canonical head with V = v1 - v0."""
    V = int(head["V"])
    if not 0 <= v0 < v1 <= V:
        raise ValueError(f"row range [{v0}, {v1}) outside [0, {V})")
    out = dict(head)
    out["V"] = v1 - v0
    for k in _ROW_KEYS:
        out[k] = np.ascontiguousarray(head[k][v0:v1])
    return out


# ---------------------------------------------------------------------------------------
# The serialised module (Sec. 3: storage is measured over every parameter and buffer the
# serialised module holds).  File layout, little-endian:
#   8 bytes   magic b"ARCHEAD1"
#   8 bytes   uint64 length L of the JSON header
#   L bytes   JSON: {"meta": {V, D, r_c, r_r, g}, "arrays": [[key, dtype, shape, offset,
#             nbytes], ...]}, offsets counted from the start of the data section
#   padding   to a multiple of 16 bytes, then the data section: every array's raw bytes
#             (C order), each starting on a 16-byte boundary
# Loading returns arrays whose bytes equal the saved ones.
# ---------------------------------------------------------------------------------------
_MAGIC = b"ARCHEAD1"
_HEAD_KEYS = ("r_nib", "r_code", "r_super", "Ac", "sAc", "Bc", "sBc", "Aw", "sAw", "Bw", "sBw")
_META_KEYS = ("V", "D", "r_c", "r_r", "g")


def _layout(head: dict):
    entries, off = [], 0
    for k in _HEAD_KEYS:
        a = np.ascontiguousarray(head[k])
        entries.append([k, a.dtype.str, list(a.shape), off, int(a.nbytes)])
        off += (a.nbytes + 15) // 16 * 16
    return entries, off


def save_head(head: dict, path: str) -> int:
    """Write the canonical packed head to `path`; returns the file size in bytes."""
    import json
    entries, data_bytes = _layout(head)
    hdr = json.dumps({"meta": {k: int(head[k]) for k in _META_KEYS}, "arrays": entries},
                     separators=(",", ":")).encode()
    pre = len(_MAGIC) + 8 + len(hdr)
    pad = (-pre) % 16
    with open(path, "wb") as f:
        f.write(_MAGIC)
        f.write(np.uint64(len(hdr)).tobytes())
        f.write(hdr)
        f.write(b"\0" * pad)
        for k, _, _, off, nb in entries:
            a = np.ascontiguousarray(head[k])
            f.write(a.tobytes())
            f.write(b"\0" * ((nb + 15) // 16 * 16 - nb))
    return pre + pad + data_bytes


def load_head(path: str) -> dict:
    """Read a head written by save_head (the arrays are copies of the saved bytes)."""
    import json
    with open(path, "rb") as f:
        if f.read(8) != _MAGIC:
            raise ValueError(f"{path}: not a packed head file")
        n = int(np.frombuffer(f.read(8), dtype=np.uint64)[0])
        hdr = json.loads(f.read(n).decode())
        f.read((-(16 + n)) % 16)
        data = f.read()
    head = {k: int(v) for k, v in hdr["meta"].items()}
    for k, dt, shape, off, nb in hdr["arrays"]:
        if off + nb > len(data):
            raise ValueError(f"{path}: truncated at array {k}")
        head[k] = np.frombuffer(data[off:off + nb], dtype=np.dtype(dt)).reshape(shape).copy()
    return head


def serialized_nbytes(head: dict) -> int:
    """Size of the file save_head writes for this head (header and padding included)."""
    import json
    entries, data_bytes = _layout(head)
    hdr = json.dumps({"meta": {k: int(head[k]) for k in _META_KEYS}, "arrays": entries},
                     separators=(",", ":")).encode()
    pre = len(_MAGIC) + 8 + len(hdr)
    return pre + (-pre) % 16 + data_bytes
