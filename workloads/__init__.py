"""Seeded synthetic inputs for the ARCHead packed LM-head logit path.

This module holds only random-number generation and the workload presets. It holds none
of the method's arithmetic: no quantisation, no metric transform, no logit evaluation.
Both the product package (benchmark, construction inputs) and the test-only oracle draw
their inputs from here, so the two sides see identical bytes.

Workload recipe (ARCHead, arXiv 2608.02703 HTML, Sec. 3 problem statement: W is V x D,
H holds N final hidden states):

* W = U diag(sigma) V^T + noise * Z, with U (V x rank) and V (D x rank) orthonormal
  (QR of a Gaussian), sigma_i = sigma0 / i, Z ~ N(0, 1).
* H = Z diag(s): Z ~ N(0, 1); s_d ~ LogNormal(0, sigma_s); k outlier channels, chosen by a
  seeded permutation, get s_d *= m.  Calibration and evaluation rows share s and the
  outlier set (same distribution) with independent Z.  Generated in fp32, cast to BF16
  with round-to-nearest-even.
* targets: int32 token ids uniform in [0, V).
* random_canonical_head: arbitrary packed-head bytes (uniform nibbles, codes, INT8 factors,
  positive scales).  The logit path must agree with the oracle on any packed bytes, not
  only on heads the construction produced.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np
import torch

__all__ = [
    "Workload",
    "WORKLOADS",
    "make_weight",
    "make_channel_scales",
    "make_hidden",
    "make_targets",
    "random_canonical_head",
    "bf16_bits",
]


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic head: shapes, generator parameters and packing parameters."""

    name: str
    index: int
    V: int
    D: int
    Ns: tuple  # token counts evaluated on this head
    r_c: int
    r_r: int
    g: int
    p: float
    lam: float
    n_cal: int
    rank: int = 64
    sigma0: float = 0.5
    noise: float = 0.02
    sigma_s: float = 0.5
    n_outliers: int = 4
    outlier_mult: float = 20.0
    nll: bool = False

    # fixed seed families per workload
    @property
    def seed_w(self) -> int:
        return 1000 + self.index

    @property
    def seed_scales(self) -> int:
        return 2000 + self.index

    @property
    def seed_hcal(self) -> int:
        return 3000 + self.index

    @property
    def seed_heval(self) -> int:
        return 4000 + self.index

    @property
    def seed_targets(self) -> int:
        return 5000 + self.index

    @property
    def seed_rsvd(self) -> int:
        return 6000 + self.index


# The five synthetic heads.  Shapes follow the model dimensions the pages name (Qwen3-8B:
# V=151936, D=4096; a Llama-3-8B-shaped head V=128256) and the wide D=5120 head.
WORKLOADS = {
    "tiny": Workload("tiny", 0, V=4096, D=512, Ns=(16,), r_c=16, r_r=16, g=64, p=0.75,
                     lam=0.01, n_cal=512),
    "qwen_decode": Workload("qwen_decode", 1, V=151936, D=4096, Ns=(1, 4, 16, 64), r_c=32,
                            r_r=32, g=128, p=0.75, lam=0.01, n_cal=2048),
    # prefill shares the decode head (same W generator seeds and packing)
    "qwen_prefill": Workload("qwen_prefill", 1, V=151936, D=4096, Ns=(4096,), r_c=32,
                             r_r=32, g=128, p=0.75, lam=0.01, n_cal=2048),
    "llama_batched": Workload("llama_batched", 3, V=128256, D=4096, Ns=(32, 128, 256),
                              r_c=64, r_r=64, g=128, p=0.5, lam=0.05, n_cal=2048,
                              sigma_s=1.0, n_outliers=16, outlier_mult=50.0),
    "wide_nll": Workload("wide_nll", 4, V=151936, D=5120, Ns=(8192,), r_c=32, r_r=32,
                         g=128, p=0.75, lam=0.01, n_cal=2048, nll=True),
}


def _gen(seed: int, device: str = "cpu") -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def make_weight(V: int, D: int, rank: int, sigma0: float, noise: float, seed: int,
                device: str = "cpu", dtype=torch.float32) -> torch.Tensor:
    """Dense synthetic head W (V x D): decaying-spectrum rank part plus Gaussian noise."""
    gen = _gen(seed, device)
    rank = min(rank, V, D)
    U = torch.randn(V, rank, generator=gen, device=device, dtype=torch.float32)
    Vt = torch.randn(D, rank, generator=gen, device=device, dtype=torch.float32)
    U, _ = torch.linalg.qr(U)
    Vt, _ = torch.linalg.qr(Vt)
    sig = sigma0 / torch.arange(1, rank + 1, device=device, dtype=torch.float32)
    W = torch.randn(V, D, generator=gen, device=device, dtype=torch.float32)
    W.mul_(noise)
    W.addmm_(U * sig, Vt.t())
    return W.to(dtype)


def make_channel_scales(D: int, sigma_s: float, n_outliers: int, outlier_mult: float,
                        seed: int) -> torch.Tensor:
    """Per-channel scales s_d ~ LogNormal(0, sigma_s), with seeded outlier channels."""
    gen = _gen(seed)
    s = torch.exp(sigma_s * torch.randn(D, generator=gen, dtype=torch.float32))
    idx = torch.randperm(D, generator=gen)[:n_outliers]
    s[idx] *= outlier_mult
    return s


def make_hidden(N: int, scales: torch.Tensor, seed: int, device: str = "cpu") -> torch.Tensor:
    """Hidden states H = Z diag(s) as BF16 (N x D), Z ~ N(0, 1) in fp32."""
    gen = _gen(seed, device)
    Z = torch.randn(N, scales.numel(), generator=gen, device=device, dtype=torch.float32)
    return (Z * scales.to(device)).to(torch.bfloat16)


def make_targets(N: int, V: int, seed: int, device: str = "cpu") -> torch.Tensor:
    """Target token ids, uniform in [0, V), int32."""
    gen = _gen(seed, device)
    return torch.randint(0, V, (N,), generator=gen, device=device, dtype=torch.int64).to(
        torch.int32)


def bf16_bits(x: torch.Tensor) -> np.ndarray:
    """The raw 16-bit patterns of a BF16 tensor, as a uint16 numpy array (CPU copy)."""
    return x.detach().to("cpu").contiguous().view(torch.int16).numpy().view(np.uint16)


def random_canonical_head(V: int, D: int, r_c: int, r_r: int, g: int, seed: int,
                          zero_rows: int = 0, zero_groups: int = 0,
                          super_exp_range=(-14, -4), factor_exp_range=(-9, -5)) -> dict:
    """Arbitrary packed-head bytes in the canonical layout (random, not constructed).

    Layout (per row v, little-endian bytes):
      r_nib   uint8  V x D/2   byte v,b holds column 2b in its low nibble, 2b+1 in its high
                               nibble; a nibble is a two's-complement INT4 in [-8, 7]
      r_code  uint8  V x D/g   group-scale code of columns [k*g, (k+1)*g)
      r_super uint16 V         BF16 bit pattern of the per-row super-scale
      Ac int8 V x r_c, sAc f32 V ;  Bc int8 r_c x D, sBc f32 r_c x D/g
      Aw int8 V x r_r, sAw f32 V ;  Bw int8 r_r x D, sBw f32 r_r x D/g
    zero_rows rows get an all-zero residual (super-scale 0, codes 0); zero_groups random
    groups get code 0.  INT8 values are drawn from [-127, 127].  Super-scales are
    2^e (1 + m/128) with e uniform in super_exp_range; INT8 scales are 2^u with u uniform in
    factor_exp_range (these two ranges set the logit magnitude).
    """
    rng = np.random.default_rng(seed)
    G = D // g
    head = {
        "V": V, "D": D, "r_c": r_c, "r_r": r_r, "g": g,
        "r_nib": rng.integers(0, 256, size=(V, D // 2), dtype=np.uint8),
        "r_code": rng.integers(0, 256, size=(V, G), dtype=np.uint8),
    }
    # positive BF16 super-scales 2^e * (1 + m/128)
    e = rng.integers(super_exp_range[0], super_exp_range[1] + 1, size=V)
    m = rng.integers(0, 128, size=V)
    sup = ((e + 127).astype(np.uint32) << 7) | m.astype(np.uint32)
    head["r_super"] = sup.astype(np.uint16)

    def i8(shape):
        return rng.integers(-127, 128, size=shape, dtype=np.int64).astype(np.int8)

    def pos_f32(shape, lo=factor_exp_range[0], hi=factor_exp_range[1]):
        return (2.0 ** rng.uniform(lo, hi, size=shape)).astype(np.float32)

    head["Ac"] = i8((V, r_c))
    head["sAc"] = pos_f32((V,))
    head["Bc"] = i8((r_c, D))
    head["sBc"] = pos_f32((r_c, G))
    head["Aw"] = i8((V, r_r))
    head["sAw"] = pos_f32((V,))
    head["Bw"] = i8((r_r, D))
    head["sBw"] = pos_f32((r_r, G))
    if zero_rows:
        rows = rng.choice(V, size=min(zero_rows, V), replace=False)
        head["r_super"][rows] = 0
        head["r_code"][rows] = 0
    if zero_groups:
        rows = rng.integers(0, V, size=zero_groups)
        cols = rng.integers(0, G, size=zero_groups)
        head["r_code"][rows, cols] = 0
    return head


def head_nbytes(head: dict) -> int:
    """Persistent bytes of a canonical head: the sum over its stored arrays."""
    return int(sum(v.nbytes for v in head.values() if isinstance(v, np.ndarray)))


def dense_bf16_nbytes(V: int, D: int) -> int:
    return 2 * V * D


def hidden_for(w: Workload, N: int, device: str = "cpu", calibration: bool = False,
               scales: Optional[torch.Tensor] = None) -> torch.Tensor:
    s = scales if scales is not None else make_channel_scales(
        w.D, w.sigma_s, w.n_outliers, w.outlier_mult, w.seed_scales)
    seed = w.seed_hcal if calibration else w.seed_heval
    return make_hidden(N, s, seed, device)
