"""ARCHead packed LM-head logits on NVIDIA B200 (sm_100a).

The GPU path is libarchead.so (include/archead.h); this module only marshals torch
tensors (device memory, streams) into its C ABI.  Every step of the logit and NLL path
runs in the library's CUDA kernels; there is no CPU fallback, and calling a GPU entry
point without the built library raises.

    head  = pack.build_head(W, H_cal, r_c, r_r, g, p, lam)     # offline, Algorithm 1
    dh    = DeviceHead.from_canonical(head, "cuda")             # upload + repack
    Y     = logits(H_bf16, dh)                                  # N x V float32
    nlls  = nll(H_bf16, dh, targets)                            # N float32, no logits
"""
from __future__ import annotations

import ctypes
from typing import Optional

import numpy as np
import torch

from . import _lib, pack
from ._lib import ArcheadError, ArcheadHead

__all__ = ["DeviceHead", "logits", "nll", "agreement", "logits_host", "nll_host", "dequant", "check",
           "last_launches", "profile", "profile_read", "ArcheadError", "pack"]

_KEYS = ("r_nib", "r_code", "r_super", "Ac", "sAc", "Bc", "sBc", "Aw", "sAw", "Bw", "sBw")


def _stream_handle(stream: Optional[torch.cuda.Stream]) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    if t is None or t.numel() == 0:
        return None
    return t.data_ptr()


FMT_SC4, FMT_ROW8 = 0, 1  # archead_format


class DeviceHead:
    """A head resident in device memory: the packed ARCHead head in the library's device
    layout, or (format "row8") the Row INT8 baseline head."""

    def __init__(self, meta: dict, tensors: dict):
        self.V, self.D = int(meta["V"]), int(meta["D"])
        self.r_c, self.r_r, self.g = int(meta["r_c"]), int(meta["r_r"]), int(meta["g"])
        self.format = FMT_ROW8 if meta.get("format") == "row8" else FMT_SC4
        self.tensors = tensors  # keeps the device buffers alive
        s = ArcheadHead()
        s.V, s.D, s.r_c, s.r_r, s.g = self.V, self.D, self.r_c, self.r_r, self.g
        s.format = self.format
        for k in _KEYS:
            setattr(s, k, _ptr(tensors.get(k)))
        s.row_scale = _ptr(tensors.get("row_scale"))
        self.struct = s

    @property
    def shape_args(self):
        return (self.V, self.D, self.r_c, self.r_r, self.g)

    def nbytes(self) -> int:
        return int(sum(t.numel() * t.element_size() for t in self.tensors.values()))

    @classmethod
    def from_canonical(cls, head: dict, device="cuda", stream=None) -> "DeviceHead":
        dev = torch.device(device)
        if head.get("format") == "row8":  # INT8 V x D row-major and FP32 row scales
            up = {"r_nib": torch.from_numpy(np.ascontiguousarray(head["q8"]).view(np.uint8)).to(dev),
                  "row_scale": torch.from_numpy(np.ascontiguousarray(head["row_scale"])).to(dev)}
            return cls(head, up)
        up = {}
        Vpad = (int(head["V"]) + 127) // 128 * 128
        for k in _KEYS:
            a = np.ascontiguousarray(head[k])
            if k == "r_code" and a.shape[0] != Vpad:
                # the device code array holds whole 128-row tiles (rows >= V are zero)
                a = np.concatenate([a, np.zeros((Vpad - a.shape[0], a.shape[1]), a.dtype)])
            if a.dtype == np.uint16:
                t = torch.from_numpy(a.view(np.int16))
            else:
                t = torch.from_numpy(a)
            up[k] = t.to(dev, non_blocking=False)
        canon = up["r_nib"]
        V, D = int(head["V"]), int(head["D"])
        # device layout: rows padded to a multiple of 128 (see archead_repack_residual)
        devnib = torch.empty((V + 127) // 128 * 128, D // 2, dtype=torch.uint8, device=dev)
        st = _stream_handle(stream)
        _lib.check(_lib.lib().archead_repack_residual(canon.data_ptr(), devnib.data_ptr(),
                                                      int(head["V"]), int(head["D"]), st),
                   "archead_repack_residual")
        torch.cuda.current_stream(dev).synchronize() if stream is None else stream.synchronize()
        up["r_nib"] = devnib
        return cls(head, up)


def _check_H(H: torch.Tensor, dh: DeviceHead):
    if H.dtype != torch.bfloat16 or H.dim() != 2 or H.shape[1] != dh.D:
        raise ValueError(f"H must be a bf16 N x {dh.D} tensor, got {H.dtype} {tuple(H.shape)}")
    if not H.is_cuda or not H.is_contiguous():
        raise ValueError("H must be a contiguous CUDA tensor")


def logits(H: torch.Tensor, dh: DeviceHead, out: Optional[torch.Tensor] = None,
           stream=None) -> torch.Tensor:
    """Y = H W_d^T + (H B_w^T) A_w^T (N x V float32), asynchronous on the stream."""
    _check_H(H, dh)
    N = H.shape[0]
    if out is None:
        out = torch.empty(N, dh.V, device=H.device, dtype=torch.float32)
    _lib.check(_lib.lib().archead_logits(H.data_ptr(), ctypes.byref(dh.struct),
                                         out.data_ptr() if N else None, N, *dh.shape_args,
                                         _stream_handle(stream)), "archead_logits")
    return out


def nll(H: torch.Tensor, dh: DeviceHead, targets: torch.Tensor,
        out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Per-token NLL (nats) = logsumexp(Y[n]) - Y[n, target[n]], without writing Y."""
    _check_H(H, dh)
    N = H.shape[0]
    if targets.dtype != torch.int32 or targets.shape != (N,) or not targets.is_cuda:
        raise ValueError("targets must be an int32 CUDA tensor of shape (N,)")
    if out is None:
        out = torch.empty(N, device=H.device, dtype=torch.float32)
    _lib.check(_lib.lib().archead_nll(H.data_ptr(), ctypes.byref(dh.struct),
                                      targets.contiguous().data_ptr(),
                                      out.data_ptr() if N else None, N, *dh.shape_args,
                                      _stream_handle(stream)), "archead_nll")
    return out


def nll_partials(H: torch.Tensor, dh: DeviceHead, targets: torch.Tensor, v_begin: int,
                 v_total: int, out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """archead_nll_partials: this vocabulary shard's (max, sum exp, target logit) per token
    (N x 3 float32).  dh holds rows [v_begin, v_begin + dh.V) of a v_total-row head."""
    _check_H(H, dh)
    N = H.shape[0]
    if targets.dtype != torch.int32 or targets.shape != (N,) or not targets.is_cuda:
        raise ValueError("targets must be an int32 CUDA tensor of shape (N,)")
    if out is None:
        out = torch.empty(N, 3, device=H.device, dtype=torch.float32)
    _lib.check(_lib.lib().archead_nll_partials(H.data_ptr(), ctypes.byref(dh.struct),
                                               targets.contiguous().data_ptr(), int(v_begin),
                                               int(v_total), out.data_ptr() if N else None, N,
                                               *dh.shape_args, _stream_handle(stream)),
               "archead_nll_partials")
    return out


def nll_merge(partials: torch.Tensor, out: Optional[torch.Tensor] = None,
              stream=None) -> torch.Tensor:
    """archead_nll_merge: per-token NLL from G shards' partials (G x N x 3 float32 CUDA)."""
    if (partials.dtype != torch.float32 or partials.dim() != 3 or partials.shape[2] != 3
            or not partials.is_cuda):
        raise ValueError("partials must be a float32 CUDA tensor of shape (G, N, 3)")
    G, N = int(partials.shape[0]), int(partials.shape[1])
    p = partials.contiguous()
    if out is None:
        out = torch.empty(N, device=partials.device, dtype=torch.float32)
    _lib.check(_lib.lib().archead_nll_merge(p.data_ptr(), G, N, out.data_ptr() if N else None,
                                            _stream_handle(stream)), "archead_nll_merge")
    return out


def vocab_parallel_nll(H: torch.Tensor, dh: DeviceHead, targets: torch.Tensor, v_begin: int,
                       v_total: int, group=None) -> torch.Tensor:
    """Per-token NLL of a head whose vocabulary rows are sharded over the ranks of `group`
    (rank k holds dh = rows [v_begin, v_begin + dh.V)): each rank reduces its shard to
    (max, sum exp, target logit) per token, one all-gather exchanges the N x 3 partials,
    and every rank merges them in rank order.  H and targets are the same on every rank."""
    import torch.distributed as dist
    part = nll_partials(H, dh, targets, v_begin, v_total)
    if not (dist.is_available() and dist.is_initialized()):  # one process holds the head
        return nll_merge(part[None])
    G = dist.get_world_size(group)
    if dist.get_backend(group) == "gloo":  # host collectives (tests without NCCL)
        host = part.cpu()
        gathered = [torch.empty_like(host) for _ in range(G)]
        dist.all_gather(gathered, host, group=group)
        return nll_merge(torch.stack(gathered).to(part.device))
    gathered = [torch.empty_like(part) for _ in range(G)]
    dist.all_gather(gathered, part, group=group)
    return nll_merge(torch.stack(gathered))


def agreement(H: torch.Tensor, dh: DeviceHead, Y_dense: torch.Tensor, k: int = 10,
              stream=None) -> dict:
    """archead_agreement: per token the ids of the k largest packed logits ("topk", N x k
    int32, decreasing, equal logits by smaller id), the dense argmax ("top1_dense", N),
    KL(P_dense || P_packed) in nats ("kl", N) and the packed log-sum-exp ("lse", N), all
    on the device.  Y_dense: N x V float32 reference logits on the same device."""
    _check_H(H, dh)
    N = H.shape[0]
    if (Y_dense.dtype != torch.float32 or tuple(Y_dense.shape) != (N, dh.V)
            or not Y_dense.is_cuda or not Y_dense.is_contiguous()):
        raise ValueError(f"Y_dense must be a contiguous float32 CUDA tensor of shape ({N}, {dh.V})")
    dev = H.device
    out = {"topk": torch.empty(N, k, dtype=torch.int32, device=dev),
           "top1_dense": torch.empty(N, dtype=torch.int32, device=dev),
           "kl": torch.empty(N, dtype=torch.float32, device=dev),
           "lse": torch.empty(N, dtype=torch.float32, device=dev)}
    _lib.check(_lib.lib().archead_agreement(
        H.data_ptr(), ctypes.byref(dh.struct), Y_dense.data_ptr(), int(k),
        *[out[x].data_ptr() if N else None for x in ("topk", "top1_dense", "kl", "lse")],
        N, *dh.shape_args, _stream_handle(stream)), "archead_agreement")
    return out


def logits_host(H: torch.Tensor, dh: DeviceHead, out: Optional[torch.Tensor] = None,
                stream=None) -> torch.Tensor:
    """archead_logits_host: host H in, host Y out (copies inside the call, synchronous)."""
    if H.dtype != torch.bfloat16 or H.is_cuda or not H.is_contiguous():
        raise ValueError("H must be a contiguous host bf16 tensor")
    N = H.shape[0]
    if out is None:
        out = torch.empty(N, dh.V, dtype=torch.float32, pin_memory=True)
    _lib.check(_lib.lib().archead_logits_host(H.data_ptr(), ctypes.byref(dh.struct),
                                              out.data_ptr(), N, *dh.shape_args,
                                              _stream_handle(stream)), "archead_logits_host")
    return out


def nll_host(H: torch.Tensor, dh: DeviceHead, targets: torch.Tensor,
             out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    if H.dtype != torch.bfloat16 or H.is_cuda or not H.is_contiguous():
        raise ValueError("H must be a contiguous host bf16 tensor")
    N = H.shape[0]
    if out is None:
        out = torch.empty(N, dtype=torch.float32, pin_memory=True)
    _lib.check(_lib.lib().archead_nll_host(H.data_ptr(), ctypes.byref(dh.struct),
                                           targets.contiguous().data_ptr(), out.data_ptr(),
                                           N, *dh.shape_args, _stream_handle(stream)),
               "archead_nll_host")
    return out


def dequant(dh: DeviceHead, row0: int = 0, nrows: Optional[int] = None, stream=None) -> dict:
    """FP32 dequantised components via the archead_dequant hook (for bit-exact checks)."""
    nrows = dh.V - row0 if nrows is None else nrows
    dev = dh.tensors["r_nib"].device
    out = {
        "R": torch.empty(nrows, dh.D, device=dev),
        "Ac": torch.empty(nrows, dh.r_c, device=dev),
        "Aw": torch.empty(nrows, dh.r_r, device=dev),
        "Bc": torch.empty(dh.r_c, dh.D, device=dev),
        "Bw": torch.empty(dh.r_r, dh.D, device=dev),
    }
    _lib.check(_lib.lib().archead_dequant(ctypes.byref(dh.struct), row0, nrows,
                                          *[_ptr(out[k]) for k in ("R", "Ac", "Aw", "Bc", "Bw")],
                                          _stream_handle(stream)), "archead_dequant")
    return out


def check(stream=None) -> None:
    """Synchronise the stream and raise if a kernel flagged an error (archead_check)."""
    _lib.check(_lib.lib().archead_check(_stream_handle(stream)), "archead_check")


def last_launches() -> int:
    """Kernels launched by the most recent archead_logits / archead_nll on this thread."""
    return int(_lib.lib().archead_last_launches())


def profile(enable: bool) -> None:
    """Start (clearing the record) or stop recording events around the main kernel."""
    _lib.check(_lib.lib().archead_profile(1 if enable else 0), "archead_profile")


def profile_read():
    """(total milliseconds, launches) of the main kernel since profile(True)."""
    ms = ctypes.c_double(0)
    n = ctypes.c_int(0)
    _lib.check(_lib.lib().archead_profile_read(ctypes.byref(ms), ctypes.byref(n)),
               "archead_profile_read")
    return float(ms.value), int(n.value)
