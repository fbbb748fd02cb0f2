"""ctypes binding of libarchead.so (include/archead.h).  Argument marshalling only."""
from __future__ import annotations

import ctypes
import os
import re

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libarchead.so")
HEADER = os.path.join(os.path.dirname(HERE), "include", "archead.h")

c_i64 = ctypes.c_int64
c_int = ctypes.c_int
c_vp = ctypes.c_void_p

STATUS = {
    0: "ARCHEAD_OK", -1: "ARCHEAD_ERR_NULLPTR", -2: "ARCHEAD_ERR_ALIGN",
    -3: "ARCHEAD_ERR_SHAPE", -4: "ARCHEAD_ERR_RANGE_H", -5: "ARCHEAD_ERR_TARGET",
    -6: "ARCHEAD_ERR_TIMEOUT", -7: "ARCHEAD_ERR_CUDA", -8: "ARCHEAD_ERR_UNSUPPORTED",
    -9: "ARCHEAD_ERR_NOMEM",
}
STATUS_CODE = {v: k for k, v in STATUS.items()}


class ArcheadHead(ctypes.Structure):
    _fields_ = [
        ("V", c_i64), ("D", c_i64),
        ("r_c", ctypes.c_int32), ("r_r", ctypes.c_int32), ("g", ctypes.c_int32),
        ("format", ctypes.c_int32),
        ("r_nib", c_vp), ("r_code", c_vp), ("r_super", c_vp),
        ("Ac", c_vp), ("sAc", c_vp), ("Bc", c_vp), ("sBc", c_vp),
        ("Aw", c_vp), ("sAw", c_vp), ("Bw", c_vp), ("sBw", c_vp),
        ("row_scale", c_vp),
    ]


_SIGS = {
    "archead_logits": (c_int, [c_vp, ctypes.POINTER(ArcheadHead), c_vp, c_i64, c_i64, c_i64,
                               c_int, c_int, c_int, c_vp]),
    "archead_nll": (c_int, [c_vp, ctypes.POINTER(ArcheadHead), c_vp, c_vp, c_i64, c_i64,
                            c_i64, c_int, c_int, c_int, c_vp]),
    "archead_logits_host": (c_int, [c_vp, ctypes.POINTER(ArcheadHead), c_vp, c_i64, c_i64,
                                    c_i64, c_int, c_int, c_int, c_vp]),
    "archead_nll_host": (c_int, [c_vp, ctypes.POINTER(ArcheadHead), c_vp, c_vp, c_i64, c_i64,
                                 c_i64, c_int, c_int, c_int, c_vp]),
    "archead_repack_residual": (c_int, [c_vp, c_vp, c_i64, c_i64, c_vp]),
    "archead_dequant": (c_int, [ctypes.POINTER(ArcheadHead), c_i64, c_i64, c_vp, c_vp, c_vp,
                                c_vp, c_vp, c_vp]),
    "archead_check": (c_int, [c_vp]),
    "archead_strerror": (ctypes.c_char_p, [c_int]),
    "archead_abi_version": (c_int, []),
    "archead_last_launches": (c_int, []),
    "archead_logits_noalloc": (c_int, [c_vp, ctypes.POINTER(ArcheadHead), c_vp, c_i64, c_i64,
                                       c_i64, c_int, c_int, c_int, c_vp]),
    "archead_nll_partials": (c_int, [c_vp, ctypes.POINTER(ArcheadHead), c_vp, c_i64, c_i64,
                                     c_vp, c_i64, c_i64, c_i64, c_int, c_int, c_int, c_vp]),
    "archead_nll_merge": (c_int, [c_vp, c_int, c_i64, c_vp, c_vp]),
    "archead_agreement": (c_int, [c_vp, ctypes.POINTER(ArcheadHead), c_vp, c_int, c_vp, c_vp,
                                  c_vp, c_vp, c_i64, c_i64, c_i64, c_int, c_int, c_int, c_vp]),
    "archead_profile": (c_int, [c_int]),
    "archead_test_hooks": (c_int, [ctypes.c_longlong, c_int]),
    "archead_profile_read": (c_int, [ctypes.POINTER(ctypes.c_double), ctypes.POINTER(c_int)]),
}

_lib = None
TESTHOOKS_PATH = os.path.join(HERE, "libarchead_testhooks.so")


def _bind(L: ctypes.CDLL) -> ctypes.CDLL:
    for name, (res, args) in _SIGS.items():
        f = getattr(L, name)
        f.restype = res
        f.argtypes = args
    return L


def testhooks_lib() -> ctypes.CDLL:
    """The failure-detection test build of the library (same entry points, plus working
    archead_test_hooks).  Only tests load it."""
    if not os.path.exists(TESTHOOKS_PATH):
        raise ImportError(f"{TESTHOOKS_PATH} is missing: build it with "
                          "`python -m packed_int4_lm_b200.build`.")
    return _bind(ctypes.CDLL(TESTHOOKS_PATH))


def lib() -> ctypes.CDLL:
    """The loaded library.  Raises if it has not been built: there is no fallback."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(
                f"{LIB_PATH} is missing: build it with `python -m packed_int4_lm_b200.build`. "
                "The packed-head logit path has no CPU or Python fallback.")
        _lib = _bind(ctypes.CDLL(LIB_PATH))
    return _lib


def header_functions(path: str = HEADER):
    """Names of the functions include/archead.h declares."""
    txt = open(path).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(archead_\w+)\s*\(", txt, re.M)))


class ArcheadError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = status
        msg = lib().archead_strerror(status).decode()
        super().__init__(f"{what}: {STATUS.get(status, status)} ({msg})")


def check(status: int, what: str = "") -> None:
    if status != 0:
        raise ArcheadError(status, what)
