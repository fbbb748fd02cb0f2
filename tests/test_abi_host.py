"""The C-ABI library on the host: it loads, exports every function include/archead.h
declares, and rejects bad arguments before touching CUDA (no GPU needed: these calls
return from argument validation and never dereference the fake device pointers)."""
import ctypes
import os

import pytest

from packed_int4_lm_b200 import _lib
from packed_int4_lm_b200._lib import ArcheadHead, STATUS_CODE


@pytest.fixture(scope="module")
def L():
    if not os.path.exists(_lib.LIB_PATH):
        from packed_int4_lm_b200 import build
        build.build()
    return _lib.lib()


def test_exports_every_declared_function(L):
    names = _lib.header_functions()
    assert len(names) >= 10
    for n in names:
        assert hasattr(L, n), n
    assert set(names) >= set(_lib._SIGS)


def test_abi_version_and_strerror(L):
    assert L.archead_abi_version() == 2
    for code in STATUS_CODE.values():
        s = L.archead_strerror(code)
        assert s and s != b"unknown status"
    assert L.archead_strerror(12345) == b"unknown status"


def _fake_head(V=1000, D=512, r_c=4, r_r=4, g=64, base=0x10000):
    h = ArcheadHead()
    h.V, h.D, h.r_c, h.r_r, h.g = V, D, r_c, r_r, g
    for i, k in enumerate(("r_nib", "r_code", "r_super", "Ac", "sAc", "Bc", "sBc", "Aw",
                           "sAw", "Bw", "sBw")):
        setattr(h, k, base + 0x100000 * (i + 1))
    return h


def _logits(L, h, N=4, V=None, D=None, r_c=None, r_r=None, g=None, H=0x9000000, Y=0xA000000):
    return L.archead_logits(H, ctypes.byref(h) if h is not None else None, Y, N,
                            h.V if V is None else V, h.D if D is None else D,
                            h.r_c if r_c is None else r_c, h.r_r if r_r is None else r_r,
                            h.g if g is None else g, None)


E = STATUS_CODE


def test_validation_errors(L):
    h = _fake_head()
    assert L.archead_logits(0x9000000, None, 0xA000000, 4, 1000, 512, 4, 4, 64, None) == E["ARCHEAD_ERR_NULLPTR"]
    assert _logits(L, h, V=999) == E["ARCHEAD_ERR_SHAPE"]          # disagrees with head
    assert _logits(L, h, r_r=5) == E["ARCHEAD_ERR_SHAPE"]
    assert _logits(L, _fake_head(g=48)) == E["ARCHEAD_ERR_SHAPE"]   # unsupported g
    assert _logits(L, _fake_head(D=640, g=256)) == E["ARCHEAD_ERR_SHAPE"]  # D % g
    assert _logits(L, _fake_head(D=200)) == E["ARCHEAD_ERR_SHAPE"]  # D % 128
    assert _logits(L, _fake_head(r_c=129)) == E["ARCHEAD_ERR_SHAPE"]
    assert _logits(L, h, N=-1) == E["ARCHEAD_ERR_SHAPE"]
    assert _logits(L, h, H=0) == E["ARCHEAD_ERR_NULLPTR"]
    assert _logits(L, h, H=0x9000008) == E["ARCHEAD_ERR_ALIGN"]      # H not 16-aligned
    bad = _fake_head()
    bad.r_code = 0x300001
    assert _logits(L, bad) == E["ARCHEAD_ERR_ALIGN"]
    nul = _fake_head()
    nul.Bw = 0
    assert _logits(L, nul) == E["ARCHEAD_ERR_NULLPTR"]
    assert _logits(L, _fake_head(D=(1 << 20) + 128)) == E["ARCHEAD_ERR_SHAPE"]  # D > 2^20
    zero_rank = _fake_head(r_r=0)
    zero_rank.Aw = zero_rank.sAw = zero_rank.Bw = zero_rank.sBw = 0
    assert _logits(L, zero_rank, N=0) == E["ARCHEAD_OK"]            # N = 0: no-op


def test_nll_and_other_entry_validation(L):
    h = _fake_head()
    assert L.archead_nll(0x9000000, ctypes.byref(h), None, 0xA000000, 4, 1000, 512, 4, 4, 64,
                         None) == E["ARCHEAD_ERR_NULLPTR"]
    assert L.archead_nll(0x9000000, ctypes.byref(h), 0xB000000, 0xA000000, 0, 1000, 512, 4, 4,
                         64, None) == E["ARCHEAD_OK"]
    # overlapping repack buffers
    assert L.archead_repack_residual(0x100000, 0x100010, 16, 128, None) == E["ARCHEAD_ERR_SHAPE"]
    assert L.archead_repack_residual(0x100000, 0x900000, 16, 100, None) == E["ARCHEAD_ERR_SHAPE"]
    assert L.archead_repack_residual(None, 0x900000, 16, 128, None) == E["ARCHEAD_ERR_NULLPTR"]
    assert L.archead_dequant(ctypes.byref(h), 990, 20, None, None, None, None, None,
                             None) == E["ARCHEAD_ERR_SHAPE"]
    assert L.archead_logits_host(0x9000000, ctypes.byref(h), 0xA000000, 4, 1000, 512, 4, 4, 16,
                                 None) == E["ARCHEAD_ERR_SHAPE"]


def test_vocab_parallel_entry_validation(L):
    h = _fake_head()  # a 1000-row shard

    def part(v_begin, v_total, N=4, targets=0xB000000, out=0xC000000):
        return L.archead_nll_partials(0x9000000, ctypes.byref(h), targets, v_begin, v_total,
                                      out, N, 1000, 512, 4, 4, 64, None)

    assert part(-1, 5000) == E["ARCHEAD_ERR_SHAPE"]          # v_begin < 0
    assert part(0, 999) == E["ARCHEAD_ERR_SHAPE"]            # shard larger than the head
    assert part(4001, 5000) == E["ARCHEAD_ERR_SHAPE"]        # shard past the end
    assert part(0, 1 << 31) == E["ARCHEAD_ERR_SHAPE"]        # ids beyond int32
    assert part(4000, 5000, N=0) == E["ARCHEAD_OK"]          # N = 0: no-op
    assert part(0, 5000, targets=0) == E["ARCHEAD_ERR_NULLPTR"]
    assert part(0, 5000, out=0xC000002) == E["ARCHEAD_ERR_ALIGN"]
    assert L.archead_nll_merge(0xC000000, 0, 4, 0xD000000, None) == E["ARCHEAD_ERR_SHAPE"]
    assert L.archead_nll_merge(0xC000000, 70000, 4, 0xD000000, None) == E["ARCHEAD_ERR_SHAPE"]
    assert L.archead_nll_merge(0xC000000, 2, -1, 0xD000000, None) == E["ARCHEAD_ERR_SHAPE"]
    assert L.archead_nll_merge(0xC000000, 2, 0, 0xD000000, None) == E["ARCHEAD_OK"]
    assert L.archead_nll_merge(None, 2, 4, 0xD000000, None) == E["ARCHEAD_ERR_NULLPTR"]
    assert L.archead_nll_merge(0xC000001, 2, 4, 0xD000000, None) == E["ARCHEAD_ERR_ALIGN"]


def test_noalloc_rejects_sizes_beyond_its_scratch_before_any_product(L):
    """archead_logits_noalloc checks the request against its fixed 2 MiB array before it
    forms any byte count, so a huge D or N cannot wrap a size and pass the check."""
    def na(h, N):
        return L.archead_logits_noalloc(0x9000000, ctypes.byref(h), 0xA000000, N, h.V, h.D,
                                        h.r_c, h.r_r, h.g, None)
    assert na(_fake_head(D=1 << 62), 4) == E["ARCHEAD_ERR_SHAPE"]
    assert na(_fake_head(D=1 << 20), 4) == E["ARCHEAD_ERR_SHAPE"]     # 8 x 2^20 x 2 B > 2 MiB
    assert na(_fake_head(D=4096), (1 << 31) - 1) == E["ARCHEAD_ERR_SHAPE"]
    assert na(_fake_head(D=4096, r_c=32, r_r=32), 256) == E["ARCHEAD_ERR_SHAPE"]
    assert na(_fake_head(), 0) == E["ARCHEAD_OK"]


def test_product_library_refuses_the_test_hooks(L):
    """archead_test_hooks works only in the failure-detection test build; the product
    library reports ARCHEAD_ERR_UNSUPPORTED and changes nothing (no device is touched)."""
    assert L.archead_test_hooks(1 << 20, 0) == E["ARCHEAD_ERR_UNSUPPORTED"]
    if os.path.exists(_lib.TESTHOOKS_PATH):
        T = _lib.testhooks_lib()
        assert set(_lib.header_functions()) <= {n for n in _lib._SIGS}
        for n in _lib.header_functions():
            assert hasattr(T, n), n
