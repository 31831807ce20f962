"""The C-ABI library loads, exports every symbol include/omnimoe.h declares and
rejects bad arguments on the host (no CUDA call is reached on these paths)."""
import ctypes as C
import os
import re

import pytest

from atomic_expert_routing_b200 import _lib
from atomic_expert_routing_b200 import build as libbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "omnimoe.h")


def _declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(omni_[a-z_]+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    libbuild.build()
    return _lib.load()


def test_every_declared_symbol_is_exported(lib):
    names = _declared()
    assert "omni_moe_forward" in names and "omni_schedule" in names
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(_lib.SIGNATURES), "binding prototypes out of sync with the header"
    assert lib.omni_abi_version() == 1


def _dims(**kw):
    base = dict(L=128, d=64, Nr=64, Nc=64, k=8, K=8, B=32, dtype=_lib.OMNI_F32, flags=0)
    base.update(kw)
    return _lib.Dims(**base)


def _wsz(lib, D, which):
    n = C.c_size_t(0)
    rc = lib.omni_workspace_size(C.byref(D), which, C.byref(n))
    return rc, n.value


@pytest.mark.parametrize("bad,code", [
    (dict(k=0), _lib.OMNI_ERR_INVALID_ARG),
    (dict(k=65), _lib.OMNI_ERR_INVALID_ARG),          # k > Nr
    (dict(K=65), _lib.OMNI_ERR_INVALID_ARG),          # K > k*k
    (dict(B=0), _lib.OMNI_ERR_INVALID_ARG),
    (dict(L=-1), _lib.OMNI_ERR_INVALID_ARG),
    (dict(dtype=7), _lib.OMNI_ERR_INVALID_ARG),
    (dict(flags=8), _lib.OMNI_ERR_INVALID_ARG),
    (dict(d=60), _lib.OMNI_ERR_UNSUPPORTED),          # not a multiple of 8
    (dict(Nr=5000, Nc=8), _lib.OMNI_ERR_UNSUPPORTED),
    (dict(Nr=512, Nc=512, k=300, K=8), _lib.OMNI_ERR_UNSUPPORTED),
])
def test_dims_validation(lib, bad, code):
    rc, _ = _wsz(lib, _dims(**bad), _lib.OMNI_WS_FUSED)
    assert rc == code
    assert lib.omni_status_string(rc)


def test_workspace_sizes(lib):
    D = _dims(dtype=_lib.OMNI_BF16)
    sizes = {w: _wsz(lib, D, w) for w in range(6)}
    assert all(rc == 0 for rc, _ in sizes.values())
    route = sizes[_lib.OMNI_WS_ROUTE][1]
    assert route >= 128 * (64 + 64) * 4            # the fp32 logits
    assert sizes[_lib.OMNI_WS_EXPERT][1] >= 128 * 64 * 4  # fp32 accumulator for bf16 output
    fused = sizes[_lib.OMNI_WS_FUSED][1]
    assert fused >= route + sizes[_lib.OMNI_WS_SCHEDULE][1] + sizes[_lib.OMNI_WS_EXPERT][1]
    assert sizes[_lib.OMNI_WS_TOKEN][1] == 0
    # fp32 storage accumulates into y directly
    assert _wsz(lib, _dims(), _lib.OMNI_WS_EXPERT)[1] == 0
    rc, _ = _wsz(lib, D, 99)
    assert rc == _lib.OMNI_ERR_INVALID_ARG


def test_host_checks_reject_before_any_launch(lib):
    D = _dims()
    fake = C.c_void_p(4096)       # aligned, never dereferenced on these paths
    odd = C.c_void_p(4096 + 4)    # misaligned for a 16-byte tensor
    # null dims
    assert lib.omni_moe_forward(None, *([fake] * 11), None, 0, None) == _lib.OMNI_ERR_INVALID_ARG
    # misaligned x
    assert lib.omni_route(C.byref(D), odd, fake, fake, None, None, fake, fake, None, None,
                          fake, 1 << 30, None) == _lib.OMNI_ERR_INVALID_ARG
    # workspace too small / misaligned
    assert lib.omni_route(C.byref(D), fake, fake, fake, None, None, fake, fake, None, None,
                          fake, 16, None) == _lib.OMNI_ERR_WORKSPACE
    assert lib.omni_route(C.byref(D), fake, fake, fake, None, None, fake, fake, None, None,
                          C.c_void_p(4096 + 16), 1 << 30, None) == _lib.OMNI_ERR_WORKSPACE
    # schedule needs counts
    assert lib.omni_schedule(C.byref(D), fake, fake, fake, fake, fake, fake, fake, None, fake,
                             1 << 30, None) == _lib.OMNI_ERR_INVALID_ARG
    # the fused call needs counts
    assert lib.omni_moe_forward(C.byref(D), *([fake] * 10), None, fake, 1 << 30,
                                None) == _lib.OMNI_ERR_INVALID_ARG
    # the wait diagnostic needs an aligned counts
    assert lib.omni_wait_selftest(None, None) == _lib.OMNI_ERR_INVALID_ARG
    assert lib.omni_wait_selftest(C.c_void_p(4096 + 2), None) == _lib.OMNI_ERR_INVALID_ARG


def test_empty_batch_is_a_no_op(lib):
    D = _dims(L=0)
    fake = C.c_void_p(4096)
    assert lib.omni_route(C.byref(D), fake, fake, fake, None, None, fake, fake, None, None, None,
                          0, None) == _lib.OMNI_OK
    assert lib.omni_expert_forward(C.byref(D), *([fake] * 10), None, 0, None) == _lib.OMNI_OK
    assert lib.omni_token_centric_forward(C.byref(D), *([fake] * 7), None, 0,
                                          None) == _lib.OMNI_OK
