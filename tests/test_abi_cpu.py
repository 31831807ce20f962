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


def _documented_code(L, d, Nr, Nc, k, K, B, dtype, flags):
    """The host checks as the header states them (invalid before unsupported)."""
    if (L < 0 or min(d, Nr, Nc, k, K, B) < 1 or dtype not in (_lib.OMNI_F32, _lib.OMNI_BF16)
            or flags & ~(_lib.OMNI_FLAG_ROUTER_SIMT | _lib.OMNI_FLAG_STAGED_SMALL
                         | _lib.OMNI_FLAG_DENSE_TENSOR_CORES)
            or k > min(Nr, Nc) or K > k * k):
        return _lib.OMNI_ERR_INVALID_ARG
    if (max(Nr, Nc) > 4096 or max(k, K) > 256 or Nr * Nc >= 2 ** 31 or L * K >= 2 ** 30
            or d % 8 or d > 65536):
        return _lib.OMNI_ERR_UNSUPPORTED
    return _lib.OMNI_OK


_I64 = 2 ** 63 - 1


def test_dims_checks_follow_the_header(lib):
    """Randomised dims, from ordinary to absurd (up to the int64 range): the
    library returns the code the header documents, and a positive workspace
    size of every kind for every accepted dims."""
    from hypothesis import HealthCheck, example, given, settings, strategies as st

    small = st.integers(-2, 5000)
    anyint = st.one_of(small, st.integers(-_I64 - 1, _I64), st.sampled_from(
        [2 ** 30, 2 ** 31, 2 ** 32 + 1, 2 ** 62, _I64]))
    field = st.one_of(small, small, anyint)

    @settings(max_examples=3000, deadline=None, database=None,
              suppress_health_check=list(HealthCheck))
    @given(L=field, d=st.one_of(st.sampled_from([8, 16, 40, 64, 2048, 65536, 65544]), field),
           Nr=field, Nc=field, k=st.one_of(st.integers(1, 300), field),
           K=st.one_of(st.integers(1, 300), field), B=field,
           dtype=st.sampled_from([0, 1, 2, -1]), flags=st.sampled_from([0, 1, 2, 3, 4, 7, 8, 15]))
    # L*K that wraps around int64; k*k that does
    @example(L=2 ** 62, d=64, Nr=64, Nc=64, k=2, K=4, B=1, dtype=1, flags=0)
    @example(L=16, d=64, Nr=2 ** 33, Nc=2 ** 33, k=2 ** 32, K=1, B=1, dtype=1, flags=0)
    def check(L, d, Nr, Nc, k, K, B, dtype, flags):
        D = _lib.Dims(L=L, d=d, Nr=Nr, Nc=Nc, k=k, K=K, B=B, dtype=dtype, flags=flags)
        want = _documented_code(L, d, Nr, Nc, k, K, B, dtype, flags)
        for which in range(6):
            rc, n = _wsz(lib, D, which)
            assert rc == want, (L, d, Nr, Nc, k, K, B, dtype, flags, which)
            if rc == _lib.OMNI_OK and which in (_lib.OMNI_WS_ROUTE, _lib.OMNI_WS_FUSED) and L > 0:
                assert n > 0

    check()


def test_selecting_calls_refuse_K_above_k(lib):
    """The top-K of the k x k candidate pairs is the top-K of all N joint
    scores only when k >= K.  The calls that select experts refuse K > k
    before any other check; scheduling and execution do not use k and pass
    the dims check (they then stop at a null pointer, not at the dims)."""
    D = _dims(k=4, K=6)
    fake = C.c_void_p(4096)
    U = _lib.OMNI_ERR_UNSUPPORTED
    assert lib.omni_route(C.byref(D), fake, fake, fake, None, None, fake, fake, None, fake,
                          fake, 1 << 30, None) == U
    assert lib.omni_route_select(C.byref(D), fake, None, None, fake, fake, None, fake, None, 0,
                                 None) == U
    assert lib.omni_moe_forward(C.byref(D), *([fake] * 11), fake, 1 << 30, None) == U
    assert lib.omni_schedule(C.byref(D), fake, fake, fake, fake, fake, fake, fake, None, fake,
                             1 << 30, None) == _lib.OMNI_ERR_INVALID_ARG
    assert lib.omni_expert_forward(C.byref(D), *([fake] * 8), None, fake, fake, 1 << 30,
                                   None) == _lib.OMNI_ERR_INVALID_ARG
    for which in range(6):
        assert _wsz(lib, D, which)[0] == _lib.OMNI_OK
    # K == k is accepted (the same null-pointer stop as above)
    D = _dims(k=6, K=6)
    assert lib.omni_moe_forward(C.byref(D), *([fake] * 10), None, fake, 1 << 30,
                                None) == _lib.OMNI_ERR_INVALID_ARG


NOALLOC_MAX = 1 << 22  # floats in the library's fixed accumulator


@pytest.mark.parametrize("L,d,code", [
    # exactly at the limit: past the size check, stopped by the null y
    (NOALLOC_MAX // 2048, 2048, _lib.OMNI_ERR_INVALID_ARG),
    (NOALLOC_MAX // 8, 8, _lib.OMNI_ERR_INVALID_ARG),
    # one row past it, and far past it
    (NOALLOC_MAX // 8 + 1, 8, _lib.OMNI_ERR_UNSUPPORTED),
    (NOALLOC_MAX // 2048 + 1, 2048, _lib.OMNI_ERR_UNSUPPORTED),
    (4096, 2048, _lib.OMNI_ERR_UNSUPPORTED),
])
def test_noalloc_size_limit(lib, L, d, code):
    """omni_expert_forward_noalloc takes batches up to L*d = 4194304 (its
    fixed accumulator) and refuses larger ones before touching the GPU."""
    D = _dims(L=L, d=d, Nr=32, Nc=32, k=4, K=4, B=16, dtype=_lib.OMNI_BF16)
    fake = C.c_void_p(4096)
    args = [fake] * 10
    args[9] = None  # y
    assert lib.omni_expert_forward_noalloc(C.byref(D), *args, None) == code


@pytest.mark.parametrize("F,dtype,code", [
    (0, _lib.OMNI_BF16, _lib.OMNI_ERR_INVALID_ARG),
    (-8, _lib.OMNI_BF16, _lib.OMNI_ERR_INVALID_ARG),
    (12, _lib.OMNI_BF16, _lib.OMNI_ERR_UNSUPPORTED),      # not a multiple of 8
    (65544, _lib.OMNI_BF16, _lib.OMNI_ERR_UNSUPPORTED),
    (64, _lib.OMNI_F32, _lib.OMNI_ERR_UNSUPPORTED),       # tensor cores: bf16 only
    (64, _lib.OMNI_BF16, _lib.OMNI_OK),
])
def test_shared_mlp_host_checks(lib, F, dtype, code):
    """The MLP width and storage checks, before any launch (null tensors
    stop the accepted case)."""
    D = _dims(dtype=dtype)
    n = C.c_size_t(0)
    assert lib.omni_mlp_workspace_size(C.byref(D), F, 0, C.byref(n)) == code
    if code == _lib.OMNI_OK:
        assert n.value == 128 * 64 * 2  # the bf16 hidden activations
        assert lib.omni_mlp_workspace_size(C.byref(D), F, 1, C.byref(n)) == _lib.OMNI_OK
        assert n.value >= 128 * 64 * 2 + _wsz(lib, D, _lib.OMNI_WS_FUSED)[1]
    fake = C.c_void_p(4096)
    rc = lib.omni_shared_mlp(C.byref(D), F, None, fake, fake, fake, 0, None, fake, 1 << 30, None)
    assert rc == (code if code != _lib.OMNI_OK else _lib.OMNI_ERR_INVALID_ARG)
    rc = lib.omni_moe_mlp_forward(C.byref(D), F, *([fake] * 12), None, fake, 1 << 30, None)
    assert rc == (code if code != _lib.OMNI_OK else _lib.OMNI_ERR_INVALID_ARG)


def test_gated_entries_check_U_like_the_other_tensors(lib):
    """The gated (SwiGLU) calls take the plain calls' checks plus U: a null or
    misaligned U is an invalid argument in a non-empty batch, an empty batch
    is a no-op, and the selecting call refuses K > k first."""
    D = _dims()
    fake = C.c_void_p(4096)
    odd = C.c_void_p(4096 + 4)
    bad = _lib.OMNI_ERR_INVALID_ARG
    for U in (None, odd):
        # x, Wr, Wc, bias_r, bias_c, W, U, V, y, idx, gate, counts
        args = [fake, fake, fake, None, None, fake, U, fake, fake, None, None, fake]
        assert lib.omni_moe_forward_glu(C.byref(D), *args, fake, 1 << 30, None) == bad
        # x, W, U, V, task_token, task_expert, task_gate, uniq, group_off, counts, y
        args = [fake, fake, U] + [fake] * 8
        assert lib.omni_expert_forward_glu(C.byref(D), *args, fake, 1 << 30, None) == bad
        # x, W, U, V, idx, gate, y, counts
        args = [fake, fake, U] + [fake] * 5
        assert lib.omni_token_centric_forward_glu(C.byref(D), *args, None, 0, None) == bad
    # a good U: the same stop as the plain calls (a null counts / task array)
    assert lib.omni_moe_forward_glu(C.byref(D), *([fake] * 11), None, fake, 1 << 30,
                                    None) == bad
    assert lib.omni_expert_forward_glu(C.byref(D), *([fake] * 9), None, fake, fake, 1 << 30,
                                       None) == bad
    E = _dims(L=0)
    assert lib.omni_expert_forward_glu(C.byref(E), *([None] * 11), None, 0, None) == _lib.OMNI_OK
    assert lib.omni_token_centric_forward_glu(C.byref(E), *([None] * 8), None, 0,
                                              None) == _lib.OMNI_OK
    assert lib.omni_moe_forward_glu(C.byref(E), *([None] * 11), fake, None, 0,
                                    None) == _lib.OMNI_OK
    K6 = _dims(k=4, K=6)
    assert lib.omni_moe_forward_glu(C.byref(K6), *([fake] * 12), fake, 1 << 30,
                                    None) == _lib.OMNI_ERR_UNSUPPORTED


def test_shard_entry_host_checks(lib):
    """omni_moe_forward_shard: the shard's id range must be a non-empty part
    of [0, N), y_part and the (optional) U 16-byte aligned; an empty batch
    is a no-op; K > k is refused as in the unsharded call."""
    D = _dims(Nr=8, Nc=8)  # N = 64
    fake = C.c_void_p(4096)
    odd = C.c_void_p(4096 + 4)
    bad = _lib.OMNI_ERR_INVALID_ARG

    def call(dims, lo, hi, U=None, y_part=fake, counts=fake):
        # x, Wr, Wc, bias_r, bias_c, W, U, V, y_part, idx, gate, counts
        args = [fake, fake, fake, None, None, fake, U, fake, y_part, None, None, counts]
        return lib.omni_moe_forward_shard(C.byref(dims), lo, hi, *args, None, 0, None)

    for lo, hi in ((-1, 4), (4, 4), (5, 4), (0, 65), (64, 65)):
        assert call(D, lo, hi) == bad, (lo, hi)
    assert call(D, 0, 64, counts=None) == bad
    assert call(D, 0, 64, y_part=odd) == bad
    assert call(D, 0, 64, U=odd) == bad
    # a valid call stops at the workspace (none given)
    assert call(D, 0, 64) == _lib.OMNI_ERR_WORKSPACE
    assert call(D, 63, 64, U=fake) == _lib.OMNI_ERR_WORKSPACE
    assert call(_dims(L=0, Nr=8, Nc=8), 3, 9) == _lib.OMNI_OK
    assert call(_dims(Nr=8, Nc=8, k=2, K=3), 0, 64) == _lib.OMNI_ERR_UNSUPPORTED


def test_cast_output_host_checks(lib):
    fake, other = C.c_void_p(4096), C.c_void_p(8192)
    D = _dims(dtype=_lib.OMNI_BF16)
    assert lib.omni_cast_output(C.byref(D), None, fake, None) == _lib.OMNI_ERR_INVALID_ARG
    assert lib.omni_cast_output(C.byref(D), fake, C.c_void_p(4100), None) == \
        _lib.OMNI_ERR_INVALID_ARG
    # in place is a bf16 error (the fp32 sum would be overwritten as it is read)
    assert lib.omni_cast_output(C.byref(D), fake, fake, None) == _lib.OMNI_ERR_INVALID_ARG
    assert lib.omni_cast_output(C.byref(_dims(L=0)), fake, other, None) == _lib.OMNI_OK
    # fp32 in place: nothing to do, no launch
    F = _dims(dtype=_lib.OMNI_F32)
    assert lib.omni_cast_output(C.byref(F), fake, fake, None) == _lib.OMNI_OK


def test_backward_host_checks(lib):
    """omni_moe_backward: bf16 storage only; null or misaligned arrays are
    invalid; the workspace is checked; an empty batch is a no-op."""
    fake = C.c_void_p(4096)
    odd = C.c_void_p(4096 + 4)
    B16 = _dims(dtype=_lib.OMNI_BF16)

    def call(dims, **over):
        names = ["x", "Wr", "Wc", "W", "V", "idx", "gate", "dy", "dx", "dW", "dV", "dWr", "dWc",
                 "dbias_r", "dbias_c", "counts"]
        args = {n: fake for n in names}
        args["dbias_r"] = args["dbias_c"] = None
        args.update(over)
        ws = over.pop("ws", None)
        return lib.omni_moe_backward(C.byref(dims), *[args[n] for n in names[:-1]], 1,
                                     args["counts"], ws, 1 << 30 if ws is not None else 0, None)

    assert call(_dims(dtype=_lib.OMNI_F32)) == _lib.OMNI_ERR_UNSUPPORTED
    assert call(B16, dy=None) == _lib.OMNI_ERR_INVALID_ARG
    assert call(B16, dW=odd) == _lib.OMNI_ERR_INVALID_ARG
    assert call(B16, counts=None) == _lib.OMNI_ERR_INVALID_ARG
    assert call(B16, dbias_r=C.c_void_p(4096 + 2)) == _lib.OMNI_ERR_INVALID_ARG
    assert call(B16) == _lib.OMNI_ERR_WORKSPACE
    assert call(_dims(L=0, dtype=_lib.OMNI_BF16), x=None) == _lib.OMNI_OK
    n = C.c_size_t(0)
    assert lib.omni_workspace_size(C.byref(B16), _lib.OMNI_WS_BACKWARD, C.byref(n)) == 0
    assert n.value > 0
