"""Host-side checks of the C ABI that need no GPU: the library loads, exports every
symbol include/q4.h declares, and rejects bad arguments before touching a device."""
import ctypes
import os
import re

import pytest
import torch

from bit_weight_only_quantize_b200 import _lib, build

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "q4.h")


def declared_functions():
    text = open(HEADER).read()
    return re.findall(r"^Q4_API\s+[\w\s\*]+?\b(q4_\w+)\s*\(", text, flags=re.M)


@pytest.fixture(scope="module")
def lib():
    build.build()
    return _lib.load()


def test_header_declares_expected(lib):
    names = declared_functions()
    assert set(names) == set(_lib.SIGNATURES), names


def test_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
        assert ctypes.cast(getattr(lib, name), ctypes.c_void_p).value


def test_version_and_strings(lib):
    assert lib.q4_abi_version() == 1
    for code in range(8):
        s = lib.q4_status_string(code).decode()
        assert s.startswith(_lib.STATUS_NAMES[code])
    assert lib.q4_status_string(99).decode() == "Q4_ERR_UNKNOWN"


# Fake, never-dereferenced addresses: every call below fails validation first.
A16 = 1 << 20
A8 = A16 + 8


def test_quantize_validation(lib):
    S = None
    assert lib.q4_quantize(A16, 4, 48, A16, A16, None, S) == 2          # K % 32
    assert lib.q4_quantize(A16, 4, 0, A16, A16, None, S) == 2           # K == 0
    assert lib.q4_quantize(A16, -1, 64, A16, A16, None, S) == 2         # N < 0
    assert lib.q4_quantize(None, 4, 64, A16, A16, None, S) == 1         # NULL W
    assert lib.q4_quantize(A16, 4, 64, None, A16, None, S) == 1
    assert lib.q4_quantize(A8, 4, 64, A16, A16, None, S) == 3           # misaligned W
    assert lib.q4_quantize(A16, 4, 64, A8, A16, None, S) == 3
    assert lib.q4_quantize(A16, 4, 64, A16, A16 + 1, None, S) == 3
    assert lib.q4_quantize(A16, 4, 64, A16, A16, A16 + 2, S) == 3
    assert lib.q4_quantize(None, 0, 64, None, None, None, S) == 0       # empty: no-op


def test_gemv_validation(lib):
    S = None
    assert lib.q4_gemv(A16, 7, 1, 64, A16, A16, 8, A16, None, 0, S) == 4        # dtype
    assert lib.q4_gemv(A16, 1, 17, 64, A16, A16, 8, A16, None, 0, S) == 2       # M > 16
    assert lib.q4_gemv(A16, 1, -1, 64, A16, A16, 8, A16, None, 0, S) == 2
    assert lib.q4_gemv(A16, 1, 1, 40, A16, A16, 8, A16, None, 0, S) == 2        # K % 32
    assert lib.q4_gemv(None, 1, 1, 64, A16, A16, 8, A16, None, 0, S) == 1
    assert lib.q4_gemv(A16, 1, 1, 64, A16, A16, 8, None, None, 0, S) == 1
    assert lib.q4_gemv(A8, 1, 1, 64, A16, A16, 8, A16, None, 0, S) == 3        # x alignment
    assert lib.q4_gemv(A16, 1, 1, 64, A8, A16, 8, A16, None, 0, S) == 3        # packed alignment
    assert lib.q4_gemv(A16, 1, 1, 64, A16, A16 + 1, 8, A16 + 2, None, 0, S) == 3
    assert lib.q4_gemv(A16, 1, 1, 64, A16, A16, 8, A16, A8, 64, S) == 3       # workspace alignment
    assert lib.q4_gemv(None, 1, 0, 64, None, None, 8, None, None, 0, S) == 0   # M == 0: no-op
    assert lib.q4_gemv(None, 1, 3, 64, None, None, 0, None, None, 0, S) == 0   # N == 0: no-op


def test_gemm_validation(lib):
    S = None
    assert lib.q4_gemm(A16, 4, 48, A16, A16, 8, A16, S) == 2           # K % 32
    assert lib.q4_gemm(A16, -1, 64, A16, A16, 8, A16, S) == 2          # M < 0
    assert lib.q4_gemm(None, 4, 64, A16, A16, 8, A16, S) == 1
    assert lib.q4_gemm(A16, 4, 64, A16, A16, 8, None, S) == 1
    assert lib.q4_gemm(A8, 4, 64, A16, A16, 8, A16, S) == 3            # x alignment
    assert lib.q4_gemm(A16, 4, 64, A8, A16, 8, A16, S) == 3            # packed alignment
    assert lib.q4_gemm(A16, 4, 64, A16, A16 + 1, 8, A16, S) == 3
    assert lib.q4_gemm(A16, 4, 64, A16, A16, 8, A16 + 1, S) == 3
    assert lib.q4_gemm(None, 0, 64, None, None, 8, None, S) == 0       # M == 0: no-op
    assert lib.q4_gemm(None, 4, 64, None, None, 0, None, S) == 0       # N == 0: no-op


def test_gemv_multi_validation(lib):
    W = _lib.Weight
    good = (W * 2)(W(A16, A16, 8, A16), W(A16, A16, 16, A16))
    vp = ctypes.cast(good, ctypes.c_void_p)
    assert lib.q4_gemv_multi(A16, 1, 1, 64, None, 1, 0, None, 0, None) == 1          # no matrices
    assert lib.q4_gemv_multi(A16, 1, 1, 64, vp, 0, 0, None, 0, None) == 1            # count 0
    assert lib.q4_gemv_multi(A16, 1, 1, 64, vp, 5, 0, None, 0, None) == 1            # count > max
    assert lib.q4_gemv_multi(A16, 1, 1, 64, vp, 2, 4, None, 0, None) == 1            # unknown flag
    assert lib.q4_gemv_multi(A16, 1, 1, 48, vp, 2, 0, None, 0, None) == 2            # K % 32
    bad = (W * 2)(W(A16, A16, 8, A16), W(A8, A16, 16, A16))
    assert lib.q4_gemv_multi(A16, 1, 1, 64, ctypes.cast(bad, ctypes.c_void_p), 2, 0, None, 0, None) == 3
    nul = (W * 2)(W(A16, A16, 8, A16), W(None, A16, 16, A16))
    assert lib.q4_gemv_multi(A16, 1, 1, 64, ctypes.cast(nul, ctypes.c_void_p), 2, 0, None, 0, None) == 1
    empty = (W * 2)(W(None, None, 0, None), W(None, None, 0, None))
    assert lib.q4_gemv_multi(A16, 1, 1, 64, ctypes.cast(empty, ctypes.c_void_p), 2, 0, None, 0, None) == 0


def test_device_error_rejects_null(lib):
    assert lib.q4_device_error(None, 0) == 1


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device path")
def test_no_device_reports_cuda_error(lib):
    assert lib.q4_quantize(A16, 4, 64, A16, A16, None, None) == 6
    assert lib.q4_gemv(A16, 1, 1, 64, A16, A16, 8, A16, None, 0, None) == 6
    assert lib.q4_gemv_workspace_size(1, 8, 64) == 0


def test_binding_raises_without_gpu_tensors():
    import bit_weight_only_quantize_b200 as q4
    with pytest.raises(ValueError):
        q4.quantize(torch.zeros(4, 64))


def test_gate_up_validation(lib):
    S = None
    f = lib.q4_gemv_gate_up
    assert f(A16, 7, 1, 256, A16, A16, A16, A16, 8, A16, 0, S) == 4            # dtype
    assert f(A16, 1, 17, 256, A16, A16, A16, A16, 8, A16, 0, S) == 2           # M > 16
    assert f(A16, 1, 1, 40, A16, A16, A16, A16, 8, A16, 0, S) == 2             # K % 32
    assert f(A16, 1, 1, 256, A16, A16, A16, A16, 8, A16, 4, S) == 1            # unknown flag
    assert f(A16, 1, 1, 256, None, A16, A16, A16, 8, A16, 0, S) == 1
    assert f(A16, 1, 1, 256, A16, A16, A16, A16, 8, None, 0, S) == 1
    assert f(A16, 1, 1, 256, A16, A16, A8, A16, 8, A16, 0, S) == 3             # up packed alignment
    assert f(A16, 1, 1, 256, A16, A8, A16, A16, 8, A16, 0, S) == 3             # gate scales: 16 bytes
    assert f(A16, 1, 1, 96, A16, A16, A16, A16, 8, A16, 0, S) == 2             # K % 256
    assert f(A16, 0, 2, 256, A16, A16, A16, A16, 8, A16, 0, S) == 2            # f32 x with M > 1
    assert f(None, 1, 0, 256, None, None, None, None, 8, None, 0, S) == 0      # M == 0: no-op
    assert f(None, 1, 3, 256, None, None, None, None, 0, None, 0, S) == 0      # N == 0: no-op


def test_argmax_validation(lib):
    S = None
    f = lib.q4_gemv_argmax
    assert lib.q4_gemv_argmax_workspace_size() >= 16 * 8 + 4
    W = 256
    assert f(A16, 7, 1, 256, A16, A16, 8, None, A16, None, 0, A16, W, S) == 4      # dtype
    assert f(A16, 1, 17, 256, A16, A16, 8, None, A16, None, 0, A16, W, S) == 2     # M > 16
    assert f(A16, 1, 1, 256, A16, A16, 8, None, None, None, 0, A16, W, S) == 1     # index required
    assert f(A16, 1, 1, 256, A16, A16, 8, None, A16, None, 0, None, 0, S) == 5     # workspace required
    assert f(A16, 1, 1, 256, A16, A16, 8, None, A16, None, 0, A16, 64, S) == 5     # workspace too small
    assert f(A16, 1, 1, 256, A16, A16, 8, None, A16 + 4, None, 0, A16, W, S) == 3  # index alignment
    assert f(A16, 1, 1, 256, A16, A8, 8, None, A16, None, 0, A16, W, S) == 3       # scales: 16 bytes
    assert f(A16, 1, 1, 96, A16, A16, 8, None, A16, None, 0, A16, W, S) == 2       # K % 256
    assert f(None, 1, 0, 256, None, None, 8, None, None, None, 0, None, 0, S) == 0  # M == 0: no-op


def test_topk_validation(lib):
    S = None
    f = lib.q4_gemv_topk
    W = 1 << 20
    ok = dict(x=A16, t=1, M=1, K=256, p=A16, s=A16, N=8, k=20, rb=0, y=None, i=A16, v=None, fl=0, ws=A16, wb=W)

    def call(**kw):
        a = {**ok, **kw}
        return f(a["x"], a["t"], a["M"], a["K"], a["p"], a["s"], a["N"], a["k"], a["rb"], a["y"], a["i"], a["v"],
                 a["fl"], a["ws"], a["wb"], S)
    assert call(t=7) == 4                                   # dtype
    assert call(M=17) == 2                                  # M > 16
    assert call(k=0) == 2 and call(k=33) == 2               # k in 1..32
    assert call(rb=-1) == 2                                 # row_base >= 0
    assert call(rb=(1 << 31) - 8) == 2                      # row_base + N past 2^31 - 1
    assert call(fl=2) == 1                                  # unknown flag
    assert call(i=None) == 1                                # index required
    assert call(ws=None, wb=0) == 5                         # workspace required
    assert call(i=A16 + 4) == 3                             # index alignment
    assert call(s=A8) == 3                                  # scales: 16 bytes
    assert call(v=A16 + 2) == 3                             # value alignment
    assert call(K=96) == 2                                  # K % 256
    assert call(t=0, M=2) == 2                              # f32 x only with M == 1
    assert call(x=None, M=0, p=None, s=None, i=None, ws=None, wb=0) == 0   # M == 0: no-op
    assert call(x=None, N=0, p=None, s=None, i=None, ws=None, wb=0) == 0   # N == 0: no-op
    assert lib.q4_gemv_topk_workspace_size(1, 8, 96, 20, 1) == 0          # K % 256: not served
    assert lib.q4_gemv_topk_workspace_size(1, 8, 256, 33, 1) == 0         # k > 32


def test_topk_merge_validation(lib):
    f = lib.q4_topk_merge
    assert f(A16, A16, 0, 1, 20, A16, None, None) == 2              # S >= 1
    assert f(A16, A16, 1 << 21, 1, 20, A16, None, None) == 2        # S <= 2^20
    assert f(A16, A16, 2, 1, 0, A16, None, None) == 2               # k >= 1
    assert f(A16, A16, 2, 1, 33, A16, None, None) == 2              # k <= 32
    assert f(A16, A16, 2, -1, 20, A16, None, None) == 2             # M >= 0
    assert f(None, A16, 2, 1, 20, A16, None, None) == 1             # values required
    assert f(A16, A16, 2, 1, 20, None, None, None) == 1             # index required
    assert f(A16 + 2, A16, 2, 1, 20, A16, None, None) == 3          # values alignment
    assert f(A16, A16 + 4, 2, 1, 20, A16, None, None) == 3          # indices alignment
    assert f(A16, A16, 2, 1, 20, A16, A16 + 2, None) == 3           # value alignment
    assert f(None, None, 2, 0, 20, None, None, None) == 0           # M == 0: no-op


def test_int8_validation(lib):
    S = None
    q = lib.q4_int8_quantize
    assert q(A16, 4, 96 + 8, A16, A16, None, S) == 2           # K % 32
    assert q(A16, -1, 64, A16, A16, None, S) == 2               # N >= 0
    assert q(None, 4, 64, A16, A16, None, S) == 1
    assert q(A16 + 4, 4, 64, A16, A16, None, S) == 3            # W: 16 bytes
    assert q(A16, 4, 64, A16 + 8, A16, None, S) == 3            # codes: 16 bytes
    assert q(A16, 4, 64, A16, A16 + 1, None, S) == 3            # scales: 2 bytes
    assert q(None, 0, 64, None, None, None, S) == 0             # N == 0: no-op
    g = lib.q4_int8_gemv
    assert g(A16, 7, 1, 64, A16, A16, 8, A16, S) == 4           # dtype
    assert g(A16, 1, 17, 64, A16, A16, 8, A16, S) == 2          # M > 16
    assert g(A16, 1, 1, 48, A16, A16, 8, A16, S) == 2           # K % 32
    assert g(A16, 1, 1, 64, None, A16, 8, A16, S) == 1
    assert g(A16 + 2, 1, 1, 64, A16, A16, 8, A16, S) == 3       # x: 16 bytes
    assert g(A16 + 4, 1, 1, 64, A16, A16, 8, A16, S) == 3
    assert g(A16, 1, 1, 64, A8, A16, 8, A16, S) == 3            # codes: 16 bytes
    assert g(A16, 1, 1, 64, A16, A16, 8, A16 + 2, S) == 3       # y: 4 bytes
    assert g(None, 1, 0, 64, None, None, 8, None, S) == 0       # M == 0: no-op


def test_f16_gemv_validation(lib):
    S = None
    f = lib.q4_f16_gemv
    assert f(A16, 7, 1, 64, A16, 8, A16, 0, S) == 4                 # dtype
    assert f(A16, 0, 2, 64, A16, 8, A16, 0, S) == 2                 # f32 x with M > 1
    assert f(A16, 1, 17, 64, A16, 8, A16, 0, S) == 2                # M > 16
    assert f(A16, 1, 1, 12, A16, 8, A16, 0, S) == 2                 # K % 8
    assert f(A16, 1, 1, 64, A16, 8, A16, 2, S) == 1                 # unknown flag
    assert f(A16, 1, 1, 64, None, 8, A16, 0, S) == 1
    assert f(A16, 1, 1, 64, A8, 8, A16, 0, S) == 3                  # w alignment
    assert f(A16, 1, 1, 64, A16, 8, A16 + 2, 0, S) == 3             # y alignment
    assert f(None, 1, 0, 64, None, 8, None, 0, S) == 0              # M == 0: no-op


def test_consumer_wait_limit_round_trips(lib):
    """The failure-path hook keeps the value it is given and defaults to 1 s."""
    prev = lib.q4_set_consumer_wait_limit(12345)
    assert prev == 10 ** 9
    assert lib.q4_set_consumer_wait_limit(prev) == 12345
    assert lib.q4_set_consumer_wait_limit(prev) == prev


def test_mixed_validation(lib):
    """q4_gemv_mixed checks its matrix list before touching a device."""
    S = None
    W = _lib.MixedWeight

    def call(mats, M=1, K=64, x=A16, dtype=1, flags=0):
        arr = (W * len(mats))(*mats)
        return lib.q4_gemv_mixed(x, dtype, M, K, ctypes.cast(arr, ctypes.c_void_p), len(mats), flags, None, 0, S)
    ok = W(A16, A16, 8, A16, 8, 0)
    assert call([ok], dtype=7) == 4                                  # dtype
    assert call([ok], M=17) == 2                                     # M > 16
    assert call([ok], K=48) == 2                                     # K % 32
    assert call([ok], flags=2) == 1                                  # unknown flag
    assert call([W(A16, A16, 8, A16, 5, 0)]) == 1                    # bits must be 4 or 8
    assert call([W(A16, A16, 8, A16, 8, 1)]) == 1                    # reserved must be 0
    assert call([W(None, A16, 8, A16, 8, 0)]) == 1                   # null codes
    assert call([W(A8, A16, 8, A16, 4, 0)]) == 3                     # codes 16-byte aligned
    assert call([ok], x=A16 + 8) == 3                                # x 16-byte aligned
    assert call([W(None, None, 0, None, 8, 0)]) == 0                 # N == 0: nothing to do
    assert call([ok], M=0) == 0                                      # M == 0: no-op
