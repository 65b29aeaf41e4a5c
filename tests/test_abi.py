"""C-ABI checks that need no GPU: the library loads, exports every entry point the public
header declares, and rejects bad arguments before making any CUDA call."""

import ctypes
import os
import re

import pytest

import exact_attention_100_b200 as ea
from exact_attention_100_b200 import build as ea_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    ea_build.build()
    return ea.lib()


def _declared_functions():
    with open(os.path.join(ROOT, "include", "attn.h")) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:int|void|const char\*|unsigned long long)\s+(attn_\w+)\s*\(", text, re.M)))


def test_header_declares_the_boundary():
    names = _declared_functions()
    assert names == sorted(["attn_fwd", "attn_hadamard_quant", "attn_fwd_fp8", "attn_device_status",
                            "attn_status_string", "attn_num_kernel_launches", "attn_shutdown",
                            "attn_fwd_noalloc", "attn_hadamard_quant_qkv", "attn_bwd",
                            "attn_bwd_workspace_bytes", "attn_fwd_qk", "attn_bwd_qk", "attn_fwd_strided",
                            "attn_fwd_varlen", "attn_rope_hadamard_quant_qkv", "attn_bwd_strided",
                            "attn_bwd_varlen", "attn_fwd_fp8_qk", "attn_merge_partials",
                            "attn_selftest_wait_timeout", "attn_noalloc_status",
                            "attn_noalloc_selftest_wait_timeout", "attn_hadamard_quant_qkv_strided",
                            "attn_fwd_fp8_strided", "attn_fwd_schedule", "attn_hadamard_quant_qkv_varlen",
                            "attn_fwd_fp8_varlen", "attn_bwd_ds_workspace_bytes", "attn_bwd_ds",
                            "attn_bwd_varlen_ds_workspace_bytes", "attn_bwd_varlen_ds"])


def test_library_exports_every_declared_symbol(L):
    for name in _declared_functions():
        assert hasattr(L, name), name


def test_status_strings(L):
    assert ea.attn_status_string(0) == "ATTN_OK"
    assert ea.attn_status_string(1) == "ATTN_ERR_INVALID_ARG"
    assert ea.attn_status_string(4) == "ATTN_ERR_TIMEOUT"
    assert ea.attn_status_string(99) == "ATTN_ERR_UNKNOWN"


# fake, 16-byte-aligned addresses: the calls below must fail their argument checks before any
# CUDA call, so these are never dereferenced
P = ctypes.c_void_p(0x10000)
P2 = ctypes.c_void_p(0x20000)
NULL = ctypes.c_void_p(0)
MIS = ctypes.c_void_p(0x10008)


def _fwd(L, q=P, k=P, v=P, o=P2, lse=NULL, B=1, H=1, N=128, d=128, scale=0.1, causal=0, dtype=0, o_dtype=0):
    return L.attn_fwd(q, k, v, o, lse, B, H, N, d, scale, causal, dtype, o_dtype, NULL)


@pytest.mark.parametrize("kw", [
    dict(q=NULL), dict(k=NULL), dict(v=NULL), dict(o=NULL), dict(q=MIS), dict(o=MIS), dict(lse=MIS),
    dict(B=0), dict(H=-1), dict(N=0), dict(scale=0.0), dict(scale=-1.0), dict(scale=float("inf")),
    dict(scale=float("nan")), dict(causal=2), dict(o_dtype=2), dict(dtype=7), dict(B=1 << 16, H=1 << 16),
])
def test_fwd_rejects_bad_arguments(L, kw):
    assert _fwd(L, **kw) == ea.ATTN_ERR_INVALID_ARG


@pytest.mark.parametrize("kw", [dict(d=96), dict(d=32), dict(d=512), dict(dtype=ea.ATTN_E4M3), dict(dtype=ea.ATTN_FP32)])
def test_fwd_reports_unsupported(L, kw):
    assert _fwd(L, **kw) == ea.ATTN_ERR_UNSUPPORTED


def test_hadamard_quant_rejects_bad_arguments(L):
    f = L.attn_hadamard_quant
    assert f(NULL, P, P2, NULL, 1, 1, 128, 128, NULL) == ea.ATTN_ERR_INVALID_ARG
    assert f(P, NULL, P2, NULL, 1, 1, 128, 128, NULL) == ea.ATTN_ERR_INVALID_ARG
    assert f(P, P, NULL, NULL, 1, 1, 128, 128, NULL) == ea.ATTN_ERR_INVALID_ARG
    assert f(P, P, P2, MIS, 1, 1, 128, 128, NULL) == ea.ATTN_ERR_INVALID_ARG
    assert f(P, P, P2, NULL, 1, 0, 128, 128, NULL) == ea.ATTN_ERR_INVALID_ARG
    assert f(P, P, P2, NULL, 1, 1, 128, 48, NULL) == ea.ATTN_ERR_UNSUPPORTED


def test_hadamard_quant_qkv_rejects_bad_arguments(L):
    f = L.attn_hadamard_quant_qkv
    ok = [P, P, P, P2, P2, P2, P2, P2, P2, P, 1, 1, 128, 128, NULL]
    for i in range(10):
        a = list(ok)
        a[i] = NULL
        assert f(*a) == ea.ATTN_ERR_INVALID_ARG, i
    a = list(ok)
    a[0] = MIS
    assert f(*a) == ea.ATTN_ERR_INVALID_ARG
    a = list(ok)
    a[13] = 32
    assert f(*a) == ea.ATTN_ERR_UNSUPPORTED


def test_fwd_fp8_rejects_bad_arguments(L):
    f = L.attn_fwd_fp8
    ok = [P, P, P, P2, P2, P2, P2, NULL, 1, 1, 128, 128, 0.1, 0, 0, NULL]
    for i in range(7):
        a = list(ok)
        a[i] = NULL
        assert f(*a) == ea.ATTN_ERR_INVALID_ARG, i
    a = list(ok)
    a[11] = 96
    assert f(*a) == ea.ATTN_ERR_UNSUPPORTED
    a = list(ok)
    a[12] = -0.5
    assert f(*a) == ea.ATTN_ERR_INVALID_ARG


def test_fwd_qk_rejects_bad_arguments(L):
    f = L.attn_fwd_qk
    ok = [P, P, P, P2, NULL, 1, 1, 128, 300, 128, 0.1, 1, 0, 0, NULL]
    for i in range(4):
        a = list(ok)
        a[i] = NULL
        assert f(*a) == ea.ATTN_ERR_INVALID_ARG, i
    for idx, val in [(7, 0), (8, 0), (8, -3), (10, 0.0), (11, 3), (13, 5)]:
        a = list(ok)
        a[idx] = val
        assert f(*a) == ea.ATTN_ERR_INVALID_ARG, (idx, val)
    a = list(ok)
    a[9] = 96
    assert f(*a) == ea.ATTN_ERR_UNSUPPORTED


def test_fwd_strided_rejects_bad_arguments(L):
    f = L.attn_fwd_strided
    B, H, Nq, Nk, d = 2, 4, 128, 300, 128

    def strides(vals):
        return ctypes.cast((ctypes.c_longlong * 12)(*vals), ctypes.c_void_p)

    # [B, N, H, d] sequence-major strides for all four tensors
    good = [Nq * H * d, d, H * d, Nk * H * d, d, H * d, Nk * H * d, d, H * d, Nq * H * d, d, H * d]
    ok = [P, P, P, P2, NULL, B, H, Nq, Nk, d, strides(good), 0.1, 1, 0, 0, NULL]
    a = list(ok)
    a[10] = NULL
    assert f(*a) == ea.ATTN_ERR_INVALID_ARG
    for i in range(4):
        a = list(ok)
        a[i] = NULL
        assert f(*a) == ea.ATTN_ERR_INVALID_ARG, i
    # strides that are not positive multiples of 8 elements, or too large
    for pos, val in [(0, 0), (1, 4), (2, -8), (5, 12), (11, 1), (9, 1 << 36)]:
        bad = list(good)
        bad[pos] = val
        a = list(ok)
        a[10] = strides(bad)
        assert f(*a) == ea.ATTN_ERR_INVALID_ARG, (pos, val)
    # a stride of an extent-1 dimension is ignored: with H = 1 the head strides may be anything,
    # so the call reaches the head-dimension check
    bad = list(good)
    bad[1] = bad[4] = bad[7] = bad[10] = 3
    a = list(ok)
    a[6], a[9], a[10] = 1, 96, strides(bad)
    assert f(*a) == ea.ATTN_ERR_UNSUPPORTED
    for idx, val in [(7, 0), (8, 0), (11, 0.0), (12, 3), (14, 5)]:
        a = list(ok)
        a[idx] = val
        assert f(*a) == ea.ATTN_ERR_INVALID_ARG, (idx, val)


def test_fwd_varlen_rejects_bad_arguments(L):
    f = L.attn_fwd_varlen
    H, d = 4, 128
    CU = ctypes.c_void_p(0x30000)  # 4-byte aligned suffices for the offset arrays

    def strides(vals):
        return ctypes.cast((ctypes.c_longlong * 8)(*vals), ctypes.c_void_p)

    good = [H * d, d] * 4  # {row, head} for q, k, v, o
    ok = [P, P, P, P2, NULL, CU, CU, 3, H, 1000, 900, 512, d, strides(good), 0.1, 1, 0, 0, NULL]
    for i in (0, 1, 2, 3, 5, 6, 13):
        a = list(ok)
        a[i] = NULL
        assert f(*a) == ea.ATTN_ERR_INVALID_ARG, i
    for i in (5, 6):
        a = list(ok)
        a[i] = ctypes.c_void_p(0x30002)
        assert f(*a) == ea.ATTN_ERR_INVALID_ARG, i
    for idx, val in [(7, 0), (8, 0), (9, 0), (10, -1), (11, 0), (14, 0.0), (15, 2), (17, 4)]:
        a = list(ok)
        a[idx] = val
        assert f(*a) == ea.ATTN_ERR_INVALID_ARG, (idx, val)
    for pos, val in [(0, 4), (1, 0), (3, -8), (6, 12), (7, 1 << 36)]:
        bad = list(good)
        bad[pos] = val
        a = list(ok)
        a[13] = strides(bad)
        assert f(*a) == ea.ATTN_ERR_INVALID_ARG, (pos, val)
    a = list(ok)
    a[12] = 96
    assert f(*a) == ea.ATTN_ERR_UNSUPPORTED
    a = list(ok)
    a[16] = 2  # E4M3 inputs are not built for packed batches
    assert f(*a) == ea.ATTN_ERR_UNSUPPORTED


def test_rope_hadamard_quant_qkv_rejects_bad_arguments(L):
    f = L.attn_rope_hadamard_quant_qkv
    ok = [P, P, P, P2, P2, P2, P2, P2, P2, P, P, P, 256, 1, 2, 256, 128, NULL]
    for i in range(12):
        a = list(ok)
        a[i] = NULL
        assert f(*a) == ea.ATTN_ERR_INVALID_ARG, i
    for i in (10, 11):
        a = list(ok)
        a[i] = MIS
        assert f(*a) == ea.ATTN_ERR_INVALID_ARG, i
    for idx, val in [(12, 255), (13, 0), (14, 0), (15, 0)]:
        a = list(ok)
        a[idx] = val
        assert f(*a) == ea.ATTN_ERR_INVALID_ARG, (idx, val)
    a = list(ok)
    a[16] = 96
    assert f(*a) == ea.ATTN_ERR_UNSUPPORTED


def _strides(vals):
    return ctypes.cast((ctypes.c_longlong * len(vals))(*vals), ctypes.c_void_p)


def test_bwd_strided_rejects_bad_arguments(L):
    f = L.attn_bwd_strided
    B, H, Nq, Nk, d = 2, 4, 128, 300, 128
    q_s, k_s = [Nq * H * d, d, H * d], [Nk * H * d, d, H * d]
    good = q_s + k_s + k_s + q_s + q_s + q_s + k_s + k_s  # q k v o dout dq dk dv
    ok = [P, P, P, P, P, P, P2, P2, P2, P2, B, H, Nq, Nk, d, _strides(good), 0.1, 1, 0, NULL]
    a = list(ok)
    a[15] = NULL
    assert f(*a) == ea.ATTN_ERR_INVALID_ARG
    for i in range(10):
        a = list(ok)
        a[i] = NULL
        assert f(*a) == ea.ATTN_ERR_INVALID_ARG, i
    for pos, val in [(2, 4), (5, 0), (14, -8), (23, 1 << 36), (20, 12)]:
        bad = list(good)
        bad[pos] = val
        a = list(ok)
        a[15] = _strides(bad)
        assert f(*a) == ea.ATTN_ERR_INVALID_ARG, (pos, val)
    a = list(ok)
    a[14] = 256
    assert f(*a) == ea.ATTN_ERR_UNSUPPORTED


def test_bwd_varlen_rejects_bad_arguments(L):
    f = L.attn_bwd_varlen
    H, d = 4, 64
    CU = ctypes.c_void_p(0x30000)
    good = [H * d, d] * 8
    ok = [P, P, P, P, P, P, P2, P2, P2, P2, CU, CU, 3, H, 1000, 900, 512, 600, d, _strides(good), 0.1, 1, 0, NULL]
    for i in (0, 4, 5, 9, 10, 11, 19):
        a = list(ok)
        a[i] = NULL
        assert f(*a) == ea.ATTN_ERR_INVALID_ARG, i
    for i in (10, 11):
        a = list(ok)
        a[i] = ctypes.c_void_p(0x30002)
        assert f(*a) == ea.ATTN_ERR_INVALID_ARG, i
    for idx, val in [(12, 0), (13, 0), (14, 0), (15, -1), (16, 0), (17, 0), (20, 0.0), (21, 2), (22, 5)]:
        a = list(ok)
        a[idx] = val
        assert f(*a) == ea.ATTN_ERR_INVALID_ARG, (idx, val)
    bad = list(good)
    bad[0] = 12
    a = list(ok)
    a[19] = _strides(bad)
    assert f(*a) == ea.ATTN_ERR_INVALID_ARG
    a = list(ok)
    a[18] = 256
    assert f(*a) == ea.ATTN_ERR_UNSUPPORTED


def test_fwd_fp8_qk_rejects_bad_arguments(L):
    f = L.attn_fwd_fp8_qk
    ok = [P, P, P, P, P, P, P2, NULL, 1, 2, 128, 300, 128, 0.1, 1, 0, NULL]
    for i in range(7):
        a = list(ok)
        a[i] = NULL
        assert f(*a) == ea.ATTN_ERR_INVALID_ARG, i
    for idx, val in [(8, 0), (10, 0), (11, 0), (11, -2), (13, 0.0), (14, 2), (15, 7)]:
        a = list(ok)
        a[idx] = val
        assert f(*a) == ea.ATTN_ERR_INVALID_ARG, (idx, val)
    a = list(ok)
    a[12] = 96
    assert f(*a) == ea.ATTN_ERR_UNSUPPORTED


def test_hadamard_quant_qkv_strided_rejects_bad_arguments(L):
    f = L.attn_hadamard_quant_qkv_strided
    B, H, N, d = 2, 4, 300, 128
    # the head views of one fused [B, N, 3, H, d] projection
    good = [N * 3 * H * d, d, 3 * H * d] * 3
    ok = [P, P, P, P2, P2, P2, P2, P2, P2, P, B, H, N, d, _strides(good), NULL]
    a = list(ok)
    a[14] = NULL
    assert f(*a) == ea.ATTN_ERR_INVALID_ARG
    for i in range(10):
        a = list(ok)
        a[i] = NULL
        assert f(*a) == ea.ATTN_ERR_INVALID_ARG, i
    for pos, val in [(0, 0), (1, 4), (2, -8), (5, 12), (8, 1 << 36)]:
        bad = list(good)
        bad[pos] = val
        a = list(ok)
        a[14] = _strides(bad)
        assert f(*a) == ea.ATTN_ERR_INVALID_ARG, (pos, val)
    for idx, val in [(10, 0), (11, 0), (12, 0)]:
        a = list(ok)
        a[idx] = val
        assert f(*a) == ea.ATTN_ERR_INVALID_ARG, (idx, val)
    a = list(ok)
    a[13] = 32
    assert f(*a) == ea.ATTN_ERR_UNSUPPORTED


def test_fwd_fp8_strided_rejects_bad_arguments(L):
    f = L.attn_fwd_fp8_strided
    B, H, Nq, Nk, d = 2, 4, 128, 300, 128
    # contiguous codes, O sequence-major [B, Nq, H, d]
    good = [H * Nq * d, Nq * d, d, H * Nk * d, Nk * d, d, H * Nk * d, Nk * d, d, Nq * H * d, d, H * d]
    ok = [P, P, P, P2, P2, P2, P2, NULL, B, H, Nq, Nk, d, _strides(good), 0.1, 1, 0, NULL]
    a = list(ok)
    a[13] = NULL
    assert f(*a) == ea.ATTN_ERR_INVALID_ARG
    for i in range(7):
        a = list(ok)
        a[i] = NULL
        assert f(*a) == ea.ATTN_ERR_INVALID_ARG, i
    # code strides must be multiples of 16 elements (16 bytes), O strides multiples of 8
    for pos, val in [(0, 8), (2, 8), (4, 24), (8, 0), (9, 4), (11, -8), (10, 1 << 36)]:
        bad = list(good)
        bad[pos] = val
        a = list(ok)
        a[13] = _strides(bad)
        assert f(*a) == ea.ATTN_ERR_INVALID_ARG, (pos, val)
    for idx, val in [(8, 0), (10, 0), (11, 0), (14, 0.0), (15, 2), (16, 7)]:
        a = list(ok)
        a[idx] = val
        assert f(*a) == ea.ATTN_ERR_INVALID_ARG, (idx, val)
    a = list(ok)
    a[12] = 96
    assert f(*a) == ea.ATTN_ERR_UNSUPPORTED


def test_hadamard_quant_qkv_varlen_rejects_bad_arguments(L):
    f = L.attn_hadamard_quant_qkv_varlen
    H, d = 4, 128
    good = [H * d, d] * 3
    ok = [P, P, P, P2, P2, P2, P2, P2, P2, P, P, P, 3, H, 1000, 900, 500, 400, d, _strides(good), NULL]
    for i in range(12):
        a = list(ok)
        a[i] = NULL
        assert f(*a) == ea.ATTN_ERR_INVALID_ARG, i
    a = list(ok)
    a[19] = NULL
    assert f(*a) == ea.ATTN_ERR_INVALID_ARG
    a = list(ok)
    a[10] = ctypes.c_void_p(0x10002)  # offsets not 4-byte aligned
    assert f(*a) == ea.ATTN_ERR_INVALID_ARG
    for idx, val in [(12, 0), (13, 0), (14, 0), (15, -1), (16, 0), (17, 0), (14, 0x7FFFFFFF)]:
        a = list(ok)
        a[idx] = val
        assert f(*a) == ea.ATTN_ERR_INVALID_ARG, (idx, val)
    bad = list(good)
    bad[0] = 12
    a = list(ok)
    a[19] = _strides(bad)
    assert f(*a) == ea.ATTN_ERR_INVALID_ARG
    a = list(ok)
    a[18] = 96
    assert f(*a) == ea.ATTN_ERR_UNSUPPORTED


def test_fwd_fp8_varlen_rejects_bad_arguments(L):
    f = L.attn_fwd_fp8_varlen
    ok = [P, P, P, P2, P2, P2, P, NULL, P, P, 3, 4, 1000, 900, 500, 400, 128, 0.1, 1, 0, NULL]
    for i in range(7):
        a = list(ok)
        a[i] = NULL
        assert f(*a) == ea.ATTN_ERR_INVALID_ARG, i
    for i in (8, 9):
        a = list(ok)
        a[i] = NULL
        assert f(*a) == ea.ATTN_ERR_INVALID_ARG, i
    for idx, val in [(10, 0), (11, 0), (12, 0), (13, 0), (14, 0), (15, 0), (17, 0.0), (18, 2), (19, 9)]:
        a = list(ok)
        a[idx] = val
        assert f(*a) == ea.ATTN_ERR_INVALID_ARG, (idx, val)
    a = list(ok)
    a[16] = 96
    assert f(*a) == ea.ATTN_ERR_UNSUPPORTED


def test_merge_partials_rejects_bad_arguments(L):
    f = L.attn_merge_partials
    ok = [P, P, P2, P2, 1000, 128, 0, NULL]
    for i in range(4):
        a = list(ok)
        a[i] = NULL
        assert f(*a) == ea.ATTN_ERR_INVALID_ARG, i
    for i in (0, 2):
        a = list(ok)
        a[i] = MIS
        assert f(*a) == ea.ATTN_ERR_INVALID_ARG, i
    a = list(ok)
    a[1] = ctypes.c_void_p(0x10002)  # LSE arrays need 4-byte alignment
    assert f(*a) == ea.ATTN_ERR_INVALID_ARG
    for idx, val in [(4, 0), (4, -1), (4, (1 << 40) + 1), (5, 0), (5, 6), (5, 2048), (6, 2)]:
        a = list(ok)
        a[idx] = val
        assert f(*a) == ea.ATTN_ERR_INVALID_ARG, (idx, val)


def test_work_unit_count_overflow_is_refused(L):
    """B * H * ceil(N / 128) units must fit an int: refused on the host, before any CUDA call."""
    for f in (L.attn_fwd, L.attn_fwd_noalloc):
        assert f(P, P, P, P2, NULL, 65536, 1024, 1 << 30, 128, 0.1, 0, 0, 0, NULL) == ea.ATTN_ERR_INVALID_ARG
    assert L.attn_fwd_qk(P, P, P, P2, NULL, 65536, 1024, 1 << 30, 128, 128, 0.1, 0, 0, 0, NULL) == \
        ea.ATTN_ERR_INVALID_ARG


def test_bwd_workspace_bytes(L):
    assert L.attn_bwd_workspace_bytes(1, 1, 1) == 2 * 128 * 4
    assert L.attn_bwd_workspace_bytes(2, 16, 8192) == 2 * 32 * 8192 * 4
    assert L.attn_bwd_workspace_bytes(1, 3, 129) == 2 * 3 * 256 * 4
    assert L.attn_bwd_workspace_bytes(0, 1, 1) == 0
    assert L.attn_bwd_workspace_bytes(1, 1, -5) == 0


def test_bwd_ds_workspace_bytes(L):
    f = L.attn_bwd_ds_workspace_bytes
    nb = 64
    head = (2 * 32 * nb * 128 * 4 + 1023) // 1024 * 1024
    assert f(2, 16, 8192, 1) == head + 32 * (nb * (nb + 1) // 2) * 32768
    assert f(2, 16, 8192, 0) == head + 32 * nb * nb * 32768
    assert f(1, 1, 1, 1) == 1024 + 32768
    for a in [(0, 1, 128, 0), (1, 0, 128, 0), (1, 1, 0, 0), (1, 1, 128, 2)]:
        assert f(*a) == 0, a
    # 2^31 - 1 tiles or more cannot be addressed by the dQ pass's tensor map
    assert f(1, 1 << 20, 1 << 14, 0) == 0


def test_bwd_ds_rejects_bad_arguments(L):
    f = L.attn_bwd_ds
    ok = [P, P, P, P, P, P2, P, P, P, P, 1, 2, 256, 128, 0.1, 1, 0, NULL]
    for i in range(10):
        a = list(ok)
        a[i] = NULL
        assert f(*a) == ea.ATTN_ERR_INVALID_ARG, i
    for idx, val in [(10, 0), (11, 0), (12, 0), (14, 0.0), (15, 2), (16, 7)]:
        a = list(ok)
        a[idx] = val
        assert f(*a) == ea.ATTN_ERR_INVALID_ARG, (idx, val)
    a = list(ok)
    a[13] = 256
    assert f(*a) == ea.ATTN_ERR_UNSUPPORTED
    a = list(ok)
    a[11], a[12], a[15] = 1 << 20, 1 << 14, 0  # too many dS tiles
    assert f(*a) == ea.ATTN_ERR_INVALID_ARG


def test_bwd_varlen_ds_workspace_bytes_and_rejections(L):
    f = L.attn_bwd_varlen_ds_workspace_bytes
    head = (2 * 128 * 27 * 128 * 4 + 1023) // 1024 * 1024
    assert f(8, 16, 3369, 3369) == head + 128 * 27 * 27 * 32768
    assert f(1, 1, 1, 300) == 1024 + 3 * 32768
    for a in [(0, 1, 1, 1), (1, 0, 1, 1), (1, 1, 0, 1), (1, 1, 1, 0)]:
        assert f(*a) == 0, a
    g = L.attn_bwd_varlen_ds
    good = [16 * 128, 128] * 8
    ok = [P, P, P, P, P, P2, P, P, P, P, P, P, 3, 16, 1000, 900, 500, 400, 128, _strides(good), 0.1, 1, 0, NULL]
    for i in range(12):
        a = list(ok)
        a[i] = NULL
        assert g(*a) == ea.ATTN_ERR_INVALID_ARG, i
    for idx, val in [(12, 0), (13, 0), (14, 0), (15, 0), (16, 0), (17, 0), (20, 0.0), (21, 2)]:
        a = list(ok)
        a[idx] = val
        assert g(*a) == ea.ATTN_ERR_INVALID_ARG, (idx, val)
    a = list(ok)
    a[18] = 256
    assert g(*a) == ea.ATTN_ERR_UNSUPPORTED


def test_bwd_rejects_bad_arguments(L):
    f = L.attn_bwd
    ok = [P, P, P, P, P, P2, P2, P2, P2, P2, 1, 1, 128, 128, 0.1, 0, 0, NULL]
    for i in range(10):
        a = list(ok)
        a[i] = NULL
        assert f(*a) == ea.ATTN_ERR_INVALID_ARG, i
    for i in range(10):
        a = list(ok)
        a[i] = MIS
        assert f(*a) == ea.ATTN_ERR_INVALID_ARG, i
    for idx, val in [(10, 0), (12, 0), (14, float("nan")), (14, -1.0), (15, 2), (16, 7)]:
        a = list(ok)
        a[idx] = val
        assert f(*a) == ea.ATTN_ERR_INVALID_ARG, (idx, val)
    for dd in (32, 256):
        a = list(ok)
        a[13] = dd
        assert f(*a) == ea.ATTN_ERR_UNSUPPORTED, dd


def test_bwd_qk_rejects_bad_arguments(L):
    f = L.attn_bwd_qk
    ok = [P, P, P, P, P, P2, P2, P2, P2, P2, 1, 1, 128, 300, 128, 0.1, 1, 0, NULL]
    for i in range(10):
        a = list(ok)
        a[i] = NULL
        assert f(*a) == ea.ATTN_ERR_INVALID_ARG, i
    for idx, val in [(12, 0), (13, 0), (13, -1), (15, 0.0), (16, 2), (17, 9)]:
        a = list(ok)
        a[idx] = val
        assert f(*a) == ea.ATTN_ERR_INVALID_ARG, (idx, val)
    a = list(ok)
    a[14] = 256
    assert f(*a) == ea.ATTN_ERR_UNSUPPORTED


def test_python_binding_has_same_names():
    for name in ["attn_fwd", "attn_hadamard_quant", "attn_fwd_fp8", "attn_device_status", "attn_status_string",
                 "attn_num_kernel_launches", "attn_shutdown", "attn_fwd_noalloc", "attn_hadamard_quant_qkv",
                 "attn_bwd", "attn_bwd_workspace_bytes", "attn_fwd_qk", "attn_bwd_qk", "attn_fwd_strided",
                 "attn_fwd_varlen", "attn_rope_hadamard_quant_qkv", "attn_bwd_strided", "attn_bwd_varlen",
                 "attn_fwd_fp8_qk", "attn_merge_partials", "attn_selftest_wait_timeout", "attn_noalloc_status",
                 "attn_noalloc_selftest_wait_timeout", "attn_hadamard_quant_qkv_strided", "attn_fwd_fp8_strided",
                 "attn_fwd_schedule", "attn_hadamard_quant_qkv_varlen", "attn_fwd_fp8_varlen",
                 "attn_bwd_ds_workspace_bytes", "attn_bwd_ds", "attn_bwd_varlen_ds_workspace_bytes",
                 "attn_bwd_varlen_ds"]:
        assert callable(getattr(ea, name)), name


def test_binding_refuses_host_tensors_before_any_library_call(L):
    """A tensor in host memory would reach a kernel as a host pointer: the binding raises before
    the call (no GPU needed to check it)."""
    torch = pytest.importorskip("torch")
    q = torch.zeros(1, 1, 128, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        ea.attn_fwd(q, q, q)
    with pytest.raises(ValueError):
        ea.attn_hadamard_quant(q)
    with pytest.raises(ValueError):  # a wrong output dtype is refused before the pointers are taken
        ea.attn_fwd(q, q, q, o=torch.zeros(1, 1, 128, 64, dtype=torch.uint8))
