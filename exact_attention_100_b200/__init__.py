"""Exact attention forward for NVIDIA B200 (sm_100a): Python binding of ``include/attn.h``.

Argument marshalling only: every step of the computation runs in the CUDA kernels of
``libattn_b200.so``; torch supplies device memory and the current stream.  There is no CPU
fallback: if the library is missing or a call fails, an exception is raised.

    import torch, exact_attention_100_b200 as ea
    o, lse = ea.attn_fwd(q, k, v, causal=True)           # q, k, v: [B, H, N, d] bf16 on cuda
    q8, qs = ea.attn_hadamard_quant(q, signs)             # E4M3 codes + per-block scales
    dq, dk, dv = ea.attn_bwd(q, k, v, o, lse, do, causal=True)  # backward (bf16 O from attn_fwd)

Entry points, by family:

* forward: ``attn_fwd``, ``attn_fwd_qk`` (key length != query length), ``attn_fwd_strided``
  (any strides, e.g. sequence-major or fused QKV), ``attn_fwd_varlen`` (packed batches),
  ``attn_fwd_noalloc`` (no device allocation; ``attn_noalloc_status`` reads its status word);
* FP8: ``attn_hadamard_quant``, ``attn_hadamard_quant_qkv``, ``attn_rope_hadamard_quant_qkv``
  (rotary embedding fused), ``attn_fwd_fp8``, ``attn_fwd_fp8_qk``;
* backward: ``attn_bwd``, ``attn_bwd_qk``, ``attn_bwd_strided``, ``attn_bwd_varlen``,
  ``attn_bwd_workspace_bytes``;
* sequence parallelism: ``attn_merge_partials`` and the ring driver in
  :mod:`exact_attention_100_b200.ring`;
* status: ``attn_device_status``, ``attn_status_string``, ``attn_num_kernel_launches``,
  ``attn_selftest_wait_timeout``, ``attn_noalloc_selftest_wait_timeout``, ``attn_shutdown``.
"""

from __future__ import annotations

import ctypes
import math
import os

ATTN_OK = 0
ATTN_ERR_INVALID_ARG = 1
ATTN_ERR_UNSUPPORTED = 2
ATTN_ERR_CUDA = 3
ATTN_ERR_TIMEOUT = 4

ATTN_BF16 = 0
ATTN_FP32 = 1
ATTN_E4M3 = 2

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libattn_b200.so")

_lib = None


class AttnError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {attn_status_string(status)}")


def lib() -> ctypes.CDLL:
    """The loaded C library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with `python -m exact_attention_100_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, i, f = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
        L.attn_fwd.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, f, i, i, i, vp]
        L.attn_fwd.restype = i
        L.attn_fwd_qk.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, f, i, i, i, vp]
        L.attn_fwd_qk.restype = i
        L.attn_fwd_strided.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, vp, f, i, i, i, vp]
        L.attn_fwd_strided.restype = i
        L.attn_fwd_varlen.argtypes = [vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, vp, f, i, i, i, vp]
        L.attn_fwd_varlen.restype = i
        L.attn_bwd_strided.argtypes = [vp] * 10 + [i, i, i, i, i, vp, f, i, i, vp]
        L.attn_bwd_strided.restype = i
        L.attn_bwd_varlen.argtypes = [vp] * 12 + [i, i, i, i, i, i, i, vp, f, i, i, vp]
        L.attn_bwd_varlen.restype = i
        L.attn_bwd_varlen_ds.argtypes = [vp] * 12 + [i, i, i, i, i, i, i, vp, f, i, i, vp]
        L.attn_bwd_varlen_ds.restype = i
        L.attn_bwd_varlen_ds_workspace_bytes.argtypes = [i, i, i, i]
        L.attn_bwd_varlen_ds_workspace_bytes.restype = ctypes.c_ulonglong
        L.attn_hadamard_quant.argtypes = [vp, vp, vp, vp, i, i, i, i, vp]
        L.attn_hadamard_quant.restype = i
        L.attn_hadamard_quant_qkv.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, vp]
        L.attn_rope_hadamard_quant_qkv.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, vp]
        L.attn_rope_hadamard_quant_qkv.restype = i
        L.attn_hadamard_quant_qkv.restype = i
        L.attn_hadamard_quant_qkv_strided.argtypes = [vp] * 10 + [i, i, i, i, vp, vp]
        L.attn_hadamard_quant_qkv_strided.restype = i
        L.attn_fwd_fp8.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, f, i, i, vp]
        L.attn_fwd_fp8.restype = i
        L.attn_fwd_fp8_qk.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, f, i, i, vp]
        L.attn_fwd_fp8_qk.restype = i
        L.attn_fwd_fp8_strided.argtypes = [vp] * 8 + [i, i, i, i, i, vp, f, i, i, vp]
        L.attn_fwd_fp8_strided.restype = i
        L.attn_hadamard_quant_qkv_varlen.argtypes = [vp] * 12 + [i] * 7 + [vp, vp]
        L.attn_hadamard_quant_qkv_varlen.restype = i
        L.attn_fwd_fp8_varlen.argtypes = [vp] * 10 + [i] * 7 + [f, i, i, vp]
        L.attn_fwd_fp8_varlen.restype = i
        L.attn_merge_partials.argtypes = [vp, vp, vp, vp, ctypes.c_longlong, i, i, vp]
        L.attn_merge_partials.restype = i
        L.attn_selftest_wait_timeout.argtypes = [vp]
        L.attn_selftest_wait_timeout.restype = i
        L.attn_fwd_noalloc.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, f, i, i, i, vp]
        L.attn_fwd_noalloc.restype = i
        L.attn_noalloc_status.argtypes = [vp]
        L.attn_noalloc_status.restype = i
        L.attn_noalloc_selftest_wait_timeout.argtypes = [vp]
        L.attn_noalloc_selftest_wait_timeout.restype = i
        L.attn_fwd_schedule.argtypes = [i, i, i, i, i, i, i, i, vp, ctypes.c_longlong, vp]
        L.attn_fwd_schedule.restype = i
        L.attn_bwd_workspace_bytes.argtypes = [i, i, i]
        L.attn_bwd_workspace_bytes.restype = ctypes.c_ulonglong
        L.attn_bwd_ds_workspace_bytes.argtypes = [i, i, i, i]
        L.attn_bwd_ds_workspace_bytes.restype = ctypes.c_ulonglong
        L.attn_bwd_ds.argtypes = [vp] * 10 + [i, i, i, i, f, i, i, vp]
        L.attn_bwd_ds.restype = i
        L.attn_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, f, i, i, vp]
        L.attn_bwd.restype = i
        L.attn_bwd_qk.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, f, i, i, vp]
        L.attn_bwd_qk.restype = i
        L.attn_device_status.argtypes = [vp]
        L.attn_device_status.restype = i
        L.attn_status_string.argtypes = [i]
        L.attn_status_string.restype = ctypes.c_char_p
        L.attn_num_kernel_launches.argtypes = []
        L.attn_num_kernel_launches.restype = ctypes.c_ulonglong
        L.attn_shutdown.argtypes = []
        L.attn_shutdown.restype = None
        _lib = L
    return _lib


def attn_status_string(status: int) -> str:
    return lib().attn_status_string(int(status)).decode()


def attn_num_kernel_launches() -> int:
    return int(lib().attn_num_kernel_launches())


def attn_shutdown() -> None:
    lib().attn_shutdown()


def _stream_ptr(stream):
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t):
    """Device pointer of a tensor on the current CUDA device (the kernels would fault on any
    other address), or NULL for None."""
    if t is None:
        return ctypes.c_void_p(0)
    import torch
    if not t.is_cuda or t.device.index != torch.cuda.current_device():
        raise ValueError(f"a {tuple(t.shape)} tensor is on {t.device}, not on the current CUDA device")
    return ctypes.c_void_p(t.data_ptr())


def _out(t, shape, dtypes, what, strided=False):
    """Checks a caller-supplied output (or scale array): the kernels write (or read) exactly
    `shape` elements of one of `dtypes`, contiguous or, with `strided`, through the tensor's own
    strides with a contiguous last dimension."""
    layout_ok = t.stride(-1) == 1 if strided else t.is_contiguous()
    if tuple(t.shape) != tuple(int(x) for x in shape) or t.dtype not in dtypes or not layout_ok:
        names = "/".join(str(x).replace("torch.", "") for x in dtypes)
        raise ValueError(f"{what} must be {names} of shape {tuple(int(x) for x in shape)}"
                         f"{' with a contiguous last dimension' if strided else ', contiguous'}")
    return t


def _signs(signs, d):
    """The transform's signs: None, or d int8 entries (the kernels read d of them)."""
    import torch
    if signs is not None:
        _out(signs, (d,), (torch.int8,), "signs")
    return signs


def _grads(dq, dk, dv, q_shape, k_shape, strided=False):
    import torch
    for g, shp, name in ((dq, q_shape, "dq"), (dk, k_shape, "dk"), (dv, k_shape, "dv")):
        _out(g, shp, (torch.bfloat16, torch.float32), name, strided)
    if not dq.dtype == dk.dtype == dv.dtype:
        raise ValueError("dq, dk and dv must have one dtype")


def _outs_qkv(outs, q_shape, k_shape, scale_q, scale_k):
    import torch
    if len(outs) != 6:
        raise ValueError("outs must be (q8, k8, v8, q_scale, k_scale, v_scale)")
    for t, shp, name in zip(outs, (q_shape, k_shape, k_shape, scale_q, scale_k, scale_k),
                            ("q8", "k8", "v8", "q_scale", "k_scale", "v_scale")):
        _out(t, shp, (torch.uint8,) if name.endswith("8") else (torch.float32,), name)


def _check(status: int, what: str) -> None:
    if status != ATTN_OK:
        raise AttnError(status, what)


def _dims(q):
    if q.dim() != 4:
        raise ValueError("expected [B, H, N, d]")
    return tuple(int(x) for x in q.shape)


def attn_fwd(q, k, v, o=None, lse=None, scale=None, causal=False, o_dtype=None, stream=None,
             want_lse=True):
    """O = softmax(scale * Q K^T) V and LSE for contiguous [B, H, N, d] bf16 cuda tensors.

    ``o`` / ``lse`` may be given (written in place) or are allocated; ``o_dtype`` is
    torch.bfloat16 (default) or torch.float32; ``scale`` defaults to 1/sqrt(d).
    Returns ``(o, lse)`` (lse is None when ``want_lse`` is False and none was given).
    """
    import torch
    B, H, N, d = _dims(q)
    for t in (q, k, v):
        if t.dtype != torch.bfloat16 or not t.is_contiguous() or t.shape != q.shape:
            raise ValueError("q, k, v must be contiguous bf16 tensors of one shape")
    if o is None:
        o = torch.empty(q.shape, dtype=o_dtype or torch.bfloat16, device=q.device)
    if lse is None and want_lse:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    _out(o, q.shape, (torch.bfloat16, torch.float32), "o")
    if lse is not None:
        _out(lse, (B, H, N), (torch.float32,), "lse")
    od = ATTN_FP32 if o.dtype == torch.float32 else ATTN_BF16
    s = float(scale) if scale is not None else 1.0 / math.sqrt(d)
    _check(lib().attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, N, d, s, int(bool(causal)),
                          ATTN_BF16, od, _stream_ptr(stream)), "attn_fwd")
    return o, lse


def attn_bwd_workspace_bytes(B: int, H: int, N: int) -> int:
    return int(lib().attn_bwd_workspace_bytes(int(B), int(H), int(N)))


def _workspace(workspace, nbytes, device, name):
    """The caller's workspace checked against the ``nbytes`` the call needs (the C entry points
    take no size and would write past a smaller buffer), or a new one of that size."""
    import torch
    if workspace is None:
        return torch.empty(nbytes, dtype=torch.uint8, device=device)
    if not workspace.is_cuda or not workspace.is_contiguous():
        raise ValueError(f"{name}: the workspace must be a contiguous cuda tensor")
    if workspace.numel() * workspace.element_size() < nbytes:
        raise ValueError(f"{name}: the workspace has {workspace.numel() * workspace.element_size()} bytes, "
                         f"{nbytes} are needed")
    return workspace


def attn_bwd(q, k, v, o, lse, dout, dq=None, dk=None, dv=None, workspace=None, scale=None, causal=False,
             g_dtype=None, stream=None):
    """(dQ, dK, dV) of attn_fwd for the upstream gradient ``dout``.

    q, k, v, o, dout: contiguous [B, H, N, d] bf16 cuda tensors (o from attn_fwd with bf16 O);
    lse: the forward's [B, H, N] float32 LSE.  dq/dk/dv may be given (written in place) or are
    allocated with ``g_dtype`` (torch.bfloat16 default, or torch.float32); ``workspace`` (a
    float32 tensor of at least attn_bwd_workspace_bytes bytes) likewise.
    """
    import torch
    B, H, N, d = _dims(q)
    for t in (q, k, v, o, dout):
        if t.dtype != torch.bfloat16 or not t.is_contiguous() or t.shape != q.shape:
            raise ValueError("q, k, v, o, dout must be contiguous bf16 tensors of one shape")
    gd = g_dtype or (dq.dtype if dq is not None else torch.bfloat16)
    dq = dq if dq is not None else torch.empty(q.shape, dtype=gd, device=q.device)
    dk = dk if dk is not None else torch.empty(q.shape, dtype=gd, device=q.device)
    dv = dv if dv is not None else torch.empty(q.shape, dtype=gd, device=q.device)
    _grads(dq, dk, dv, q.shape, q.shape)
    _out(lse, (B, H, N), (torch.float32,), "lse")
    workspace = _workspace(workspace, attn_bwd_workspace_bytes(B, H, N), q.device, "attn_bwd")
    gcode = ATTN_FP32 if dq.dtype == torch.float32 else ATTN_BF16
    s = float(scale) if scale is not None else 1.0 / math.sqrt(d)
    _check(lib().attn_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dout), _ptr(lse), _ptr(dq), _ptr(dk), _ptr(dv),
                          _ptr(workspace), B, H, N, d, s, int(bool(causal)), gcode, _stream_ptr(stream)),
           "attn_bwd")
    return dq, dk, dv


def attn_bwd_ds_workspace_bytes(B, H, N, causal):
    """Bytes of the workspace :func:`attn_bwd_ds` needs (0 if the shape has too many tiles)."""
    return int(lib().attn_bwd_ds_workspace_bytes(B, H, N, int(bool(causal))))


def attn_bwd_ds(q, k, v, o, lse, dout, dq=None, dk=None, dv=None, workspace=None, scale=None, causal=False,
                g_dtype=None, stream=None):
    """attn_bwd with the dS tiles kept in the workspace: dQ is formed from the stored dS instead
    of recomputing S and dP (five products instead of seven), for
    ``attn_bwd_ds_workspace_bytes(B, H, N, causal)`` bytes of workspace (a uint8 tensor) instead
    of attn_bwd_workspace_bytes.  Arguments and results otherwise as :func:`attn_bwd`."""
    import torch
    B, H, N, d = _dims(q)
    for t in (q, k, v, o, dout):
        if t.dtype != torch.bfloat16 or not t.is_contiguous() or t.shape != q.shape:
            raise ValueError("q, k, v, o, dout must be contiguous bf16 tensors of one shape")
    gd = g_dtype or (dq.dtype if dq is not None else torch.bfloat16)
    dq = dq if dq is not None else torch.empty(q.shape, dtype=gd, device=q.device)
    dk = dk if dk is not None else torch.empty(q.shape, dtype=gd, device=q.device)
    dv = dv if dv is not None else torch.empty(q.shape, dtype=gd, device=q.device)
    _grads(dq, dk, dv, q.shape, q.shape)
    _out(lse, (B, H, N), (torch.float32,), "lse")
    nbytes = attn_bwd_ds_workspace_bytes(B, H, N, causal)
    if nbytes == 0:
        raise ValueError("too many dS tiles for this shape: use attn_bwd")
    workspace = _workspace(workspace, nbytes, q.device, "attn_bwd_ds")
    gcode = ATTN_FP32 if dq.dtype == torch.float32 else ATTN_BF16
    s = float(scale) if scale is not None else 1.0 / math.sqrt(d)
    _check(lib().attn_bwd_ds(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dout), _ptr(lse), _ptr(dq), _ptr(dk),
                             _ptr(dv), _ptr(workspace), B, H, N, d, s, int(bool(causal)), gcode,
                             _stream_ptr(stream)), "attn_bwd_ds")
    return dq, dk, dv


def attn_fwd_qk(q, k, v, o=None, lse=None, scale=None, causal=False, o_dtype=None, stream=None):
    """attn_fwd with keys/values [B, H, Nk, d] whose length may differ from the queries'
    [B, H, Nq, d].  Causal masking is bottom-right aligned (key j visible to query i iff
    j <= i + Nk - Nq); rows that see no key get O = 0 and LSE = -inf.  Returns ``(o, lse)``."""
    import torch
    B, H, Nq, d = _dims(q)
    Bk, Hk, Nk, dk = _dims(k)
    if (Bk, Hk, dk) != (B, H, d) or v.shape != k.shape:
        raise ValueError("k and v must be [B, H, Nk, d] with q's B, H, d")
    for t in (q, k, v):
        if t.dtype != torch.bfloat16 or not t.is_contiguous():
            raise ValueError("q, k, v must be contiguous bf16 tensors")
    if o is None:
        o = torch.empty(q.shape, dtype=o_dtype or torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty((B, H, Nq), dtype=torch.float32, device=q.device)
    _out(o, q.shape, (torch.bfloat16, torch.float32), "o")
    _out(lse, (B, H, Nq), (torch.float32,), "lse")
    od = ATTN_FP32 if o.dtype == torch.float32 else ATTN_BF16
    s = float(scale) if scale is not None else 1.0 / math.sqrt(d)
    _check(lib().attn_fwd_qk(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, Nq, Nk, d, s,
                             int(bool(causal)), ATTN_BF16, od, _stream_ptr(stream)), "attn_fwd_qk")
    return o, lse


def attn_fwd_strided(q, k, v, o=None, lse=None, scale=None, causal=False, o_dtype=None, stream=None):
    """attn_fwd_qk on logical [B, H, N, d] bf16 views with any strides whose last one is 1, e.g.
    ``x.view(B, N, H, d).transpose(1, 2)`` of a sequence-major projection; no copy is made.  ``o``
    defaults to a tensor with q's memory order.  Returns ``(o, lse)``."""
    import torch
    B, H, Nq, d = _dims(q)
    Bk, Hk, Nk, dk = _dims(k)
    if (Bk, Hk, dk) != (B, H, d) or v.shape != k.shape:
        raise ValueError("k and v must be [B, H, Nk, d] with q's B, H, d")
    for t in (q, k, v):
        if t.dtype != torch.bfloat16 or t.stride(-1) != 1:
            raise ValueError("q, k, v must be bf16 with a contiguous last dimension")
    if o is None:
        o = torch.empty_like(q, dtype=o_dtype or torch.bfloat16)
    _out(o, q.shape, (torch.bfloat16, torch.float32), "o", strided=True)
    if lse is None:
        lse = torch.empty((B, H, Nq), dtype=torch.float32, device=q.device)
    _out(lse, (B, H, Nq), (torch.float32,), "lse")
    strides = (ctypes.c_longlong * 12)(*[int(x) for t in (q, k, v, o) for x in t.stride()[:3]])
    od = ATTN_FP32 if o.dtype == torch.float32 else ATTN_BF16
    s = float(scale) if scale is not None else 1.0 / math.sqrt(d)
    _check(lib().attn_fwd_strided(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, Nq, Nk, d,
                                  ctypes.cast(strides, ctypes.c_void_p), s, int(bool(causal)), ATTN_BF16, od,
                                  _stream_ptr(stream)), "attn_fwd_strided")
    return o, lse


def attn_fwd_varlen(q, k, v, cu_seqlens_q, cu_seqlens_k, max_seqlen_q, o=None, lse=None, scale=None,
                    causal=False, o_dtype=None, stream=None):
    """Packed variable-length batch: ``q`` [total_q, H, d], ``k``, ``v`` [total_k, H, d] bf16 (any
    row and head strides, last dimension contiguous); sequence b owns query rows
    ``cu_seqlens_q[b]:cu_seqlens_q[b+1]`` and key rows ``cu_seqlens_k[b]:cu_seqlens_k[b+1]``
    (int32 cuda tensors of B + 1 offsets); ``max_seqlen_q`` bounds every query length.
    Returns ``(o [total_q, H, d], lse [H, total_q])``.  Offsets that break their rules are
    reported by the next :func:`attn_device_status`."""
    import torch
    if q.dim() != 3 or k.dim() != 3 or v.shape != k.shape:
        raise ValueError("q must be [total_q, H, d], k and v [total_k, H, d]")
    total_q, H, d = (int(x) for x in q.shape)
    total_k = int(k.shape[0])
    if (int(k.shape[1]), int(k.shape[2])) != (H, d):
        raise ValueError("k and v must have q's H and d")
    for t in (q, k, v):
        if t.dtype != torch.bfloat16 or t.stride(-1) != 1:
            raise ValueError("q, k, v must be bf16 with a contiguous last dimension")
    for c in (cu_seqlens_q, cu_seqlens_k):
        if c.dtype != torch.int32 or c.dim() != 1 or not c.is_contiguous() or not c.is_cuda:
            raise ValueError("cu_seqlens must be contiguous int32 cuda tensors")
    if cu_seqlens_k.shape != cu_seqlens_q.shape:
        raise ValueError("cu_seqlens_q and cu_seqlens_k must both have B + 1 entries")
    B = int(cu_seqlens_q.shape[0]) - 1
    if o is None:
        o = torch.empty_like(q, dtype=o_dtype or torch.bfloat16)
    _out(o, q.shape, (torch.bfloat16, torch.float32), "o", strided=True)
    if lse is None:
        lse = torch.empty((H, total_q), dtype=torch.float32, device=q.device)
    _out(lse, (H, total_q), (torch.float32,), "lse")
    strides = (ctypes.c_longlong * 8)(*[int(x) for t in (q, k, v, o) for x in t.stride()[:2]])
    od = ATTN_FP32 if o.dtype == torch.float32 else ATTN_BF16
    s = float(scale) if scale is not None else 1.0 / math.sqrt(d)
    _check(lib().attn_fwd_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(cu_seqlens_q),
                                 _ptr(cu_seqlens_k), B, H, total_q, total_k, int(max_seqlen_q), d,
                                 ctypes.cast(strides, ctypes.c_void_p), s, int(bool(causal)), ATTN_BF16, od,
                                 _stream_ptr(stream)), "attn_fwd_varlen")
    return o, lse


def attn_bwd_qk(q, k, v, o, lse, dout, dq=None, dk=None, dv=None, workspace=None, scale=None, causal=False,
                g_dtype=None, stream=None):
    """attn_bwd for attn_fwd_qk: q, o, dout [B, H, Nq, d], k, v [B, H, Nk, d] (bf16); returns
    (dq [B, H, Nq, d], dk, dv [B, H, Nk, d])."""
    import torch
    B, H, Nq, d = _dims(q)
    Nk = int(k.shape[2])
    if k.shape != v.shape or tuple(k.shape) != (B, H, Nk, d) or o.shape != q.shape or dout.shape != q.shape:
        raise ValueError("expected q, o, dout [B, H, Nq, d] and k, v [B, H, Nk, d]")
    for t in (q, k, v, o, dout):
        if t.dtype != torch.bfloat16 or not t.is_contiguous():
            raise ValueError("q, k, v, o, dout must be contiguous bf16 tensors")
    gd = g_dtype or (dq.dtype if dq is not None else torch.bfloat16)
    dq = dq if dq is not None else torch.empty(q.shape, dtype=gd, device=q.device)
    dk = dk if dk is not None else torch.empty(k.shape, dtype=gd, device=q.device)
    dv = dv if dv is not None else torch.empty(k.shape, dtype=gd, device=q.device)
    _grads(dq, dk, dv, q.shape, k.shape)
    _out(lse, (B, H, Nq), (torch.float32,), "lse")
    workspace = _workspace(workspace, attn_bwd_workspace_bytes(B, H, Nq), q.device, "attn_bwd")
    gcode = ATTN_FP32 if dq.dtype == torch.float32 else ATTN_BF16
    s = float(scale) if scale is not None else 1.0 / math.sqrt(d)
    _check(lib().attn_bwd_qk(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dout), _ptr(lse), _ptr(dq), _ptr(dk), _ptr(dv),
                             _ptr(workspace), B, H, Nq, Nk, d, s, int(bool(causal)), gcode, _stream_ptr(stream)),
           "attn_bwd_qk")
    return dq, dk, dv


def attn_bwd_strided(q, k, v, o, lse, dout, dq=None, dk=None, dv=None, workspace=None, scale=None, causal=False,
                     g_dtype=None, stream=None):
    """attn_bwd_qk on logical [B, H, N, d] bf16 views with any strides whose last one is 1 (the
    backward of :func:`attn_fwd_strided`); ``lse`` [B, H, Nq] contiguous.  Gradients default to
    tensors with their input's memory order.  Returns ``(dq, dk, dv)``."""
    import torch
    B, H, Nq, d = _dims(q)
    Nk = int(k.shape[2])
    if k.shape != v.shape or tuple(k.shape) != (B, H, Nk, d) or o.shape != q.shape or dout.shape != q.shape:
        raise ValueError("expected q, o, dout [B, H, Nq, d] and k, v [B, H, Nk, d]")
    for t in (q, k, v, o, dout):
        if t.dtype != torch.bfloat16 or t.stride(-1) != 1:
            raise ValueError("q, k, v, o, dout must be bf16 with a contiguous last dimension")
    if lse.dtype != torch.float32 or not lse.is_contiguous() or tuple(lse.shape) != (B, H, Nq):
        raise ValueError("lse must be contiguous float32 [B, H, Nq]")
    gd = g_dtype or (dq.dtype if dq is not None else torch.bfloat16)
    dq = dq if dq is not None else torch.empty_like(q, dtype=gd)
    dk = dk if dk is not None else torch.empty_like(k, dtype=gd)
    dv = dv if dv is not None else torch.empty_like(v, dtype=gd)
    _grads(dq, dk, dv, q.shape, k.shape, strided=True)
    workspace = _workspace(workspace, attn_bwd_workspace_bytes(B, H, Nq), q.device, "attn_bwd")
    strides = (ctypes.c_longlong * 24)(*[int(x) for t in (q, k, v, o, dout, dq, dk, dv) for x in t.stride()[:3]])
    gcode = ATTN_FP32 if dq.dtype == torch.float32 else ATTN_BF16
    s = float(scale) if scale is not None else 1.0 / math.sqrt(d)
    _check(lib().attn_bwd_strided(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dout), _ptr(lse), _ptr(dq), _ptr(dk),
                                  _ptr(dv), _ptr(workspace), B, H, Nq, Nk, d, ctypes.cast(strides, ctypes.c_void_p),
                                  s, int(bool(causal)), gcode, _stream_ptr(stream)), "attn_bwd_strided")
    return dq, dk, dv


def attn_bwd_varlen(q, k, v, o, lse, dout, cu_seqlens_q, cu_seqlens_k, max_seqlen_q, max_seqlen_k, dq=None, dk=None,
                    dv=None, workspace=None, scale=None, causal=False, g_dtype=None, stream=None):
    """The backward of :func:`attn_fwd_varlen`: ``q``, ``o``, ``dout`` [total_q, H, d], ``k``, ``v``
    [total_k, H, d] (bf16, row and head strides free, last dimension contiguous), ``lse``
    [H, total_q].  Returns ``(dq, dk, dv)``."""
    return _bwd_varlen(q, k, v, o, lse, dout, cu_seqlens_q, cu_seqlens_k, max_seqlen_q, max_seqlen_k, dq, dk, dv,
                       workspace, scale, causal, g_dtype, stream, False)


def attn_bwd_varlen_ds_workspace_bytes(B, H, max_seqlen_q, max_seqlen_k):
    """Bytes of the workspace :func:`attn_bwd_varlen_ds` needs (0 if too many tiles)."""
    return int(lib().attn_bwd_varlen_ds_workspace_bytes(B, H, int(max_seqlen_q), int(max_seqlen_k)))


def attn_bwd_varlen_ds(q, k, v, o, lse, dout, cu_seqlens_q, cu_seqlens_k, max_seqlen_q, max_seqlen_k, dq=None,
                       dk=None, dv=None, workspace=None, scale=None, causal=False, g_dtype=None, stream=None):
    """:func:`attn_bwd_varlen` with the dS tiles kept in the workspace (a uint8 tensor of
    :func:`attn_bwd_varlen_ds_workspace_bytes` bytes), as :func:`attn_bwd_ds` for fixed lengths."""
    return _bwd_varlen(q, k, v, o, lse, dout, cu_seqlens_q, cu_seqlens_k, max_seqlen_q, max_seqlen_k, dq, dk, dv,
                       workspace, scale, causal, g_dtype, stream, True)


def _bwd_varlen(q, k, v, o, lse, dout, cu_seqlens_q, cu_seqlens_k, max_seqlen_q, max_seqlen_k, dq, dk, dv,
                workspace, scale, causal, g_dtype, stream, ds):
    import torch
    if q.dim() != 3 or k.dim() != 3 or v.shape != k.shape or o.shape != q.shape or dout.shape != q.shape:
        raise ValueError("expected q, o, dout [total_q, H, d] and k, v [total_k, H, d]")
    total_q, H, d = (int(x) for x in q.shape)
    total_k = int(k.shape[0])
    if (int(k.shape[1]), int(k.shape[2])) != (H, d):
        raise ValueError("k and v must have q's H and d")
    for t in (q, k, v, o, dout):
        if t.dtype != torch.bfloat16 or t.stride(-1) != 1:
            raise ValueError("q, k, v, o, dout must be bf16 with a contiguous last dimension")
    for c in (cu_seqlens_q, cu_seqlens_k):
        if c.dtype != torch.int32 or c.dim() != 1 or not c.is_contiguous() or not c.is_cuda:
            raise ValueError("cu_seqlens must be contiguous int32 cuda tensors")
    if cu_seqlens_k.shape != cu_seqlens_q.shape:
        raise ValueError("cu_seqlens_q and cu_seqlens_k must both have B + 1 entries")
    if lse.dtype != torch.float32 or not lse.is_contiguous() or tuple(lse.shape) != (H, total_q):
        raise ValueError("lse must be contiguous float32 [H, total_q]")
    B = int(cu_seqlens_q.shape[0]) - 1
    gd = g_dtype or (dq.dtype if dq is not None else torch.bfloat16)
    dq = dq if dq is not None else torch.empty_like(q, dtype=gd)
    dk = dk if dk is not None else torch.empty_like(k, dtype=gd)
    dv = dv if dv is not None else torch.empty_like(v, dtype=gd)
    _grads(dq, dk, dv, q.shape, k.shape, strided=True)
    mq = min(int(max_seqlen_q), total_q)
    if ds:
        nbytes = attn_bwd_varlen_ds_workspace_bytes(B, H, int(max_seqlen_q), int(max_seqlen_k))
        if nbytes == 0:
            raise ValueError("too many dS tiles for this batch: use attn_bwd_varlen")
    else:
        nbytes = attn_bwd_workspace_bytes(B, H, mq)
    workspace = _workspace(workspace, nbytes, q.device, "attn_bwd_varlen_ds" if ds else "attn_bwd_varlen")
    strides = (ctypes.c_longlong * 16)(*[int(x) for t in (q, k, v, o, dout, dq, dk, dv) for x in t.stride()[:2]])
    gcode = ATTN_FP32 if dq.dtype == torch.float32 else ATTN_BF16
    s = float(scale) if scale is not None else 1.0 / math.sqrt(d)
    fn, name = (lib().attn_bwd_varlen_ds, "attn_bwd_varlen_ds") if ds else (lib().attn_bwd_varlen, "attn_bwd_varlen")
    _check(fn(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dout), _ptr(lse), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(workspace),
              _ptr(cu_seqlens_q), _ptr(cu_seqlens_k), B, H, total_q, total_k, int(max_seqlen_q), int(max_seqlen_k), d,
              ctypes.cast(strides, ctypes.c_void_p), s, int(bool(causal)), gcode, _stream_ptr(stream)), name)
    return dq, dk, dv


def attn_fwd_noalloc(q, k, v, o, lse=None, scale=None, causal=False, stream=None):
    """``attn_fwd`` through the entry point that allocates no device memory (its scratch is a
    static device array of the library).  ``o`` (bf16 or f32) must be given; ``lse`` may be
    None.  The first call on a device does a one-time set-up."""
    import torch
    B, H, N, d = _dims(q)
    _out(o, q.shape, (torch.bfloat16, torch.float32), "o")
    if lse is not None:
        _out(lse, (B, H, N), (torch.float32,), "lse")
    od = ATTN_FP32 if o.dtype == torch.float32 else ATTN_BF16
    s = float(scale) if scale is not None else 1.0 / math.sqrt(d)
    _check(lib().attn_fwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, N, d, s,
                                  int(bool(causal)), ATTN_BF16, od, _stream_ptr(stream)), "attn_fwd_noalloc")
    return o, lse


def attn_noalloc_status(stream=None) -> int:
    """Status word of ``attn_fwd_noalloc`` on the current device (synchronises ``stream``, then
    clears the word); allocates nothing."""
    return int(lib().attn_noalloc_status(_stream_ptr(stream)))


def attn_noalloc_selftest_wait_timeout(stream=None) -> None:
    """The bounded-wait self-test aimed at the status word of ``attn_fwd_noalloc``."""
    _check(lib().attn_noalloc_selftest_wait_timeout(_stream_ptr(stream)), "attn_noalloc_selftest_wait_timeout")


def attn_hadamard_quant(x, signs=None, x8=None, scales=None, stream=None):
    """Per-block E4M3 quantisation of a [B, H, N, d] bf16 tensor, after H_d D when ``signs``.

    ``signs``: int8 cuda tensor of d entries +-1, or None.  Returns ``(x8 uint8, scales f32)``.
    """
    import torch
    B, H, N, d = _dims(x)
    if x.dtype != torch.bfloat16 or not x.is_contiguous():
        raise ValueError("x must be a contiguous bf16 tensor")
    nb = (N + 127) // 128
    if x8 is None:
        x8 = torch.empty(x.shape, dtype=torch.uint8, device=x.device)
    if scales is None:
        scales = torch.empty((B, H, nb), dtype=torch.float32, device=x.device)
    _out(x8, x.shape, (torch.uint8,), "x8")
    _out(scales, (B, H, nb), (torch.float32,), "scales")
    _check(lib().attn_hadamard_quant(_ptr(x), _ptr(x8), _ptr(scales), _ptr(_signs(signs, d)), B, H, N, d,
                                     _stream_ptr(stream)), "attn_hadamard_quant")
    return x8, scales


def attn_hadamard_quant_qkv(q, k, v, signs, outs=None, stream=None):
    """One launch: Q and K through H_d D then E4M3, V straight to E4M3 (per-block scales).

    Returns ``(q8, k8, v8, q_scale, k_scale, v_scale)``; ``outs`` may supply them.
    """
    import torch
    B, H, N, d = _dims(q)
    for t in (q, k, v):
        if t.dtype != torch.bfloat16 or not t.is_contiguous() or t.shape != q.shape:
            raise ValueError("q, k, v must be contiguous bf16 tensors of one shape")
    nb = (N + 127) // 128
    if outs is None:
        outs = tuple(torch.empty(q.shape, dtype=torch.uint8, device=q.device) for _ in range(3)) + \
            tuple(torch.empty((B, H, nb), dtype=torch.float32, device=q.device) for _ in range(3))
    _outs_qkv(outs, q.shape, q.shape, (B, H, nb), (B, H, nb))
    q8, k8, v8, qs, ks, vs = outs
    _check(lib().attn_hadamard_quant_qkv(_ptr(q), _ptr(k), _ptr(v), _ptr(q8), _ptr(k8), _ptr(v8), _ptr(qs), _ptr(ks),
                                         _ptr(vs), _ptr(_signs(signs, d)), B, H, N, d, _stream_ptr(stream)),
           "attn_hadamard_quant_qkv")
    return outs


def attn_hadamard_quant_qkv_strided(q, k, v, signs, outs=None, stream=None):
    """attn_hadamard_quant_qkv on logical [B, H, N, d] bf16 views with any strides whose last one
    is 1 (e.g. the head views of one fused [B, N, 3, H, d] projection), without a copy.  The
    outputs are contiguous, bit-identical to attn_hadamard_quant_qkv on contiguous copies.
    Returns ``(q8, k8, v8, q_scale, k_scale, v_scale)``; ``outs`` may supply them."""
    import torch
    B, H, N, d = _dims(q)
    for t in (q, k, v):
        if t.dtype != torch.bfloat16 or t.stride(-1) != 1 or t.shape != q.shape:
            raise ValueError("q, k, v must be bf16 of one shape with a contiguous last dimension")
    nb = (N + 127) // 128
    if outs is None:
        outs = tuple(torch.empty(q.shape, dtype=torch.uint8, device=q.device) for _ in range(3)) + \
            tuple(torch.empty((B, H, nb), dtype=torch.float32, device=q.device) for _ in range(3))
    _outs_qkv(outs, q.shape, q.shape, (B, H, nb), (B, H, nb))
    q8, k8, v8, qs, ks, vs = outs
    strides = (ctypes.c_longlong * 9)(*[int(x) for t in (q, k, v) for x in t.stride()[:3]])
    _check(lib().attn_hadamard_quant_qkv_strided(_ptr(q), _ptr(k), _ptr(v), _ptr(q8), _ptr(k8), _ptr(v8), _ptr(qs),
                                                 _ptr(ks), _ptr(vs), _ptr(_signs(signs, d)), B, H, N, d,
                                                 ctypes.cast(strides, ctypes.c_void_p), _stream_ptr(stream)),
           "attn_hadamard_quant_qkv_strided")
    return outs


def attn_rope_hadamard_quant_qkv(q, k, v, signs, cos, sin, outs=None, stream=None):
    """attn_hadamard_quant_qkv with Q and K first rotated by the rotary tables ``cos``, ``sin``
    (frequency-major [d/2, n_pos] float32 cuda tensors, n_pos >= N; row n of each sequence uses
    column n).  Returns ``(q8, k8, v8, q_scale, k_scale, v_scale)``."""
    import torch
    B, H, N, d = _dims(q)
    for t in (q, k, v):
        if t.dtype != torch.bfloat16 or not t.is_contiguous() or t.shape != q.shape:
            raise ValueError("q, k, v must be contiguous bf16 tensors of one shape")
    for t in (cos, sin):
        if t.dtype != torch.float32 or not t.is_contiguous() or t.dim() != 2 or t.shape[0] != d // 2:
            raise ValueError("cos and sin must be contiguous float32 [d/2, n_pos]")
    if cos.shape != sin.shape:
        raise ValueError("cos and sin must have one shape")
    nb = (N + 127) // 128
    if outs is None:
        outs = tuple(torch.empty(q.shape, dtype=torch.uint8, device=q.device) for _ in range(3)) + \
            tuple(torch.empty((B, H, nb), dtype=torch.float32, device=q.device) for _ in range(3))
    _outs_qkv(outs, q.shape, q.shape, (B, H, nb), (B, H, nb))
    q8, k8, v8, qs, ks, vs = outs
    _check(lib().attn_rope_hadamard_quant_qkv(_ptr(q), _ptr(k), _ptr(v), _ptr(q8), _ptr(k8), _ptr(v8), _ptr(qs),
                                              _ptr(ks), _ptr(vs), _ptr(_signs(signs, d)), _ptr(cos), _ptr(sin),
                                              int(cos.shape[1]), B, H, N, d, _stream_ptr(stream)),
           "attn_rope_hadamard_quant_qkv")
    return outs


def attn_fwd_fp8(q8, k8, v8, q_scale, k_scale, v_scale, o=None, lse=None, scale=None, causal=False,
                 o_dtype=None, stream=None):
    """Attention on E4M3 inputs with per-block scales (from ``attn_hadamard_quant``)."""
    import torch
    B, H, N, d = _dims(q8)
    nb = (N + 127) // 128
    for t, name in ((q8, "q8"), (k8, "k8"), (v8, "v8")):
        _out(t, (B, H, N, d), (torch.uint8,), name)
    for t, name in ((q_scale, "q_scale"), (k_scale, "k_scale"), (v_scale, "v_scale")):
        _out(t, (B, H, nb), (torch.float32,), name)
    if o is None:
        o = torch.empty((B, H, N, d), dtype=o_dtype or torch.bfloat16, device=q8.device)
    if lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=q8.device)
    _out(o, (B, H, N, d), (torch.bfloat16, torch.float32), "o")
    _out(lse, (B, H, N), (torch.float32,), "lse")
    od = ATTN_FP32 if o.dtype == torch.float32 else ATTN_BF16
    s = float(scale) if scale is not None else 1.0 / math.sqrt(d)
    _check(lib().attn_fwd_fp8(_ptr(q8), _ptr(k8), _ptr(v8), _ptr(q_scale), _ptr(k_scale), _ptr(v_scale),
                              _ptr(o), _ptr(lse), B, H, N, d, s, int(bool(causal)), od, _stream_ptr(stream)),
           "attn_fwd_fp8")
    return o, lse


def attn_fwd_fp8_qk(q8, k8, v8, q_scale, k_scale, v_scale, o=None, lse=None, scale=None, causal=False,
                    o_dtype=None, stream=None):
    """attn_fwd_fp8 with keys/values [B, H, Nk, d] of another length than the queries
    [B, H, Nq, d] (bottom-right causal alignment, as attn_fwd_qk)."""
    import torch
    B, H, Nq, d = _dims(q8)
    Nk = int(k8.shape[2])
    if tuple(k8.shape) != (B, H, Nk, d) or v8.shape != k8.shape:
        raise ValueError("k8 and v8 must be [B, H, Nk, d] with q8's B, H, d")
    for t, name in ((q8, "q8"), (k8, "k8"), (v8, "v8")):
        _out(t, t.shape, (torch.uint8,), name)
    _out(q_scale, (B, H, (Nq + 127) // 128), (torch.float32,), "q_scale")
    for t, name in ((k_scale, "k_scale"), (v_scale, "v_scale")):
        _out(t, (B, H, (Nk + 127) // 128), (torch.float32,), name)
    if o is None:
        o = torch.empty((B, H, Nq, d), dtype=o_dtype or torch.bfloat16, device=q8.device)
    if lse is None:
        lse = torch.empty((B, H, Nq), dtype=torch.float32, device=q8.device)
    _out(o, (B, H, Nq, d), (torch.bfloat16, torch.float32), "o")
    _out(lse, (B, H, Nq), (torch.float32,), "lse")
    od = ATTN_FP32 if o.dtype == torch.float32 else ATTN_BF16
    s = float(scale) if scale is not None else 1.0 / math.sqrt(d)
    _check(lib().attn_fwd_fp8_qk(_ptr(q8), _ptr(k8), _ptr(v8), _ptr(q_scale), _ptr(k_scale), _ptr(v_scale),
                                 _ptr(o), _ptr(lse), B, H, Nq, Nk, d, s, int(bool(causal)), od, _stream_ptr(stream)),
           "attn_fwd_fp8_qk")
    return o, lse


def attn_fwd_fp8_strided(q8, k8, v8, q_scale, k_scale, v_scale, o=None, lse=None, scale=None, causal=False,
                        o_dtype=None, stream=None):
    """attn_fwd_fp8_qk on logical [B, H, N, d] uint8 (E4M3) views and an output ``o`` with any
    strides whose last one is 1 (E4M3 strides multiples of 16, O strides multiples of 8), e.g. O
    written straight into a sequence-major [B, N, H, d] buffer.  The scales stay contiguous
    [B, H, ceil(N/128)].  ``o`` defaults to a contiguous tensor.  Returns ``(o, lse)``."""
    import torch
    B, H, Nq, d = _dims(q8)
    Nk = int(k8.shape[2])
    if tuple(k8.shape) != (B, H, Nk, d) or v8.shape != k8.shape:
        raise ValueError("k8 and v8 must be [B, H, Nk, d] with q8's B, H, d")
    for t in (q8, k8, v8):
        if t.dtype != torch.uint8 or t.stride(-1) != 1:
            raise ValueError("q8, k8, v8 must be uint8 with a contiguous last dimension")
    _out(q_scale, (B, H, (Nq + 127) // 128), (torch.float32,), "q_scale")
    for t, name in ((k_scale, "k_scale"), (v_scale, "v_scale")):
        _out(t, (B, H, (Nk + 127) // 128), (torch.float32,), name)
    if o is None:
        o = torch.empty((B, H, Nq, d), dtype=o_dtype or torch.bfloat16, device=q8.device)
    _out(o, (B, H, Nq, d), (torch.bfloat16, torch.float32), "o", strided=True)
    if lse is None:
        lse = torch.empty((B, H, Nq), dtype=torch.float32, device=q8.device)
    _out(lse, (B, H, Nq), (torch.float32,), "lse")
    strides = (ctypes.c_longlong * 12)(*[int(x) for t in (q8, k8, v8, o) for x in t.stride()[:3]])
    od = ATTN_FP32 if o.dtype == torch.float32 else ATTN_BF16
    s = float(scale) if scale is not None else 1.0 / math.sqrt(d)
    _check(lib().attn_fwd_fp8_strided(_ptr(q8), _ptr(k8), _ptr(v8), _ptr(q_scale), _ptr(k_scale), _ptr(v_scale),
                                      _ptr(o), _ptr(lse), B, H, Nq, Nk, d, ctypes.cast(strides, ctypes.c_void_p), s,
                                      int(bool(causal)), od, _stream_ptr(stream)), "attn_fwd_fp8_strided")
    return o, lse


def attn_fwd_schedule(B, H, Nq, Nk, d, causal=False, fp8=False, num_ctas=148):
    """The forward kernels' work lists for a fixed-length launch (host only, no CUDA call).

    Returns ``None`` if the launch keeps the kernels' round-robin order, else a list with, for
    each CTA, the unit ids it computes in order (unit u: batch*head ``u % (B*H)``, round
    ``u // (B*H)``, see ``attn_fwd_schedule`` in ``include/attn.h``)."""
    need = ctypes.c_longlong(0)
    dt = ATTN_E4M3 if fp8 else ATTN_BF16
    _check(lib().attn_fwd_schedule(B, H, Nq, Nk, d, int(bool(causal)), dt, num_ctas, None, 0, ctypes.byref(need)),
           "attn_fwd_schedule")
    if need.value == 0:
        return None
    buf = (ctypes.c_int * need.value)()
    _check(lib().attn_fwd_schedule(B, H, Nq, Nk, d, int(bool(causal)), dt, num_ctas, ctypes.cast(buf, ctypes.c_void_p),
                                   need.value, ctypes.byref(need)), "attn_fwd_schedule")
    t = list(buf)
    grid = len(t) - 1 - _units(B, H, Nq, d)  # the table is [grid + 1 offsets][units]
    return [t[grid + 1 + t[b]: grid + 1 + t[b + 1]] for b in range(grid)]


def _units(B, H, Nq, d):
    tiles = 1 if d == 256 else 2
    return B * H * (((Nq + 127) // 128 + tiles - 1) // tiles)


def _check_cu(cu_seqlens_q, cu_seqlens_k):
    import torch
    for c in (cu_seqlens_q, cu_seqlens_k):
        if c.dtype != torch.int32 or c.dim() != 1 or not c.is_contiguous() or not c.is_cuda:
            raise ValueError("cu_seqlens must be contiguous int32 cuda tensors")
    if cu_seqlens_k.shape != cu_seqlens_q.shape:
        raise ValueError("cu_seqlens_q and cu_seqlens_k must both have B + 1 entries")
    return int(cu_seqlens_q.shape[0]) - 1


def attn_hadamard_quant_qkv_varlen(q, k, v, signs, cu_seqlens_q, cu_seqlens_k, max_seqlen_q, max_seqlen_k,
                                   outs=None, stream=None):
    """Packed batch: ``q`` [total_q, H, d], ``k``, ``v`` [total_k, H, d] bf16 (row and head strides
    free, last dimension contiguous) quantised per 128-row block of each sequence.  Returns
    ``(q8, k8, v8, q_scale, k_scale, v_scale)``: codes [total, H, d] uint8 and scales
    [B, H, ceil(max_seqlen / 128)] float32."""
    import torch
    if q.dim() != 3 or k.dim() != 3 or v.shape != k.shape:
        raise ValueError("q must be [total_q, H, d], k and v [total_k, H, d]")
    total_q, H, d = (int(x) for x in q.shape)
    total_k = int(k.shape[0])
    if (int(k.shape[1]), int(k.shape[2])) != (H, d):
        raise ValueError("k and v must have q's H and d")
    for t in (q, k, v):
        if t.dtype != torch.bfloat16 or t.stride(-1) != 1:
            raise ValueError("q, k, v must be bf16 with a contiguous last dimension")
    B = _check_cu(cu_seqlens_q, cu_seqlens_k)
    nbq, nbk = (int(max_seqlen_q) + 127) // 128, (int(max_seqlen_k) + 127) // 128
    if outs is None:
        dev = q.device
        outs = (torch.empty((total_q, H, d), dtype=torch.uint8, device=dev),
                torch.empty((total_k, H, d), dtype=torch.uint8, device=dev),
                torch.empty((total_k, H, d), dtype=torch.uint8, device=dev),
                torch.empty((B, H, nbq), dtype=torch.float32, device=dev),
                torch.empty((B, H, nbk), dtype=torch.float32, device=dev),
                torch.empty((B, H, nbk), dtype=torch.float32, device=dev))
    _outs_qkv(outs, (total_q, H, d), (total_k, H, d), (B, H, nbq), (B, H, nbk))
    q8, k8, v8, qs, ks, vs = outs
    strides = (ctypes.c_longlong * 6)(*[int(x) for t in (q, k, v) for x in t.stride()[:2]])
    _check(lib().attn_hadamard_quant_qkv_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(q8), _ptr(k8), _ptr(v8), _ptr(qs),
                                                _ptr(ks), _ptr(vs), _ptr(_signs(signs, d)), _ptr(cu_seqlens_q),
                                                _ptr(cu_seqlens_k), B, H, total_q, total_k, int(max_seqlen_q),
                                                int(max_seqlen_k), d, ctypes.cast(strides, ctypes.c_void_p),
                                                _stream_ptr(stream)), "attn_hadamard_quant_qkv_varlen")
    return outs


def attn_fwd_fp8_varlen(q8, k8, v8, q_scale, k_scale, v_scale, cu_seqlens_q, cu_seqlens_k, max_seqlen_q,
                        max_seqlen_k, o=None, lse=None, scale=None, causal=False, o_dtype=None, stream=None):
    """The E4M3 forward over a packed batch (codes and scales from
    :func:`attn_hadamard_quant_qkv_varlen`, with the same offsets and longest lengths).
    Returns ``(o [total_q, H, d], lse [H, total_q])``."""
    import torch
    total_q, H, d = (int(x) for x in q8.shape)
    total_k = int(k8.shape[0])
    for t in (q8, k8, v8):
        if t.dtype != torch.uint8 or not t.is_contiguous() or t.dim() != 3:
            raise ValueError("q8, k8, v8 must be contiguous uint8 [total, H, d]")
    B = _check_cu(cu_seqlens_q, cu_seqlens_k)
    _out(q_scale, (B, H, (int(max_seqlen_q) + 127) // 128), (torch.float32,), "q_scale")
    for t, name in ((k_scale, "k_scale"), (v_scale, "v_scale")):
        _out(t, (B, H, (int(max_seqlen_k) + 127) // 128), (torch.float32,), name)
    if o is None:
        o = torch.empty((total_q, H, d), dtype=o_dtype or torch.bfloat16, device=q8.device)
    _out(o, (total_q, H, d), (torch.bfloat16, torch.float32), "o")
    if lse is None:
        lse = torch.empty((H, total_q), dtype=torch.float32, device=q8.device)
    _out(lse, (H, total_q), (torch.float32,), "lse")
    od = ATTN_FP32 if o.dtype == torch.float32 else ATTN_BF16
    s = float(scale) if scale is not None else 1.0 / math.sqrt(d)
    _check(lib().attn_fwd_fp8_varlen(_ptr(q8), _ptr(k8), _ptr(v8), _ptr(q_scale), _ptr(k_scale), _ptr(v_scale),
                                     _ptr(o), _ptr(lse), _ptr(cu_seqlens_q), _ptr(cu_seqlens_k), B, H, total_q,
                                     total_k, int(max_seqlen_q), int(max_seqlen_k), d, s, int(bool(causal)), od,
                                     _stream_ptr(stream)), "attn_fwd_fp8_varlen")
    return o, lse


def attn_merge_partials(o_acc, lse_acc, o_part, lse_part, stream=None):
    """In place: (o_acc float32 [..., N, d], lse_acc float32 [..., N]) <- the attention result over
    the union of their keys and those of (o_part [..., N, d] bf16 or float32, lse_part)."""
    import torch
    if o_acc.dtype != torch.float32 or lse_acc.dtype != torch.float32 or lse_part.dtype != torch.float32:
        raise ValueError("o_acc, lse_acc and lse_part must be float32")
    if o_part.dtype not in (torch.bfloat16, torch.float32) or o_part.shape != o_acc.shape:
        raise ValueError("o_part must be bf16 or float32 with o_acc's shape")
    if lse_acc.shape != o_acc.shape[:-1] or lse_part.shape != lse_acc.shape:
        raise ValueError("lse_acc and lse_part must be o_acc's shape without its last dimension")
    for t in (o_acc, lse_acc, o_part, lse_part):
        if not t.is_contiguous():
            raise ValueError("all tensors must be contiguous")
    d = int(o_acc.shape[-1])
    rows = int(lse_acc.numel())
    pd = ATTN_FP32 if o_part.dtype == torch.float32 else ATTN_BF16
    _check(lib().attn_merge_partials(_ptr(o_acc), _ptr(lse_acc), _ptr(o_part), _ptr(lse_part), rows, d, pd,
                                     _stream_ptr(stream)), "attn_merge_partials")
    return o_acc, lse_acc


def attn_selftest_wait_timeout(stream=None) -> None:
    """Launches the bounded-wait diagnostic: a wait that nothing satisfies gives up after its limit;
    the next :func:`attn_device_status` returns ATTN_ERR_TIMEOUT."""
    _check(lib().attn_selftest_wait_timeout(_stream_ptr(stream)), "attn_selftest_wait_timeout")


def attn_device_status(stream=None) -> int:
    """Synchronises the stream; returns and clears the device status word (0 = ATTN_OK)."""
    return int(lib().attn_device_status(_stream_ptr(stream)))
