"""The Python binding refuses buffers the kernels would read or write out of bounds.

The C entry points take device pointers and sizes, not tensor shapes, so a caller's output of
the wrong shape or dtype, a scale array that is too short, or a tensor in host memory would be
read or written past its end on the GPU.  The binding checks every caller-supplied buffer and
raises ValueError before any launch: the launch counter does not move and the device status
stays ATTN_OK."""

import pytest
import torch

import exact_attention_100_b200 as ea
from exact_attention_100_b200 import build as ea_build
from exact_attention_100_b200.inputs import hadamard_signs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    ea_build.build()
    ea.lib()


def _qkv(B=1, H=2, N=300, d=64, seed=0):
    g = torch.Generator(device="cuda").manual_seed(seed)
    return [torch.randn(B, H, N, d, device="cuda", generator=g).to(torch.bfloat16) for _ in range(3)]


def _refused(fn):
    torch.cuda.synchronize()
    before = ea.attn_num_kernel_launches()
    with pytest.raises(ValueError):
        fn()
    assert ea.attn_num_kernel_launches() == before
    torch.cuda.synchronize()
    assert ea.attn_device_status() == ea.ATTN_OK


def test_forward_outputs_and_inputs():
    q, k, v = _qkv()
    _refused(lambda: ea.attn_fwd(q, k, v, o=torch.empty(q.shape, dtype=torch.uint8, device="cuda")))
    _refused(lambda: ea.attn_fwd(q, k, v, o=torch.empty(1, 2, 299, 64, dtype=torch.bfloat16, device="cuda")))
    _refused(lambda: ea.attn_fwd(q, k, v, lse=torch.empty(1, 2, 300, dtype=torch.float16, device="cuda")))
    _refused(lambda: ea.attn_fwd(q, k, v, o=torch.empty(q.shape, dtype=torch.bfloat16)))  # host memory
    _refused(lambda: ea.attn_fwd(q.cpu(), k, v))
    _refused(lambda: ea.attn_fwd_noalloc(q, k, v, torch.empty(1, 2, 300, 32, dtype=torch.float32, device="cuda")))


def test_backward_gradients():
    q, k, v = _qkv()
    o, lse = ea.attn_fwd(q, k, v)
    do = torch.ones_like(q)
    f32 = lambda *s: torch.empty(*s, dtype=torch.float32, device="cuda")
    _refused(lambda: ea.attn_bwd(q, k, v, o, lse, do, dq=f32(q.shape), dk=torch.empty_like(q), dv=f32(q.shape)))
    _refused(lambda: ea.attn_bwd(q, k, v, o, lse, do, dq=f32(1, 2, 300, 32)))
    _refused(lambda: ea.attn_bwd_ds(q, k, v, o, lse[:, :, :200].contiguous(), do))


def test_fp8_scales_and_pre_kernel_outputs():
    q, k, v = _qkv(N=384)
    signs = torch.from_numpy(hadamard_signs(64)).cuda()
    q8, k8, v8, qs, ks, vs = ea.attn_hadamard_quant_qkv(q, k, v, signs)
    _refused(lambda: ea.attn_fwd_fp8(q8, k8, v8, qs, ks[:, :, :2].contiguous(), vs))
    _refused(lambda: ea.attn_fwd_fp8(q8, k8, v8, qs, ks, vs, o=torch.empty(1, 2, 384, 64, dtype=torch.float16,
                                                                            device="cuda")))
    bad_outs = (q8, k8, v8, qs, ks, vs[:, :1].contiguous())
    _refused(lambda: ea.attn_hadamard_quant_qkv(q, k, v, signs, outs=bad_outs))
    _refused(lambda: ea.attn_hadamard_quant_qkv(q, k, v, signs, outs=(q8, k8, v8, qs, ks)))
    _refused(lambda: ea.attn_hadamard_quant_qkv(q, k, v, signs[:32].contiguous()))  # d = 64 signs read
    _refused(lambda: ea.attn_hadamard_quant(q.to(torch.float16), signs))
