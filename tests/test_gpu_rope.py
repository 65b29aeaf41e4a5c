"""attn_rope_hadamard_quant_qkv: rotary embedding fused into the Hadamard/E4M3 pre-kernel.

Codes and scales must be bit-identical to the oracle's composition
``hadamard_quant_ref(rope_ref(x, cos, sin), signs)`` for Q and K and ``hadamard_quant_ref(v)``
for V (the quantisation decisions are taken in float32 on both sides, rotation included), and
the E4M3 forward on the rotated codes must stay within the FP8 bar of the float64 attention of
the rotated inputs."""

import math

import numpy as np
import pytest
import torch

import exact_attention_100_b200 as ea
from exact_attention_100_b200.inputs import hadamard_signs, normal_qkv, rope_tables
from oracle import attention_ref, hadamard_quant_ref, rope_ref

pytestmark = pytest.mark.gpu


def _run(q, k, v, signs, cos, sin):
    """cos, sin as the oracle takes them ([n_pos, d/2]); the kernel gets them frequency-major."""
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    tq, tk, tv = (dev(a).to(torch.bfloat16) for a in (q, k, v))
    outs = ea.attn_rope_hadamard_quant_qkv(tq, tk, tv, dev(signs), dev(cos.T), dev(sin.T))
    torch.cuda.synchronize()
    assert ea.attn_device_status() == ea.ATTN_OK
    return [t.cpu().numpy() for t in outs]


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("B,H,N", [(1, 1, 1), (1, 2, 127), (2, 3, 300), (1, 1, 513)])
def test_bit_exact_against_oracle(B, H, N, d):
    q, k, v = normal_qkv(B, H, N, d, seed=N + d, outlier_frac=1e-3)
    signs = hadamard_signs(d)
    cos, sin = rope_tables(N + 37, d)  # more table rows than positions
    q8, k8, v8, qs, ks, vs = _run(q, k, v, signs, cos, sin)
    for got, x in (((q8, qs), q), ((k8, ks), k)):
        rc, rs = hadamard_quant_ref(rope_ref(x, cos, sin).astype(np.float64), signs)
        np.testing.assert_array_equal(got[1], rs)
        np.testing.assert_array_equal(got[0], rc)
    rc, rs = hadamard_quant_ref(v, None)
    np.testing.assert_array_equal(vs, rs)
    np.testing.assert_array_equal(v8, rc)


@pytest.mark.parametrize("B,H,N,d", [(1, 4, 8192, 128), (1, 1, 20000, 64)])
def test_bit_exact_where_blocks_of_a_cta_span_positions(B, H, N, d):
    """Sizes at which most CTAs of the d = 64/128 kernel work on blocks of two position blocks,
    so that the staged table slice is replaced mid-range (and the next one prefetched); the
    second has a ragged last block and more table rows than positions."""
    q, k, v = normal_qkv(B, H, N, d, seed=N + d + H, outlier_frac=1e-3)
    signs = hadamard_signs(d)
    cos, sin = rope_tables(N + 5, d)
    q8, k8, v8, qs, ks, vs = _run(q, k, v, signs, cos, sin)
    for got, x in (((q8, qs), q), ((k8, ks), k)):
        rc, rs = hadamard_quant_ref(rope_ref(x, cos, sin).astype(np.float64), signs)
        np.testing.assert_array_equal(got[1], rs)
        np.testing.assert_array_equal(got[0], rc)
    rc, rs = hadamard_quant_ref(v, None)
    np.testing.assert_array_equal(vs, rs)
    np.testing.assert_array_equal(v8, rc)


def test_identity_tables_give_the_unrotated_preprocessing():
    """cos = 1, sin = 0 at every position: the same bits as attn_hadamard_quant_qkv."""
    B, H, N, d = 2, 2, 260, 128
    q, k, v = normal_qkv(B, H, N, d, seed=3)
    signs = hadamard_signs(d)
    one = np.ones((N, d // 2), np.float32)
    got = _run(q, k, v, signs, one, np.zeros_like(one))
    tq, tk, tv = (torch.from_numpy(a).to(torch.bfloat16).cuda() for a in (q, k, v))
    ref = ea.attn_hadamard_quant_qkv(tq, tk, tv, torch.from_numpy(signs).cuda())
    torch.cuda.synchronize()
    for a, b in zip(got, ref):
        np.testing.assert_array_equal(a, b.cpu().numpy())


@pytest.mark.parametrize("causal", [False, True])
def test_fp8_forward_on_rotated_codes(causal):
    """End to end: rotate + transform + quantise, E4M3 forward; RMSE of O against the float64
    attention of the rotated bf16 inputs within the FP8 bar (3e-2)."""
    B, H, N, d = 1, 2, 1024, 128
    q, k, v = normal_qkv(B, H, N, d, seed=8, outlier_frac=1e-3)
    signs = hadamard_signs(d)
    cos, sin = rope_tables(N, d)
    tq, tk, tv = (torch.from_numpy(a).to(torch.bfloat16).cuda() for a in (q, k, v))
    dev_t = lambda a: torch.from_numpy(np.ascontiguousarray(a.T)).cuda()
    q8, k8, v8, qs, ks, vs = ea.attn_rope_hadamard_quant_qkv(tq, tk, tv, torch.from_numpy(signs).cuda(), dev_t(cos),
                                                             dev_t(sin))
    o, _ = ea.attn_fwd_fp8(q8, k8, v8, qs, ks, vs, causal=causal, o_dtype=torch.float32)
    torch.cuda.synchronize()
    assert ea.attn_device_status() == ea.ATTN_OK
    o_ref, _ = attention_ref(rope_ref(q, cos, sin), rope_ref(k, cos, sin), v, 1.0 / math.sqrt(d), causal)
    rmse = float(np.sqrt(np.mean((o.cpu().numpy().astype(np.float64) - o_ref) ** 2)))
    assert rmse <= 3e-2, rmse
