"""GPU parity of the Hadamard + per-block E4M3 pre-kernel against the oracle: codes and scales
must be bit-identical (the quantisation decision is taken in float32 on both sides)."""

import numpy as np
import pytest

torch = pytest.importorskip("torch")

import exact_attention_100_b200 as ea
from exact_attention_100_b200 import build as ea_build
from exact_attention_100_b200.inputs import hadamard_signs, normal_qkv, round_to_bf16
from oracle import hadamard_quant_ref

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    ea_build.build()
    ea.lib()


def _run(x_np, signs_np):
    x = torch.from_numpy(x_np).to(torch.bfloat16).cuda()
    s = torch.from_numpy(signs_np).cuda() if signs_np is not None else None
    x8, sc = ea.attn_hadamard_quant(x, s)
    torch.cuda.synchronize()
    return x8.cpu().numpy(), sc.cpu().numpy()


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("use_signs", [True, False])
@pytest.mark.parametrize("shape", [(1, 1, 1), (1, 2, 127), (2, 3, 300), (1, 1, 1024)])
def test_bit_exact_against_oracle(d, use_signs, shape):
    B, H, N = shape
    q, _, _ = normal_qkv(B, H, N, d, seed=N + d, outlier_frac=1e-3)
    signs = hadamard_signs(d) if use_signs else None
    codes, scales = _run(q, signs)
    rc, rs = hadamard_quant_ref(q, signs)
    np.testing.assert_array_equal(scales, rs)
    np.testing.assert_array_equal(codes, rc)


def test_fp8_config_q_tensor_bit_exact():
    # B=2 H=16 N=8192 d=128 with 0.1% N(0, 10^2) outliers, seeded signs (the FP8 workload)
    q, _, _ = normal_qkv(2, 16, 8192, 128, seed=0, outlier_frac=1e-3)
    signs = hadamard_signs(128)
    codes, scales = _run(q, signs)
    rc, rs = hadamard_quant_ref(q, signs)
    np.testing.assert_array_equal(scales, rs)
    np.testing.assert_array_equal(codes, rc)


@pytest.mark.parametrize("d", [64, 128, 256])
def test_zero_block_and_large_values(d):
    """A block of zero rows (the signs of D turn them into zeros of both signs, which the
    butterflies must carry as the sequential transform does: E4M3 keeps the sign of zero),
    rows whose butterflies cancel exactly, a block of large values and tiny ones."""
    x = np.zeros((1, 1, 260, d), dtype=np.float32)
    x[0, 0, 128:256] = 3.0e4
    x[0, 0, 256:, ::2] = -1.0e-30
    x[0, 0, 10] = 1.0
    x[0, 0, 11, ::3] = -2.0
    x[0, 0, 12] = np.tile([1.5, -1.5], d // 2)
    x = round_to_bf16(x)
    signs = hadamard_signs(d)
    codes, scales = _run(x, signs)
    rc, rs = hadamard_quant_ref(x.astype(np.float64), signs)
    np.testing.assert_array_equal(scales, rs)
    np.testing.assert_array_equal(codes, rc)


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("n", [1, 300, 1024])
def test_qkv_launch_matches_oracle(d, n):
    q, k, v = normal_qkv(2, 3, n, d, seed=n + 7 * d, outlier_frac=1e-3)
    signs = hadamard_signs(d)
    dev = lambda a: torch.from_numpy(a).to(torch.bfloat16).cuda()
    outs = ea.attn_hadamard_quant_qkv(dev(q), dev(k), dev(v), torch.from_numpy(signs).cuda())
    torch.cuda.synchronize()
    for x, s, c8, sc in ((q, signs, outs[0], outs[3]), (k, signs, outs[1], outs[4]), (v, None, outs[2], outs[5])):
        rc, rs = hadamard_quant_ref(x, s)
        np.testing.assert_array_equal(sc.cpu().numpy(), rs)
        np.testing.assert_array_equal(c8.cpu().numpy(), rc)


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("B,H,n", [(2, 3, 300), (1, 1, 1), (1, 4, 1024)])
def test_strided_qkv_launch_on_a_fused_projection(d, B, H, n):
    """attn_hadamard_quant_qkv_strided on the head views of one fused [B, N, 3, H, d] buffer with
    a padded row (8 spare elements): the codes and scales are the oracle's and bit-identical to
    attn_hadamard_quant_qkv on contiguous copies."""
    q, k, v = normal_qkv(B, H, n, d, seed=n + 11 * d, outlier_frac=1e-3)
    signs = hadamard_signs(d)
    s = torch.from_numpy(signs).cuda()
    fused = torch.zeros((B, n, 3 * H * d + 8), dtype=torch.bfloat16, device="cuda")
    views = []
    for j, x in enumerate((q, k, v)):
        view = fused[:, :, j * H * d:(j + 1) * H * d].view(B, n, H, d).transpose(1, 2)
        view.copy_(torch.from_numpy(x).to(torch.bfloat16).cuda())
        views.append(view)
    assert not views[0].is_contiguous() or (H == 1 and n == 1)
    outs = ea.attn_hadamard_quant_qkv_strided(*views, s)
    ref = ea.attn_hadamard_quant_qkv(*[t.contiguous() for t in views], s)
    torch.cuda.synchronize()
    for a, b in zip(outs, ref):
        assert torch.equal(a, b)
    for x, sg, c8, sc in ((q, signs, outs[0], outs[3]), (k, signs, outs[1], outs[4]), (v, None, outs[2], outs[5])):
        rc, rs = hadamard_quant_ref(x, sg)
        np.testing.assert_array_equal(sc.cpu().numpy(), rs)
        np.testing.assert_array_equal(c8.cpu().numpy(), rc)
