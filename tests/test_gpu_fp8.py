"""GPU checks of the E4M3 forward (attn_fwd_fp8) fed by the Hadamard/E4M3 pre-kernel.

Two references:
* the float64 oracle on the dequantised inputs (codes x block scales): the only difference
  left is the E4M3 rounding of P, so the RMSE must be small (<= 1e-2) and LSE, which is summed
  from float32 p, must match to 1e-3 relative;
* the float64 oracle on the original bf16 inputs (the spec's reference): RMSE <= 3e-2 with and
  without the Hadamard transform on the FP8 workload (B=2 H=16 N=8192 d=128, 0.1% N(0, 10^2)
  outliers), sampled rows.  The transform must lower the error ("FlashAttention-3", section
  "FP8 路径与低精度误差": incoherent processing reduces the FP8 error).
"""

import math

import numpy as np
import pytest

torch = pytest.importorskip("torch")

import exact_attention_100_b200 as ea
from exact_attention_100_b200 import build as ea_build
from exact_attention_100_b200.inputs import hadamard_signs, normal_qkv
from oracle import attention_ref, dequant_ref, hadamard_rotate_ref

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    ea_build.build()
    ea.lib()
    yield
    torch.cuda.synchronize()
    assert ea.attn_device_status() == ea.ATTN_OK


def _quantise(q, k, v, signs):
    dev = lambda a: torch.from_numpy(a).to(torch.bfloat16).cuda()
    s = torch.from_numpy(signs).cuda() if signs is not None else None
    q8, qs = ea.attn_hadamard_quant(dev(q), s)
    k8, ks = ea.attn_hadamard_quant(dev(k), s)
    v8, vs = ea.attn_hadamard_quant(dev(v), None)
    return q8, qs, k8, ks, v8, vs


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("n", [1, 127, 300, 1024])
@pytest.mark.parametrize("use_signs", [True, False])
@pytest.mark.parametrize("d", [64, 128, 256])
def test_against_oracle_on_dequantised_inputs(causal, n, use_signs, d):
    q, k, v = normal_qkv(1, 2, n, d, seed=n + d, outlier_frac=1e-3)
    signs = hadamard_signs(d) if use_signs else None
    q8, qs, k8, ks, v8, vs = _quantise(q, k, v, signs)
    o, lse = ea.attn_fwd_fp8(q8, k8, v8, qs, ks, vs, causal=causal, o_dtype=torch.float32)
    torch.cuda.synchronize()
    qd = dequant_ref(q8.cpu().numpy(), qs.cpu().numpy())
    kd = dequant_ref(k8.cpu().numpy(), ks.cpu().numpy())
    vd = dequant_ref(v8.cpu().numpy(), vs.cpu().numpy())
    o_ref, lse_ref = attention_ref(qd, kd, vd, 1 / math.sqrt(d), causal)
    og = o.cpu().numpy().astype(np.float64)
    assert np.isfinite(og).all()
    rmse = float(np.sqrt(np.mean((og - o_ref) ** 2)))
    assert rmse <= 1e-2, rmse
    # element bound: E4M3 keeps 3 fraction bits, so each P entry carries a relative rounding of
    # at most 2^-4 (normal range), i.e. |O_kernel - O| <= 2^-4 max|v| (+ the subnormal floor)
    assert np.abs(og - o_ref).max() <= (2.0 ** -4 + 1e-2) * np.abs(vd).max()
    lrel = np.abs(lse.cpu().numpy() - lse_ref) / np.abs(lse_ref)
    assert lrel.max() <= 1e-3, lrel.max()


@pytest.mark.parametrize("B,H,N,d", [(2, 16, 8192, 128), (2, 8, 8192, 256), (2, 32, 8192, 64)])
def test_fp8_workload_rmse_with_and_without_hadamard(B, H, N, d):
    """The FP8 workload (d = 128, the configuration the 3e-2 bar is set on, with and without the
    transform) and the same token count at d = 256 and d = 64 (the sweep's H = 2048 / d).  At
    the other head dims the bar holds on the transformed path; without the transform the error
    of quantising the outlier inputs alone is already about 2.3e-2 at d = 256 (the float64 oracle
    on the dequantised inputs, exact P), so there the test only requires that the transform
    lowers the error."""
    q, k, v = normal_qkv(B, H, N, d, seed=0, outlier_frac=1e-3)
    rng = np.random.default_rng(3)
    rows = [(int(rng.integers(B)), int(rng.integers(H)), int(rng.integers(N))) for _ in range(48)]
    rmse = {}
    for use in (True, False):
        q8, qs, k8, ks, v8, vs = _quantise(q, k, v, hadamard_signs(d) if use else None)
        o, _ = ea.attn_fwd_fp8(q8, k8, v8, qs, ks, vs, causal=False, o_dtype=torch.float32)
        torch.cuda.synchronize()
        err = []
        for (b, h, i) in rows:
            o_ref, _ = attention_ref(q[b, h, i:i + 1], k[b, h], v[b, h], 1 / math.sqrt(d), False)
            err.append(o[b, h, i].cpu().numpy().astype(np.float64) - o_ref[0])
        rmse[use] = float(np.sqrt(np.mean(np.square(err))))
    assert rmse[True] <= 3e-2, rmse
    if d == 128:
        assert rmse[False] <= 3e-2, rmse
    assert rmse[True] < rmse[False], rmse


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("nq,nk,d", [(128, 300, 128), (300, 128, 128), (1, 513, 128), (513, 1, 128), (640, 130, 128),
                                     (300, 700, 256), (513, 129, 256), (300, 700, 64), (513, 129, 64)])
def test_fp8_qk_against_oracle_on_dequantised_inputs(nq, nk, d, causal):
    """attn_fwd_fp8_qk: key length different from the query length (bottom-right causal); the
    same bars as the equal-length case on rows that see a key, O = 0 and LSE = -inf on rows
    that see none."""
    from exact_attention_100_b200.inputs import normal_qkv_lengths
    q, k, v = normal_qkv_lengths(1, 2, nq, nk, d, seed=nq + nk)
    q8, qs, k8, ks, v8, vs = _quantise(q, k, v, hadamard_signs(d))
    o, lse = ea.attn_fwd_fp8_qk(q8, k8, v8, qs, ks, vs, causal=causal, o_dtype=torch.float32)
    torch.cuda.synchronize()
    assert ea.attn_device_status() == ea.ATTN_OK
    qd = dequant_ref(q8.cpu().numpy(), qs.cpu().numpy())
    kd = dequant_ref(k8.cpu().numpy(), ks.cpu().numpy())
    vd = dequant_ref(v8.cpu().numpy(), vs.cpu().numpy())
    o_ref, lse_ref = attention_ref(qd, kd, vd, 1 / math.sqrt(d), causal)
    og = o.cpu().numpy().astype(np.float64)
    lg = lse.cpu().numpy().astype(np.float64)
    empty = np.isneginf(lse_ref)
    assert np.array_equal(np.isneginf(lg), empty) and np.all(og[empty] == 0.0)
    err = (og - o_ref)[~empty]
    if err.size:
        assert float(np.sqrt(np.mean(err ** 2))) <= 1e-2
        assert np.abs(err).max() <= (2.0 ** -4 + 1e-2) * np.abs(vd).max()
        assert (np.abs(lg[~empty] - lse_ref[~empty]) / np.abs(lse_ref[~empty])).max() <= 1e-3


def test_fp8_qk_equal_lengths_is_attn_fwd_fp8():
    d = 128
    q, k, v = normal_qkv(1, 2, 333, d, seed=4)
    q8, qs, k8, ks, v8, vs = _quantise(q, k, v, hadamard_signs(d))
    a = ea.attn_fwd_fp8(q8, k8, v8, qs, ks, vs, causal=True)
    b = ea.attn_fwd_fp8_qk(q8, k8, v8, qs, ks, vs, causal=True)
    torch.cuda.synchronize()
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("B,H,nq,nk,d", [(2, 3, 300, 513, 128), (1, 2, 257, 257, 256), (1, 1, 1, 130, 128),
                                          (1, 2, 300, 257, 64)])
def test_fp8_strided_sequence_major_matches_contiguous(B, H, nq, nk, d, causal):
    """attn_fwd_fp8_strided on E4M3 codes held as head views of padded sequence-major buffers,
    writing O into a padded sequence-major [B, Nq, H, d] buffer: O and LSE are bit-identical to
    attn_fwd_fp8_qk on the contiguous codes, the padding is untouched, and O is within the E4M3
    bounds of the oracle on the dequantised inputs."""
    q, _, _ = normal_qkv(B, H, nq, d, seed=nq + d, outlier_frac=1e-3)
    _, k, v = normal_qkv(B, H, nk, d, seed=nk + 3 * d, outlier_frac=1e-3)
    q8, qs, k8, ks, v8, vs = _quantise(q, k, v, hadamard_signs(d))
    ref_o, ref_lse = ea.attn_fwd_fp8_qk(q8, k8, v8, qs, ks, vs, causal=causal, o_dtype=torch.float32)

    def seq_major(x8):
        b, h, n, dd = x8.shape
        buf = torch.zeros((b, n, h, dd + 16), dtype=torch.uint8, device="cuda")
        view = buf[..., :dd].transpose(1, 2)
        view.copy_(x8)
        return view

    o_buf = torch.full((B, nq, H, d + 8), float("nan"), dtype=torch.float32, device="cuda")
    o_view = o_buf[..., :d].transpose(1, 2)
    o, lse = ea.attn_fwd_fp8_strided(seq_major(q8), seq_major(k8), seq_major(v8), qs, ks, vs, o=o_view,
                                     causal=causal)
    torch.cuda.synchronize()
    assert torch.equal(o.contiguous(), ref_o) and torch.equal(lse, ref_lse)
    # the padding columns of the output buffer are not written
    assert torch.isnan(o_buf[..., d:]).all()
    qd = dequant_ref(q8.cpu().numpy(), qs.cpu().numpy())
    kd = dequant_ref(k8.cpu().numpy(), ks.cpu().numpy())
    vd = dequant_ref(v8.cpu().numpy(), vs.cpu().numpy())
    o_ref, lse_ref = attention_ref(qd, kd, vd, 1 / math.sqrt(d), causal)
    og = o.cpu().numpy().astype(np.float64)
    seen = np.isfinite(lse_ref)
    err = og[seen] - o_ref[seen]
    assert float(np.sqrt(np.mean(err ** 2))) <= 1e-2
    assert np.abs(err).max() <= (2.0 ** -4 + 1e-2) * np.abs(vd).max()
