"""GPU parity of the bf16 attention forward (C ABI through the Python binding) against the
float64 oracle, on seeded N(0,1) inputs.

Tolerances (fixed by the spec for bf16 inputs ~ N(0,1)): O max-abs <= 1e-2 and mean-abs <=
1e-3, LSE relative <= 1e-3.  Small problems are compared element by element; the headline
size (B=2 H=16 N=8192 d=128 causal, the configuration the bench times) and the sweep points
are compared on sampled rows that the oracle computes one at a time.
"""

import math

import numpy as np
import pytest

torch = pytest.importorskip("torch")

import exact_attention_100_b200 as ea
from exact_attention_100_b200 import build as ea_build
from gpu_util import assert_within, compare_full, compare_rows, default_scale, device_qkv, sampled_rows

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    ea_build.build()
    ea.lib()
    yield
    torch.cuda.synchronize()
    assert ea.attn_device_status() == ea.ATTN_OK


def test_small_config_fp32_out():
    # B=1 H=1 N=256 d=64, non-causal, scale 1/sqrt(64), seed 0, fp32 O + LSE
    (q, k, v), (qd, kd, vd) = device_qkv(1, 1, 256, 64, seed=0)
    o, lse = ea.attn_fwd(qd, kd, vd, scale=1 / 8.0, causal=False, o_dtype=torch.float32)
    torch.cuda.synchronize()
    assert_within(compare_full(o, lse, q, k, v, 1 / 8.0, False), "config 0")


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("o_dtype", ["bf16", "fp32"])
def test_config_b4_h16_n2048_d128(causal, o_dtype):
    (q, k, v), (qd, kd, vd) = device_qkv(4, 16, 2048, 128, seed=0)
    od = torch.float32 if o_dtype == "fp32" else torch.bfloat16
    o, lse = ea.attn_fwd(qd, kd, vd, scale=default_scale(128), causal=causal, o_dtype=od)
    torch.cuda.synchronize()
    assert_within(compare_full(o, lse, q, k, v, default_scale(128), causal), (causal, o_dtype))


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("n", [1, 7, 127, 128, 129, 255, 256, 257, 300, 513])
def test_ragged_lengths(d, causal, n):
    (q, k, v), (qd, kd, vd) = device_qkv(1, 3, n, d, seed=n + d)
    o, lse = ea.attn_fwd(qd, kd, vd, scale=default_scale(d), causal=causal, o_dtype=torch.float32)
    torch.cuda.synchronize()
    assert_within(compare_full(o, lse, q, k, v, default_scale(d), causal), (d, causal, n))


@pytest.mark.parametrize("d", [64, 256])
@pytest.mark.parametrize("causal", [False, True])
def test_other_head_dims_multi_tile(d, causal):
    (q, k, v), (qd, kd, vd) = device_qkv(2, 4, 1000, d, seed=3)
    o, lse = ea.attn_fwd(qd, kd, vd, scale=default_scale(d), causal=causal)
    torch.cuda.synchronize()
    assert_within(compare_full(o, lse, q, k, v, default_scale(d), causal), (d, causal))


def test_headline_config_sampled_rows():
    # B=2 H=16 N=8192 d=128 causal: the configuration and launch the bench times
    (q, k, v), (qd, kd, vd) = device_qkv(2, 16, 8192, 128, seed=0)
    o, lse = ea.attn_fwd(qd, kd, vd, scale=default_scale(128), causal=True)
    torch.cuda.synchronize()
    assert torch.isfinite(o.float()).all() and torch.isfinite(lse).all()
    rows = sampled_rows(2, 16, 8192, 64, seed=7)
    assert_within(compare_rows(o, lse, q, k, v, default_scale(128), True, rows), "headline")


_SWEEP_CACHE = {}


def _sweep_inputs(d, n):
    """Inputs of one sweep point (B = 16384 / N, H = 2048 / d, seed 1), kept for the next test
    (the causal and non-causal cases of a point share them); one point at a time."""
    key = (d, n)
    if key not in _SWEEP_CACHE:
        _SWEEP_CACHE.clear()
        _SWEEP_CACHE[key] = device_qkv(16384 // n, 2048 // d, n, d, seed=1)
    return _SWEEP_CACHE[key]


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("n", [512, 1024, 2048, 4096, 8192, 16384])
@pytest.mark.parametrize("d", [64, 128, 256])
def test_sweep_points_sampled_rows(d, n, causal):
    """Every point of the head-dim x length sweep the bench times (16384 tokens per
    head-batch), at its full size, on 32 sampled rows that the oracle computes one by one."""
    B, H = 16384 // n, 2048 // d
    (q, k, v), (qd, kd, vd) = _sweep_inputs(d, n)
    o, lse = ea.attn_fwd(qd, kd, vd, scale=default_scale(d), causal=causal)
    torch.cuda.synchronize()
    assert torch.isfinite(o.float()).all() and torch.isfinite(lse).all()
    rows = sampled_rows(B, H, n, 32, seed=d + n)
    assert_within(compare_rows(o, lse, q, k, v, default_scale(d), causal, rows), (d, n, causal))


# ---- properties that hold at any size ----------------------------------------------------

def test_identical_keys_give_prefix_means():
    B, H, N, d = 1, 2, 1200, 128
    (q, k, v), (qd, kd, vd) = device_qkv(B, H, N, d, seed=5)
    kd = kd[:, :, :1].expand(B, H, N, d).contiguous()
    o, lse = ea.attn_fwd(qd, kd, vd, causal=True, o_dtype=torch.float32)
    vv = vd.float()
    want = torch.cumsum(vv, dim=2) / torch.arange(1, N + 1, device=vv.device, dtype=torch.float32)[None, None, :, None]
    assert (o - want).abs().max().item() <= 1e-2


def test_causal_row0_equals_v0_and_dominant_key():
    (q, k, v), (qd, kd, vd) = device_qkv(2, 3, 700, 64, seed=6)
    o, lse = ea.attn_fwd(qd, kd, vd, causal=True, o_dtype=torch.float32)
    assert (o[:, :, 0] - vd[:, :, 0].float()).abs().max().item() <= 1e-5
    # one key dominates every score of a non-causal problem: score 80 against 0.  Every other
    # weight underflows; the dominant weight is 2^(80 log2e - m) with m the once-rounded max,
    # i.e. 1 within ~80 * log2(e) * 2^-24 relative, which bounds the error
    qd2 = torch.zeros_like(qd)
    qd2[..., 0] = 1.0
    kd2 = torch.zeros_like(kd)
    kd2[:, :, 333, 0] = 80.0
    o2, _ = ea.attn_fwd(qd2, kd2, vd, scale=1.0, causal=False, o_dtype=torch.float32)
    tol = 80 * math.log2(math.e) * 2.0 ** -24 * 2 * vd.float().abs().max().item()
    assert (o2 - vd[:, :, 333:334].float()).abs().max().item() <= tol


def test_joint_kv_permutation_invariance():
    (q, k, v), (qd, kd, vd) = device_qkv(1, 4, 1024, 128, seed=8)
    perm = torch.randperm(1024, generator=torch.Generator().manual_seed(0)).cuda()
    o1, l1 = ea.attn_fwd(qd, kd, vd, o_dtype=torch.float32)
    o2, l2 = ea.attn_fwd(qd, kd[:, :, perm].contiguous(), vd[:, :, perm].contiguous(), o_dtype=torch.float32)
    assert (o1 - o2).abs().max().item() <= 2e-3
    assert ((l1 - l2).abs() / l1.abs()).max().item() <= 1e-5


def test_deterministic_and_stream_ordered():
    (q, k, v), (qd, kd, vd) = device_qkv(2, 8, 3000, 128, seed=9)
    o1, l1 = ea.attn_fwd(qd, kd, vd, causal=True)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        o2, l2 = ea.attn_fwd(qd, kd, vd, causal=True, stream=s)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_lse_optional_and_launch_count():
    (q, k, v), (qd, kd, vd) = device_qkv(1, 2, 300, 128, seed=10)
    n0 = ea.attn_num_kernel_launches()
    o1, _ = ea.attn_fwd(qd, kd, vd, want_lse=False)
    o2, _ = ea.attn_fwd(qd, kd, vd)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2)
    assert ea.attn_num_kernel_launches() - n0 == 2
    assert ea.attn_device_status() == ea.ATTN_OK


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("causal", [False, True])
def test_growing_scores_exercise_lazy_rescale(d, causal):
    # key magnitudes ramp up along the sequence, so the running max of late rows climbs by far
    # more than the lazy threshold several times: O must be rescaled in TMEM on the way
    B, H, N = 1, 2, 1100
    (q, k, v), _ = device_qkv(B, H, N, d, seed=11)
    ramp = (1.0 + 6.0 * np.arange(N) / N).astype(np.float32)[None, None, :, None]
    from exact_attention_100_b200.inputs import round_to_bf16
    k = round_to_bf16(k * ramp)
    qd, kd, vd = (torch.from_numpy(a).to(torch.bfloat16).cuda() for a in (q, k, v))
    o, lse = ea.attn_fwd(qd, kd, vd, scale=1.0 / math.sqrt(d), causal=causal, o_dtype=torch.float32)
    torch.cuda.synchronize()
    res = compare_full(o, lse, q, k, v, 1.0 / math.sqrt(d), causal)
    # These scores are far from iid N(0,1): the weights are peaked, so the bf16 rounding of P no
    # longer averages out.  With P = bf16(p) = p (1 + e), |e| <= 2^-8, and l summed from f32 p,
    # |O_kernel - O| <= 2^-8 * sum_j w_j |v_j| <= 2^-8 max|v| (plus ~1e-4 relative from exp2).
    bound = (2.0 ** -8 + 2e-4) * float(np.abs(v).max())
    assert res["finite"] and res["o_max_abs"] <= bound and res["o_mean_abs"] <= 1e-3, (d, causal, res, bound)
    assert res["lse_max_rel"] <= 1e-3, (d, causal, res)
