"""GPU parity of the packed-batch FP8 path.

* attn_hadamard_quant_qkv_varlen: for every sequence, codes and scales bit-identical to the
  oracle's per-block quantisation (hadamard_quant_ref) of that sequence alone, so no block mixes
  two sequences ("Flash Attention V3 解析", section 3.3: FP8 with per-block scales; the blocks are
  the sequence's own 128-row blocks).
* attn_fwd_fp8_varlen: for every sequence, O and LSE bit-identical to attn_fwd_fp8_qk on that
  sequence's codes and scales alone, and within the E4M3 bounds of the float64 oracle on the
  dequantised inputs (RMSE <= 1e-2, |error| <= (2^-4 + 1e-2) max|v|, LSE relative <= 1e-3), as
  for the fixed-length FP8 forward.
"""

import math

import numpy as np
import pytest

torch = pytest.importorskip("torch")

import exact_attention_100_b200 as ea
from exact_attention_100_b200 import build as ea_build
from exact_attention_100_b200.inputs import hadamard_signs, normal_qkv_packed
from oracle import attention_ref, dequant_ref, hadamard_quant_ref

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    ea_build.build()
    ea.lib()
    yield
    torch.cuda.synchronize()
    assert ea.attn_device_status() == ea.ATTN_OK


def _quantise(lq, lk, H, d, seed, max_q=None, max_k=None):
    qn, kn, vn, cq, ck = normal_qkv_packed(lq, lk, H, d, seed=seed)
    dev = lambda a: torch.from_numpy(a).to(torch.bfloat16).cuda()
    signs = hadamard_signs(d)
    tcq, tck = torch.from_numpy(cq).cuda(), torch.from_numpy(ck).cuda()
    mq, mk = max_q or max(max(lq), 1), max_k or max(max(lk), 1)
    outs = ea.attn_hadamard_quant_qkv_varlen(dev(qn), dev(kn), dev(vn), torch.from_numpy(signs).cuda(), tcq, tck,
                                             mq, mk)
    torch.cuda.synchronize()
    return (qn, kn, vn, cq, ck, signs, tcq, tck, mq, mk), outs


def _seq(x, cu, b):
    """rows of sequence b of a packed [total, H, d] array as [H, len, d]"""
    return np.ascontiguousarray(np.asarray(x)[cu[b]:cu[b + 1]].transpose(1, 0, 2))


@pytest.mark.parametrize("d", [64, 128, 256])
def test_prekernel_blocks_per_sequence_bit_exact(d):
    lq = [300, 1, 128, 513, 0, 257]
    lk = [129, 300, 128, 0, 5, 257]
    (qn, kn, vn, cq, ck, signs, *_), (q8, k8, v8, qs, ks, vs) = _quantise(lq, lk, 3, d, seed=d)
    for x, cu, codes, sc, sg in ((qn, cq, q8, qs, signs), (kn, ck, k8, ks, signs), (vn, ck, v8, vs, None)):
        codes, sc = codes.cpu().numpy(), sc.cpu().numpy()
        for b in range(len(lq)):
            n = int(cu[b + 1] - cu[b])
            if n == 0:
                continue
            rc, rs = hadamard_quant_ref(_seq(x, cu, b), sg)
            np.testing.assert_array_equal(_seq(codes, cu, b), rc)
            np.testing.assert_array_equal(sc[b, :, :rs.shape[-1]], rs)


def _check_forward(lq, lk, H, d, causal, seed, o_dtype=torch.float32, oracle_heads=None):
    (qn, kn, vn, cq, ck, signs, tcq, tck, mq, mk), (q8, k8, v8, qs, ks, vs) = _quantise(lq, lk, H, d, seed)
    o, lse = ea.attn_fwd_fp8_varlen(q8, k8, v8, qs, ks, vs, tcq, tck, mq, mk, causal=causal, o_dtype=o_dtype)
    torch.cuda.synchronize()
    assert ea.attn_device_status() == ea.ATTN_OK
    og, lg = o.cpu(), lse.cpu()
    q8c, k8c, v8c, qsc, ksc, vsc = (t.cpu().numpy() for t in (q8, k8, v8, qs, ks, vs))
    for b in range(len(lq)):
        nq, nk = int(cq[b + 1] - cq[b]), int(ck[b + 1] - ck[b])
        if nq == 0:
            continue
        ob = og[cq[b]:cq[b + 1]].permute(1, 0, 2)
        lb = lg[:, cq[b]:cq[b + 1]]
        if nk == 0:  # no key: O = 0 and LSE = -inf
            assert torch.all(ob == 0) and torch.all(torch.isneginf(lb))
            continue
        nbq, nbk = (nq + 127) // 128, (nk + 127) // 128
        sq = lambda t, cu: torch.from_numpy(_seq(t, cu, b)).cuda()[None]
        # fresh copies: a slice that is already contiguous would sit at an unaligned offset
        cp = lambda t, n: t[b:b + 1, :, :n].contiguous().clone()
        ref_o, ref_lse = ea.attn_fwd_fp8_qk(sq(q8c, cq), sq(k8c, ck), sq(v8c, ck), cp(qs, nbq), cp(ks, nbk),
                                            cp(vs, nbk), causal=causal, o_dtype=o_dtype)
        torch.cuda.synchronize()
        assert torch.equal(ob, ref_o[0].cpu()), b
        assert torch.equal(lb, ref_lse[0].cpu()), b
        heads = range(H) if oracle_heads is None else range(min(H, oracle_heads))
        for h in heads:
            qd = dequant_ref(_seq(q8c, cq, b)[h], qsc[b, h, :nbq])
            kd = dequant_ref(_seq(k8c, ck, b)[h], ksc[b, h, :nbk])
            vd = dequant_ref(_seq(v8c, ck, b)[h], vsc[b, h, :nbk])
            o_ref, lse_ref = attention_ref(qd[None, None], kd[None, None], vd[None, None], 1 / math.sqrt(d), causal)
            o_ref, lse_ref = o_ref[0, 0], lse_ref[0, 0]
            seen = np.isfinite(lse_ref)
            err = ob[h].float().numpy().astype(np.float64)[seen] - o_ref[seen]
            if err.size:
                assert float(np.sqrt(np.mean(err ** 2))) <= 1e-2, (b, h)
                assert np.abs(err).max() <= (2.0 ** -4 + 1e-2) * np.abs(vd).max(), (b, h)
                lrel = np.abs(lb[h].numpy()[seen] - lse_ref[seen]) / np.abs(lse_ref[seen])
                assert lrel.max() <= 1e-3, (b, h)
            assert np.all(np.isneginf(lb[h].numpy()[~seen]))


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("d", [64, 128, 256])
def test_forward_per_sequence_matches_fixed_length_and_oracle(d, causal):
    # ragged lengths, an empty key sequence, a single row, Nq != Nk both ways
    lq = [300, 1, 128, 513, 7, 257, 0]
    lk = [129, 300, 128, 513, 0, 130, 9]
    _check_forward(lq, lk, 2, d, causal, seed=3 * d + causal)


@pytest.mark.parametrize("causal", [True, False])
def test_bench_packed_batch(causal):
    """The packed batch the bench times (8 sequences of 391..3369 tokens, H=16, d=128): every
    sequence bit-identical to the fixed-length FP8 forward, the first two heads of each against
    the oracle."""
    from bench import VARLEN_WORKLOAD, varlen_lengths
    w = VARLEN_WORKLOAD
    lens = varlen_lengths(w["total"], w["lo"], w["hi"], w["seed"])
    _check_forward(lens, lens, w["H"], w["d"], causal, seed=w["seed"], o_dtype=torch.bfloat16, oracle_heads=2)


def test_shorter_max_seqlen_is_reported_not_read_past():
    """A key sequence longer than max_seqlen_k is skipped and reported; the others are computed."""
    lq, lk = [200, 300], [200, 300]
    (qn, kn, vn, cq, ck, signs, tcq, tck, mq, mk), (q8, k8, v8, qs, ks, vs) = _quantise(lq, lk, 2, 128, seed=5)
    ks2, vs2 = ks[:, :, :2].contiguous(), vs[:, :, :2].contiguous()  # room for 256 keys only
    o = torch.full((500, 2, 128), 7.0, dtype=torch.float32, device="cuda")
    ea.attn_fwd_fp8_varlen(q8, k8, v8, qs, ks2, vs2, tcq, tck, mq, 256, o=o, causal=True)
    torch.cuda.synchronize()
    assert ea.attn_device_status() == ea.ATTN_ERR_INVALID_ARG
    assert torch.all(o[200:] == 7.0)  # sequence 1 (300 keys > 256) untouched
    first = lambda t: t[:200].permute(1, 0, 2).contiguous()[None]
    ref_o, _ = ea.attn_fwd_fp8_qk(first(q8), first(k8), first(v8), qs[:1, :, :2].contiguous(),
                                  ks[:1, :, :2].contiguous(), vs[:1, :, :2].contiguous(), causal=True,
                                  o_dtype=torch.float32)
    torch.cuda.synchronize()
    assert torch.equal(o[:200].permute(1, 0, 2), ref_o[0])
