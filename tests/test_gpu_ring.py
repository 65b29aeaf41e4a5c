"""The merge kernel (attn_merge_partials) against the oracle's merge, and the ring attention
driver run with the library's kernels for W simulated ranks on one GPU (their exchange replaced
by handing each rank the chunk the ring would deliver), against the oracle's attention over the
whole sequence."""

import math

import numpy as np
import pytest
import torch

import exact_attention_100_b200 as ea
from exact_attention_100_b200.inputs import normal_qkv
from exact_attention_100_b200.ring import ring_attention_fwd
from oracle import attention_ref, merge_partials_ref

from gpu_util import LSE_REL, O_MAX_ABS, O_MEAN_ABS

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("part_dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("d", [64, 128, 256])
def test_merge_kernel_matches_oracle(d, part_dtype):
    rng = np.random.default_rng(d)
    rows = 3001
    oa, ob = rng.standard_normal((rows, d)), rng.standard_normal((rows, d))
    la, lb = rng.normal(0, 3, rows), rng.normal(0, 3, rows)
    la[::7] = -np.inf  # rows whose accumulated part has no key yet
    lb[::11] = -np.inf  # rows whose new part sees no key
    oa[::7] = 0.0
    ob_dev = torch.from_numpy(ob).to(part_dtype)
    ob_used = ob_dev.double().numpy()  # what the kernel reads
    acc_o = torch.from_numpy(oa).float().cuda()
    acc_l = torch.from_numpy(la).float().cuda()
    ea.attn_merge_partials(acc_o, acc_l, ob_dev.cuda(), torch.from_numpy(lb).float().cuda())
    torch.cuda.synchronize()
    ro, rl = merge_partials_ref(oa.astype(np.float32).astype(np.float64), la.astype(np.float32).astype(np.float64),
                                ob_used, lb.astype(np.float32).astype(np.float64))
    go, gl = acc_o.double().cpu().numpy(), acc_l.double().cpu().numpy()
    both = np.isneginf(rl)
    assert np.array_equal(np.isneginf(gl), both)
    assert np.all(go[both] == 0)
    assert np.abs(go - ro).max() <= 1e-5 * max(1.0, np.abs(ro).max())
    assert np.abs(gl[~both] - rl[~both]).max() <= 1e-5 * max(1.0, np.abs(rl[~both]).max())


class _Emulated:
    """The ring's delivery for rank r: at hop s it holds chunk (r - s) mod W."""

    def __init__(self, chunks, rank):
        self.chunks, self.rank, self.hop = chunks, rank, 0

    def start(self, kv):
        self.hop += 1
        nxt = self.chunks[(self.rank - self.hop) % len(self.chunks)]

        class _P:
            def wait(_self):
                return nxt
        return _P()


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("world", [1, 2, 4])
def test_ring_driver_zigzag_on_one_gpu(world, causal):
    """The zig-zag layout with the library's kernels, each rank emulated on one GPU: rank r holds
    chunks r and 2W - 1 - r of 2W; its rows of the whole-sequence result within the bf16 bars."""
    from exact_attention_100_b200.ring import zigzag_chunks
    B, H, N, d = 1, 2, 1024, 128
    q, k, v = normal_qkv(B, H, N, d, seed=10 + world)
    tq, tk, tv = (torch.from_numpy(a).to(torch.bfloat16).cuda() for a in (q, k, v))
    c = N // (2 * world)
    rows = [np.r_[a * c:(a + 1) * c, b * c:(b + 1) * c] for a, b in (zigzag_chunks(r, world) for r in range(world))]
    idx = [torch.from_numpy(r).cuda() for r in rows]
    held = [(tk[:, :, i].contiguous(), tv[:, :, i].contiguous()) for i in idx]
    bufs = [torch.stack([torch.stack([kk[:, :, :c], vv[:, :, :c]]), torch.stack([kk[:, :, c:], vv[:, :, c:]])])
            for kk, vv in held]
    scale = 1.0 / math.sqrt(d)
    o_ref, lse_ref = attention_ref(q, k, v, scale, causal)
    for r in range(world):
        o, lse = ring_attention_fwd(tq[:, :, idx[r]].contiguous(), held[r][0], held[r][1], causal=causal,
                                    scale=scale, rank=r, world=world, exchange=_Emulated(bufs, r), layout="zigzag")
        torch.cuda.synchronize()
        assert ea.attn_device_status() == ea.ATTN_OK
        err = np.abs(o.double().cpu().numpy() - o_ref[:, :, rows[r]])
        assert err.max() <= O_MAX_ABS and err.mean() <= O_MEAN_ABS, (r, err.max())
        rel = np.abs(lse.double().cpu().numpy() - lse_ref[:, :, rows[r]]) / np.abs(lse_ref[:, :, rows[r]])
        assert rel.max() <= LSE_REL, (r, rel.max())


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("world", [1, 2, 4])
def test_ring_driver_on_one_gpu(world, causal):
    B, H, N, d = 1, 2, 1024, 128
    q, k, v = normal_qkv(B, H, N, d, seed=world)
    tq, tk, tv = (torch.from_numpy(a).to(torch.bfloat16).cuda() for a in (q, k, v))
    nc = N // world
    chunks = [torch.stack([tk[:, :, r * nc:(r + 1) * nc], tv[:, :, r * nc:(r + 1) * nc]]).contiguous()
              for r in range(world)]
    scale = 1.0 / math.sqrt(d)
    o_ref, lse_ref = attention_ref(q, k, v, scale, causal)
    for r in range(world):
        sl = slice(r * nc, (r + 1) * nc)
        o, lse = ring_attention_fwd(tq[:, :, sl].contiguous(), chunks[r][0], chunks[r][1], causal=causal, scale=scale,
                                    rank=r, world=world, exchange=_Emulated(chunks, r))
        torch.cuda.synchronize()
        assert ea.attn_device_status() == ea.ATTN_OK
        err = np.abs(o.double().cpu().numpy() - o_ref[:, :, sl])
        assert err.max() <= O_MAX_ABS and err.mean() <= O_MEAN_ABS, (r, err.max())
        rel = np.abs(lse.double().cpu().numpy() - lse_ref[:, :, sl]) / np.abs(lse_ref[:, :, sl])
        assert rel.max() <= LSE_REL, (r, rel.max())
