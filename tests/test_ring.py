"""Host logic of the ring (sequence-parallel) attention, CPU only: the hop schedule, and the
driver run over ``torch.distributed`` with the gloo backend on 2 and 3 processes.  The CUDA
kernels cannot run here, so these processes hand the driver CPU stand-ins for the attention of a
hop and for the merge (the float64 oracle); the exchange is the driver's own
``DistExchange``.  The result must be the oracle's attention over the whole sequence."""

import os
import socket

import numpy as np
import pytest
import torch

from exact_attention_100_b200.ring import ring_steps, ring_steps_zigzag, zigzag_chunks


@pytest.mark.parametrize("world", [1, 2, 3, 5])
@pytest.mark.parametrize("causal", [False, True])
def test_every_chunk_once_and_causal_modes(world, causal):
    for rank in range(world):
        steps = ring_steps(rank, world, causal)
        assert sorted(c for c, _ in steps) == list(range(world))
        assert steps[0] == (rank, "causal" if causal else "full")  # a rank starts with its own chunk
        for c, mode in steps:
            if not causal:
                assert mode == "full"
            else:
                assert mode == ("full" if c < rank else "causal" if c == rank else "skip")


def test_rejects_bad_rank():
    with pytest.raises(ValueError):
        ring_steps(3, 3, True)
    with pytest.raises(ValueError):
        ring_steps_zigzag(-1, 3, True)


@pytest.mark.parametrize("world", [1, 2, 3, 4, 7])
@pytest.mark.parametrize("causal", [False, True])
def test_zigzag_covers_every_visible_pair_once_and_balances_work(world, causal):
    """Every (query chunk, key chunk) pair that causality allows is attended exactly once, by the
    rank holding the query chunk, with the right mode; with causal masking every rank attends
    2W - 1 chunks fully and two diagonals (the contiguous layout: rank r attends r + 1)."""
    seen = {}
    work = []
    for rank in range(world):
        qa = zigzag_chunks(rank, world)
        w = 0
        steps = ring_steps_zigzag(rank, world, causal)
        assert sorted(src for src, _ in steps) == list(range(world))
        for src, pairs in steps:
            kc = zigzag_chunks(src, world)
            for qh, kh, mode in pairs:
                key = (qa[qh], kc[kh])
                assert key not in seen, key
                seen[key] = mode
                w += 2 if mode == "full" else 1
        work.append(w)
    n = 2 * world
    for a in range(n):
        for b in range(n):
            if causal and b > a:
                assert (a, b) not in seen
            else:
                assert seen[(a, b)] == ("causal" if causal and a == b else "full"), (a, b)
    assert len(set(work)) == 1, work


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, causal, out_dir, layout="contiguous"):
    import datetime
    import torch.distributed as dist
    from oracle import attention_ref, merge_partials_ref
    from exact_attention_100_b200.ring import ring_attention_fwd

    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        B, H, Nc, d = 1, 2, 5, 4
        rng = np.random.default_rng(0)
        if layout == "zigzag":  # 2W chunks of Nc rows; this rank holds chunks rank and 2W - 1 - rank
            q, k, v = (rng.standard_normal((B, H, 2 * world * Nc, d)) for _ in range(3))
            a, b = zigzag_chunks(rank, world)
            sl = np.r_[a * Nc:(a + 1) * Nc, b * Nc:(b + 1) * Nc]
        else:
            q, k, v = (rng.standard_normal((B, H, world * Nc, d)) for _ in range(3))
            sl = np.r_[rank * Nc:(rank + 1) * Nc]
        tq, tk, tv = (torch.from_numpy(np.ascontiguousarray(x[:, :, sl])) for x in (q, k, v))

        def compute(q_, k_, v_, causal_):
            o, lse = attention_ref(q_.numpy(), k_.numpy(), v_.numpy(), 0.5, causal_)
            return torch.from_numpy(o), torch.from_numpy(lse)

        def merge(o_acc, lse_acc, o_p, lse_p):
            o, lse = merge_partials_ref(o_acc.numpy(), lse_acc.numpy(), o_p.numpy(), lse_p.numpy())
            o_acc.copy_(torch.from_numpy(o))
            lse_acc.copy_(torch.from_numpy(lse))

        q64 = tq.double()
        o, lse = ring_attention_fwd(q64, tk.double(), tv.double(), causal=causal, scale=0.5, compute=compute,
                                    merge=merge, layout=layout)
        o_ref, lse_ref = attention_ref(q, k, v, 0.5, causal)
        np.save(os.path.join(out_dir, f"r{rank}.npy"), np.array([
            float(np.abs(o.numpy() - o_ref[:, :, sl]).max()), float(np.abs(lse.numpy() - lse_ref[:, :, sl]).max())]))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("layout", ["contiguous", "zigzag"])
@pytest.mark.parametrize("world", [2, 3])
@pytest.mark.parametrize("causal", [False, True])
def test_gloo_ring_matches_whole_sequence(world, causal, layout, tmp_path):
    import torch.multiprocessing as mp
    mp.start_processes(_worker, args=(world, _free_port(), causal, str(tmp_path), layout), nprocs=world, join=True,
                       start_method="spawn")
    for r in range(world):
        err_o, err_l = np.load(tmp_path / f"r{r}.npy")
        # the driver keeps its running O and LSE in float32 (as the GPU path does)
        assert err_o < 1e-6 and err_l < 1e-6, (r, err_o, err_l)
