"""Sequence-parallel (ring) attention forward over the library's kernels.

"FlashAttention-2/3" names sequence parallelism across devices as the way to long contexts;
the pages give no algorithm for it, and the plainest reading is the ring: the sequence is cut
into W contiguous chunks, rank r holds query, key and value chunk r, and the key/value chunks
travel around the ring (rank r sends to r + 1 and receives from r - 1) for W - 1 hops.  At hop
s rank r holds key chunk (r - s) mod W and attends to it -- fully when it precedes its own
chunk, causally when it is its own chunk, not at all when it follows (causal) -- and merges
the partial (O, LSE) into its running result with ``attn_merge_partials``.  The exchange for
the next hop is posted before the current hop's attention, so the transfer overlaps it.

Only the host logic lives here: the attention of a hop is ``attn_fwd_qk`` (float32 O) and the
merge is ``attn_merge_partials``, both CUDA kernels of the library.  The exchange goes through
``torch.distributed`` point-to-point operations (NCCL between GPUs: copies into this GPU's
memory, no kernel reads another GPU's memory).
"""

from __future__ import annotations

from typing import Callable, List, Optional, Tuple


def ring_steps(rank: int, world: int, causal: bool) -> List[Tuple[int, str]]:
    """(key chunk, mode) for hops 0 .. world - 1 of ``rank``: at hop s the rank holds key chunk
    (rank - s) mod world; mode is "full", "causal" (its own chunk, the diagonal) or "skip"
    (causal, a chunk after its own)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("need 0 <= rank < world")
    out = []
    for s in range(world):
        c = (rank - s) % world
        if not causal or c < rank:
            mode = "full"
        elif c == rank:
            mode = "causal"
        else:
            mode = "skip"
        out.append((c, mode))
    return out


class _Pending:
    def __init__(self, reqs, buf):
        self.reqs, self.buf = reqs, buf

    def wait(self):
        for r in self.reqs:
            r.wait()
        return self.buf


class DistExchange:
    """Ring exchange through ``torch.distributed``: ``start(kv)`` posts the send of ``kv`` to the
    next rank and the receive of the previous rank's chunk into a fresh buffer; ``wait()`` on
    the result returns that buffer."""

    def __init__(self, group=None):
        import torch.distributed as dist
        self.dist, self.group = dist, group
        self.rank = dist.get_rank(group)
        self.world = dist.get_world_size(group)

    def start(self, kv):
        import torch
        dist = self.dist
        nxt = dist.get_global_rank(self.group, (self.rank + 1) % self.world) if self.group is not None \
            else (self.rank + 1) % self.world
        prv = dist.get_global_rank(self.group, (self.rank - 1) % self.world) if self.group is not None \
            else (self.rank - 1) % self.world
        recv = torch.empty_like(kv)
        ops = [dist.P2POp(dist.isend, kv, nxt, self.group), dist.P2POp(dist.irecv, recv, prv, self.group)]
        return _Pending(dist.batch_isend_irecv(ops), recv)


def ring_attention_fwd(q, k, v, causal: bool = False, scale: Optional[float] = None, group=None, *,
                       rank: Optional[int] = None, world: Optional[int] = None, exchange=None,
                       compute: Optional[Callable] = None, merge: Optional[Callable] = None):
    """Attention of this rank's query chunk ``q`` [B, H, Nc, d] over the whole sequence, whose
    key/value chunks ``k``, ``v`` [B, H, Nc, d] are spread over the ranks of ``group`` in rank
    order (chunk r on rank r; all chunks of one length).  Returns ``(O float32 [B, H, Nc, d],
    LSE float32 [B, H, Nc])`` of the rows of this chunk.

    ``rank``, ``world`` and ``exchange`` default to ``torch.distributed`` (a single process with
    no process group is rank 0 of 1); ``compute(q, k, v, causal) -> (O, LSE)`` and
    ``merge(o_acc, lse_acc, o_part, lse_part)`` default to the library's kernels.
    """
    import math
    import torch
    from . import attn_fwd_qk, attn_merge_partials

    if rank is None or world is None:
        import torch.distributed as dist
        if dist.is_available() and dist.is_initialized():
            rank, world = dist.get_rank(group), dist.get_world_size(group)
        else:
            rank, world = 0, 1
    if world > 1 and exchange is None:
        exchange = DistExchange(group)
    s = float(scale) if scale is not None else 1.0 / math.sqrt(int(q.shape[-1]))
    if compute is None:
        def compute(q_, k_, v_, causal_):
            return attn_fwd_qk(q_, k_, v_, scale=s, causal=causal_, o_dtype=torch.float32)
    if merge is None:
        merge = attn_merge_partials
    if k.shape != v.shape or k.shape[:2] != q.shape[:2] or k.shape[-1] != q.shape[-1]:
        raise ValueError("q, k, v must be [B, H, Nc, d] chunks of one head layout")
    if causal and k.shape[2] != q.shape[2]:
        raise ValueError("causal ring attention needs query and key chunks of one length")
    acc_o = torch.zeros(q.shape, dtype=torch.float32, device=q.device)
    acc_lse = torch.full(q.shape[:-1], float("-inf"), dtype=torch.float32, device=q.device)
    kv = torch.stack([k, v])  # one buffer per hop: K and V travel together
    for hop, (_, mode) in enumerate(ring_steps(rank, world, causal)):
        pending = exchange.start(kv) if hop + 1 < world else None
        if mode != "skip":
            o_p, lse_p = compute(q, kv[0], kv[1], mode == "causal")
            merge(acc_o, acc_lse, o_p, lse_p)
        if pending is not None:
            kv = pending.wait()
    return acc_o, acc_lse
