"""Sequence-parallel (ring) attention forward over the library's kernels.

"FlashAttention-2/3" names sequence parallelism across devices as the way to long contexts;
the pages give no algorithm for it, and the plainest reading is the ring: the sequence is cut
into W contiguous chunks, rank r holds query, key and value chunk r, and the key/value chunks
travel around the ring (rank r sends to r + 1 and receives from r - 1) for W - 1 hops.  At hop
s rank r holds key chunk (r - s) mod W and attends to it -- fully when it precedes its own
chunk, causally when it is its own chunk, not at all when it follows (causal) -- and merges
the partial (O, LSE) into its running result with ``attn_merge_partials``.  The exchange for
the next hop is posted before the current hop's attention, so the transfer overlaps it.

With causal masking the contiguous cut leaves the work unbalanced: rank r attends to r + 1
chunks.  The zig-zag layout balances it: the sequence is cut into 2W chunks and rank r holds
chunks r and 2W - 1 - r, so every rank attends to 2W - 1 chunks fully and to two diagonals.
The two chunks travel together; at each hop a rank attends each of its query chunks to each
held key chunk that precedes it (fully) or is the same chunk (causally).

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


def zigzag_chunks(rank: int, world: int) -> Tuple[int, int]:
    """The two chunks of the 2 * world that rank ``rank`` holds in the zig-zag layout."""
    return rank, 2 * world - 1 - rank


def ring_steps_zigzag(rank: int, world: int, causal: bool) -> List[Tuple[int, List[Tuple[int, int, str]]]]:
    """For hops 0 .. world - 1 of ``rank`` in the zig-zag layout: (source rank, pairs), where the
    rank holds the two chunks of source rank (rank - s) mod world and pairs lists (query half,
    key half, mode) for every pair it attends -- mode "full" (the key chunk precedes the query
    chunk, or not causal) or "causal" (the same chunk); pairs whose key chunk follows are left
    out."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("need 0 <= rank < world")
    qa = zigzag_chunks(rank, world)
    out = []
    for s in range(world):
        src = (rank - s) % world
        kc = zigzag_chunks(src, world)
        pairs = []
        for qh in (0, 1):
            for kh in (0, 1):
                if not causal or kc[kh] < qa[qh]:
                    pairs.append((qh, kh, "full"))
                elif kc[kh] == qa[qh]:
                    pairs.append((qh, kh, "causal"))
        out.append((src, pairs))
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
                       compute: Optional[Callable] = None, merge: Optional[Callable] = None,
                       layout: str = "contiguous"):
    """Attention of this rank's query chunk ``q`` [B, H, Nc, d] over the whole sequence, whose
    key/value chunks ``k``, ``v`` [B, H, Nc, d] are spread over the ranks of ``group`` in rank
    order (chunk r on rank r; all chunks of one length).  Returns ``(O float32 [B, H, Nc, d],
    LSE float32 [B, H, Nc])`` of the rows of this chunk.

    ``layout="zigzag"``: q, k, v [B, H, 2C, d] hold the rank's two chunks of the 2 * world (chunk
    rank, then chunk 2 * world - 1 - rank, each of C rows, see :func:`zigzag_chunks`), and the
    result covers the same rows in the same order; with causal masking every rank then does the
    same work.

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
    if layout == "zigzag":
        if q.shape[2] % 2 != 0 or k.shape[2] != q.shape[2]:
            raise ValueError("the zig-zag layout needs two query and two key chunks of one length")
        c = q.shape[2] // 2
        halves = [q[:, :, :c].contiguous(), q[:, :, c:].contiguous()]
        accs = [(torch.zeros(h.shape, dtype=torch.float32, device=q.device),
                 torch.full(h.shape[:-1], float("-inf"), dtype=torch.float32, device=q.device)) for h in halves]
        # one buffer per hop, each half contiguous: [half][K or V][B, H, C, d]
        kv = torch.stack([torch.stack([k[:, :, :c], v[:, :, :c]]), torch.stack([k[:, :, c:], v[:, :, c:]])])
        for hop, (_, pairs) in enumerate(ring_steps_zigzag(rank, world, causal)):
            pending = exchange.start(kv) if hop + 1 < world else None
            for qh, kh, mode in pairs:
                o_p, lse_p = compute(halves[qh], kv[kh][0], kv[kh][1], mode == "causal")
                merge(accs[qh][0], accs[qh][1], o_p, lse_p)
            if pending is not None:
                kv = pending.wait()
        return torch.cat([accs[0][0], accs[1][0]], dim=2), torch.cat([accs[0][1], accs[1][1]], dim=2)
    if layout != "contiguous":
        raise ValueError("layout must be 'contiguous' or 'zigzag'")
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
