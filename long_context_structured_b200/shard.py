"""Head sharding across ranks (one process per GPU).

Every (batch, query head) of the structured attention is an independent
problem given Q/K/V, so a layer shards over heads with no data-path
collective: rank r takes a contiguous block of key/value heads together with
all the query heads that read them (GQA groups never split), computes its
heads on its own GPU, and the caller either keeps the shard or gathers the
head blocks back in head order.
"""
from __future__ import annotations

from typing import Callable, Optional, Tuple


def head_shard(Hq: int, Hkv: int, world: int, rank: int) -> Tuple[int, int, int, int]:
    """(q0, q1, kv0, kv1): the query-head and kv-head ranges of `rank`.

    KV heads are split as evenly as possible (the first Hkv % world ranks get
    one more); each rank's query heads are the groups of its kv heads.  A
    rank may get an empty range when world > Hkv.
    """
    if Hq % Hkv:
        raise ValueError("Hq must be a multiple of Hkv")
    if not (0 <= rank < world):
        raise ValueError("rank out of range")
    rep = Hq // Hkv
    base, extra = divmod(Hkv, world)
    kv0 = rank * base + min(rank, extra)
    kv1 = kv0 + base + (1 if rank < extra else 0)
    return kv0 * rep, kv1 * rep, kv0, kv1


def sharded_fwd(q, k, v, *, world: int, rank: int, compute: Optional[Callable] = None, group=None,
                gather: bool = False, **kw):
    """Run this rank's head block of a forward.

    q [B,Hq,T,d], k/v [B,Hkv,T,d] hold the full layer (or at least this
    rank's heads).  `compute(q, k, v, **kw) -> (O, lse)` defaults to
    `long_context_structured_b200.fwd`.  With gather=True the head blocks of
    all ranks are gathered (torch.distributed all_gather over `group`) and
    the full (O, lse) is returned; otherwise this rank's block and its range.
    """
    import torch

    if compute is None:
        from . import fwd as compute
    if kw.get("alibi"):
        # the ALiBi slope of a head depends on its index among all Hq heads,
        # which a head block run on its own does not know
        raise NotImplementedError("head sharding with ALiBi is not supported")
    Hq, Hkv = q.shape[1], k.shape[1]
    q0, q1, kv0, kv1 = head_shard(Hq, Hkv, world, rank)
    if q1 > q0:
        O, lse = compute(q[:, q0:q1], k[:, kv0:kv1], v[:, kv0:kv1], **kw)
    else:
        O = q.new_empty((q.shape[0], 0, q.shape[2], q.shape[3]))
        lse = torch.empty((q.shape[0], 0, q.shape[2]), dtype=torch.float32, device=q.device)
    if not gather:
        return O, lse, (q0, q1)
    O_full, l_full = gather_heads(O, lse, Hq, Hkv, world, group=group)
    return O_full, l_full, (0, Hq)


def gather_heads(O, lse, Hq: int, Hkv: int, world: int, group=None):
    """All-gather every rank's head block (O [B, h_r, T, d], lse [B, h_r, T])
    into the full layer in head order.  Blocks are padded to the largest so
    that one all_gather of equal shapes moves them."""
    import torch
    import torch.distributed as dist

    sizes = [head_shard(Hq, Hkv, world, r)[1] - head_shard(Hq, Hkv, world, r)[0] for r in range(world)]
    hmax = max(sizes)
    Op = O.new_zeros((O.shape[0], hmax, O.shape[2], O.shape[3]))
    lp = lse.new_zeros((lse.shape[0], hmax, lse.shape[2]))
    Op[:, : O.shape[1]] = O
    lp[:, : lse.shape[1]] = lse
    Os = [torch.empty_like(Op) for _ in range(world)]
    ls = [torch.empty_like(lp) for _ in range(world)]
    dist.all_gather(Os, Op.contiguous(), group=group)
    dist.all_gather(ls, lp.contiguous(), group=group)
    O_full = torch.cat([Os[r][:, : sizes[r]] for r in range(world)], dim=1)
    l_full = torch.cat([ls[r][:, : sizes[r]] for r in range(world)], dim=1)
    return O_full, l_full


def max_over_ranks(value: float, group=None, device=None) -> float:
    """Largest `value` over all ranks (timings are reported as the slowest rank)."""
    import torch
    import torch.distributed as dist

    if not dist.is_available() or not dist.is_initialized():
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return float(t.item())
