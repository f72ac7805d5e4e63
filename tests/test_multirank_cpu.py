"""Multi-rank host logic on CPU: world-size-2 `gloo` ranks.

The path shards over heads with no data-path collective.  These tests check
the head partition (GQA groups kept whole, every head once), that the
gathered sharded result equals the unsharded one bit for bit (computed here
with the CPU oracle standing in for each rank's device), and the
max-over-ranks timing reduction the benchmark uses.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from long_context_structured_b200.shard import head_shard, max_over_ranks, sharded_fwd


def test_head_shard_partitions_heads():
    for Hq, Hkv in [(32, 32), (32, 8), (8, 1), (6, 3)]:
        for world in (1, 2, 3, 4, 8, 16):
            seen = []
            for r in range(world):
                q0, q1, kv0, kv1 = head_shard(Hq, Hkv, world, r)
                rep = Hq // Hkv
                assert q0 == kv0 * rep and q1 == kv1 * rep
                seen += list(range(q0, q1))
            assert seen == list(range(Hq)), (Hq, Hkv, world)
    with pytest.raises(ValueError):
        head_shard(6, 4, 2, 0)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _oracle_compute(q, k, v, **kw):
    """Stand-in for a rank's device: the fp64 oracle on the shard."""
    from oracle import oracle as O
    B, Hq, T, d = q.shape
    Hkv = k.shape[1]
    bits = lambda t: t.contiguous().view(torch.int16).numpy().view(np.uint16)
    p = O.params(B, Hq, Hkv, T, d, "bf16", kw["n_start"], kw["window"], kw["L_pretrain"], 0, kw["rope_theta"])
    sep = kw.get("is_sep")
    sep = None if sep is None else sep.numpy().astype(np.uint8)
    Oo, lse, *_ = O.fwd_rows(p, bits(q), bits(k), bits(v), sep, O.all_rows(B, Hq, T), nthreads=2)
    return torch.from_numpy(Oo.reshape(B, Hq, T, d)), torch.from_numpy(lse.reshape(B, Hq, T))


def _inputs(B=1):
    g = torch.Generator().manual_seed(42)
    Hq, Hkv, T, d = 6, 3, 40, 16
    q = torch.randn(B, Hq, T, d, generator=g).bfloat16()
    k = torch.randn(B, Hkv, T, d, generator=g).bfloat16()
    v = torch.randn(B, Hkv, T, d, generator=g).bfloat16()
    return q, k, v


KW = dict(n_start=2, window=5, L_pretrain=5, rope_theta=1e4)


def _kw_sep():
    """Separators (per sequence, shared by every head) and a window below the
    cap: the flags travel whole to every rank."""
    g = torch.Generator().manual_seed(7)
    sep = (torch.rand(2, 40, generator=g) < 0.25).to(torch.uint8)
    return dict(n_start=2, window=4, L_pretrain=9, rope_theta=1e4, is_sep=sep)


def _worker(rank, world, port, out, with_sep):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        q, k, v = _inputs(2 if with_sep else 1)
        kw = _kw_sep() if with_sep else KW
        O, lse, rng = sharded_fwd(q, k, v, world=world, rank=rank, compute=_oracle_compute, gather=True, **kw)
        t = max_over_ranks(1.0 + rank)
        if rank == 0:
            torch.save({"O": O, "lse": lse, "t": t}, out)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("with_sep", [False, True])
def test_sharded_equals_unsharded_two_ranks(tmp_path, with_sep):
    """Two ranks over three kv heads (an uneven split: 2 + 1), the head
    blocks all-gathered back in head order; equal bit for bit to the oracle
    run on the whole layer."""
    out = str(tmp_path / "res.pt")
    port = _free_port()
    mp.start_processes(_worker, args=(2, port, out, with_sep), nprocs=2, start_method="spawn", join=True)
    res = torch.load(out)
    q, k, v = _inputs(2 if with_sep else 1)
    O_ref, lse_ref = _oracle_compute(q, k, v, **(_kw_sep() if with_sep else KW))
    assert torch.equal(res["O"], O_ref) and torch.equal(res["lse"], lse_ref)
    assert res["t"] == 2.0  # the slowest rank's time


def test_sharding_refuses_alibi():
    q, k, v = _inputs()
    with pytest.raises(NotImplementedError):
        sharded_fwd(q, k, v, world=2, rank=0, compute=_oracle_compute, alibi=True, **KW)


def test_single_rank_no_collective():
    q, k, v = _inputs()
    O, lse, rng = sharded_fwd(q, k, v, world=1, rank=0, compute=_oracle_compute, **KW)
    O_ref, lse_ref = _oracle_compute(q, k, v, **KW)
    assert rng == (0, 6) and torch.equal(O, O_ref)
    assert max_over_ranks(3.5) == 3.5
