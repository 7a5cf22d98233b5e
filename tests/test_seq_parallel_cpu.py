"""Host logic of the sequence-parallel decode on CPU: the page ranges the ranks
take, and the gather of their partials over gloo ranks (world size 2 and 3)
in the layout xmla_combine_shards reads.  The partials are made by the
oracle in the library's layout and units (M in log2 units), so the test
checks the plumbing and the layout contract, not the kernels."""
import math
import os
import socket
import sys
from datetime import timedelta

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from mla_latent_kv_yarn_b200 import seq_parallel as sp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("npages", [0, 1, 2, 7, 64, 4097])
@pytest.mark.parametrize("world", [1, 2, 3, 8])
def test_shard_pages_partition_the_pages(npages, world):
    ranges = [sp.shard_pages(npages, world, r) for r in range(world)]
    assert ranges[0][0] == 0 and ranges[-1][1] == npages
    for (lo, hi), (lo2, _) in zip(ranges[:-1], ranges[1:]):
        assert hi == lo2                                   # contiguous, disjoint
    sizes = [hi - lo for lo, hi in ranges]
    assert min(sizes) >= 0 and max(sizes) - min(sizes) <= 1
    assert sizes == sorted(sizes, reverse=True)            # the larger shares come first


def test_shard_pages_rejects_bad_requests():
    for args in [(10, 0, 0), (10, 2, 2), (10, 2, -1), (-1, 2, 0)]:
        with pytest.raises(ValueError):
            sp.shard_pages(*args)


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


class _HostShard(sp.ShardDecoder):
    """The buffers of a ShardDecoder on the CPU (no library calls)."""

    def __init__(self, batch, q_len, max_seqlen, world, rank):
        self.batch, self.q_len, self.max_seqlen = batch, q_len, max_seqlen
        self.world, self.rank = world, rank
        self.page_lo, self.page_hi = sp.shard_pages((max_seqlen + 63) // 64, world, rank)
        R = batch * q_len * 32
        self.partial_floats = R * 514
        self.partial = torch.zeros(self.partial_floats, dtype=torch.float32)
        self.gathered = torch.zeros(world * self.partial_floats, dtype=torch.float32)


def _case(seed, seqlens, q_len):
    from oracle import mla_oracle as om
    rng = np.random.default_rng(seed)
    B = len(seqlens)
    q = rng.standard_normal((B, q_len, 32, 192))
    seqs = [(rng.standard_normal((n, 512)), rng.standard_normal((n, 64))) for n in seqlens]
    W_UK = rng.standard_normal((32, 128, 512)) / math.sqrt(512)
    W_UV = rng.standard_normal((32, 512, 128)) / math.sqrt(512)
    return om, q, seqs, W_UK, W_UV


def _worker(rank, world, port, seqlens, q_len, res):
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        om, q, seqs, W_UK, W_UV = _case(3, seqlens, q_len)
        cfg = om.YarnConfig()
        sh = _HostShard(len(seqlens), q_len, max(seqlens), world, rank)
        O, ML = sp.partial_views(sh.partial, sh.batch, q_len)
        for b, (c, k) in enumerate(seqs):
            n = c.shape[0]
            t_lo, t_hi = min(n, 64 * sh.page_lo), min(n, 64 * sh.page_hi)
            k_rot = om.rope(k, np.arange(n), cfg)
            m, l, o = om.attention_partial(q[b], c[t_lo:t_hi], k_rot[t_lo:t_hi], W_UK, cfg, n,
                                           t_lo, t_hi)
            rows = slice(b * q_len * 32, (b + 1) * q_len * 32)
            O[rows] = torch.from_numpy(o.reshape(-1, 512))
            ML[rows, 0] = torch.from_numpy(m.reshape(-1) / math.log(2.0))   # log2 units
            ML[rows, 1] = torch.from_numpy(l.reshape(-1))
        sh.gather()
        # what xmla_combine_shards computes, read from the gathered buffer
        R = sh.batch * q_len * 32
        parts = []
        for g in range(world):
            Og, MLg = sp.partial_views(sh.gathered[g * sh.partial_floats:], sh.batch, q_len)
            parts.append((MLg[:, 0].double().numpy() * math.log(2.0), MLg[:, 1].double().numpy(),
                          Og.double().numpy()))
        m, l, o = om.merge_partials(parts)
        got = om.finish_partial(m.reshape(sh.batch * q_len, 32), l.reshape(sh.batch * q_len, 32),
                                o.reshape(sh.batch * q_len, 32, 512), W_UV)
        err = 0.0
        for b, (c, k) in enumerate(seqs):
            want = om.mla_attention_expanded(q[b], c, k, W_UK, W_UV, cfg)
            err = max(err, float(np.abs(got[b * q_len:(b + 1) * q_len] - want).max()))
        assert R == sh.partial_floats // 514
        res.put((rank, err))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,seqlens,q_len", [(2, [300], 1), (3, [200, 1000], 2)])
def test_gathered_partials_merge_to_the_full_attention(world, seqlens, q_len):
    # float32 partials (the library's layout) against the fp64 expanded oracle
    ctx = mp.get_context("spawn")
    res = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, seqlens, q_len, res))
             for r in range(world)]
    for p in procs:
        p.start()
    got = sorted(res.get(timeout=180) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [g[0] for g in got] == list(range(world))
    assert max(g[1] for g in got) < 1e-5
