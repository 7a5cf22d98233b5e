"""Sequence-parallel decode: the pages of long sequences spread over G GPUs.

The absorbed attention of a query is a softmax-weighted sum over the cached
latent rows ([P5] "mHC+MLA+MTP 是什么？拆开给 Agent 用的百亿 MoE", section
"MLA：256K 上下文的'内存革命'"), so it splits over any partition of a
sequence's tokens and the parts merge exactly by their log-sum-exp.  Rank g of
G keeps logical pages [page_lo, page_hi) of every sequence in its own pool
(pages are dealt out contiguously, `shard_pages`), and one decode is:

  1. xmla_decode_shard on every rank: query absorb, split-K attention over the
     rank's pages, merge of its splits into one partial per (query row, head)
     -- 514 floats: O[512], M, L -- 66 KB per rank for one 32-head query;
  2. an all-gather of the partials (NCCL over NVLink between GPUs);
  3. xmla_combine_shards on every rank: the log-sum-exp merge of the G
     partials and the W_UV product, out[B, q_len, 32, 128] (bf16).

Only plumbing lives here (buffers, page ranges, the collective); every step
of the computation runs in libxmla's kernels.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import xmla
from .session import LayerState, new_pool, num_sms
from .workloads import D_LATENT, D_V, N_HEADS, PAGE


def shard_pages(npages: int, world: int, rank: int) -> tuple[int, int]:
    """Logical page range [lo, hi) of `rank` when `npages` pages are dealt out
    contiguously over `world` ranks, the first npages % world ranks taking one
    page more."""
    if world < 1 or not 0 <= rank < world or npages < 0:
        raise ValueError(f"bad shard request: npages={npages} world={world} rank={rank}")
    base, extra = divmod(npages, world)
    lo = rank * base + min(rank, extra)
    return lo, lo + base + (1 if rank < extra else 0)


def shard_layer(st: LayerState, page_lo: int, page_hi: int) -> LayerState:
    """The part of a layer's cache one rank keeps: the blocks of logical pages
    [page_lo, page_hi) of every sequence, copied into a pool of their own, and a
    block table indexed by the logical page (entries outside the range are -1
    and are never read by xmla_decode_shard)."""
    bt = st.block_table
    B, max_blocks = bt.shape
    lo = min(page_lo, max_blocks)
    hi = min(page_hi, max_blocks)
    width = max(0, hi - lo)
    src = bt[:, lo:hi].reshape(-1).long()
    keep = src >= 0
    n = int(keep.sum().item())
    pool = new_pool(max(1, n), st.pool.device, 0.0)
    local_bt = torch.full_like(bt, -1)
    if n > 0:
        pool[:n] = st.pool[src[keep]]
        ids = torch.full((B * width,), -1, dtype=torch.int32, device=bt.device)
        ids[keep] = torch.arange(n, dtype=torch.int32, device=bt.device)
        local_bt[:, lo:hi] = ids.view(B, width)
    return LayerState(pool=pool, block_table=local_bt, seqlens=st.seqlens, W_UK=st.W_UK,
                      W_UV=st.W_UV, num_blocks=max(1, n), max_blocks=max_blocks)


class ShardDecoder:
    """One rank's buffers for a sequence-parallel decode at fixed sizes."""

    def __init__(self, batch: int, q_len: int, max_seqlen: int, world: int, rank: int, device,
                 num_splits: int = 0):
        self.batch, self.q_len, self.max_seqlen = batch, q_len, max_seqlen
        self.world, self.rank = world, rank
        self.num_splits = num_splits
        npages = (max_seqlen + PAGE - 1) // PAGE
        self.page_lo, self.page_hi = shard_pages(npages, world, rank)
        self.sms = num_sms(device)
        self.ws_bytes = xmla.xmla_decode_shard_workspace_size(
            batch, q_len, max_seqlen, self.page_lo, self.page_hi, self.sms, num_splits)
        if self.ws_bytes == 0:
            raise ValueError("unsupported sizes for a sequence-parallel decode")
        self.partial_floats = xmla.xmla_shard_partial_floats(batch, q_len)
        self.workspace = torch.empty(self.ws_bytes, dtype=torch.uint8, device=device)
        self.partial = torch.empty(self.partial_floats, dtype=torch.float32, device=device)
        self.gathered = torch.empty(world * self.partial_floats, dtype=torch.float32,
                                    device=device)
        self.out = torch.empty((batch, q_len, N_HEADS, D_V), dtype=torch.bfloat16, device=device)
        self.status = torch.zeros(1, dtype=torch.int32, device=device)

    def decode_shard(self, cfg, st: LayerState, q: torch.Tensor, softmax_scale: float,
                     stream=None) -> torch.Tensor:
        """Step 1: this rank's merged partial (in self.partial)."""
        xmla.xmla_decode_shard(cfg, q, st.W_UK, st.pool, st.num_blocks, st.block_table,
                               st.max_blocks, st.seqlens, self.batch, self.q_len, self.max_seqlen,
                               softmax_scale, self.page_lo, self.page_hi, self.num_splits,
                               self.workspace, self.ws_bytes, self.status, self.partial, stream)
        return self.partial

    def gather(self, group=None) -> torch.Tensor:
        """Step 2: every rank's partial, rank-major, in self.gathered."""
        if self.world == 1:
            self.gathered.copy_(self.partial)
        else:
            dist.all_gather_into_tensor(self.gathered, self.partial, group=group)
        return self.gathered

    def combine(self, W_UV: torch.Tensor, stream=None) -> torch.Tensor:
        """Step 3: merge of the gathered partials and the W_UV product."""
        xmla.xmla_combine_shards(self.gathered, self.world, W_UV, self.batch, self.q_len, self.out,
                                 stream)
        return self.out

    def decode(self, cfg, st: LayerState, q: torch.Tensor, softmax_scale: float, group=None,
               stream=None) -> torch.Tensor:
        self.decode_shard(cfg, st, q, softmax_scale, stream)
        self.gather(group)
        return self.combine(st.W_UV, stream)


def partial_views(buf: torch.Tensor, batch: int, q_len: int):
    """(O [R, 512], ML [R, 2]) views of one rank's partial, R = batch*q_len*32,
    row index (b*q_len + j)*32 + h."""
    R = batch * q_len * N_HEADS
    return buf[:R * D_LATENT].view(R, D_LATENT), buf[R * D_LATENT:R * (D_LATENT + 2)].view(R, 2)
