"""Device-side state and call sequencing for MLA decode through libxmla.

Holds the caller-owned buffers the C ABI expects (paged latent cache, block
table, sequence lengths, weights, workspace, output) and issues the library
calls in decode order.  No arithmetic of the method happens here.

One decode step over a layer ("the hot path"):
  1. xmla_cache_append of the step's q_len new tokens per sequence, rotating
     their k_pe with YaRN RoPE as it stores [c_kv | rotated k_pe],
  2. xmla_decode (q absorb with RoPE of q_pe -> split-K latent attention ->
     combine with W_UV).
With the 8-bit cache (cache="q8") the same two steps run as
xmla_cache_append_q8 and xmla_decode_q8 over a [num_blocks, 64, 608] byte pool.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch

from . import xmla
from .workloads import (D_LATENT, D_NOPE, D_ROPE, D_V, N_HEADS, PAGE, LayerInputs, Workload,
                        new_token_rows)


def num_sms(device=None) -> int:
    return torch.cuda.get_device_properties(device or torch.cuda.current_device()).multi_processor_count


@dataclass
class LayerState:
    pool: torch.Tensor         # [num_blocks, 64, 576] bf16
    block_table: torch.Tensor  # [B, max_blocks] int32
    seqlens: torch.Tensor      # [B] int32
    W_UK: torch.Tensor
    W_UV: torch.Tensor
    num_blocks: int
    max_blocks: int
    cache: str = "bf16"        # "bf16" or "q8" (pool [num_blocks, 64, 608] uint8)


def new_pool(num_blocks: int, device, fill: float | None = 0.0) -> torch.Tensor:
    if fill is None:
        return torch.empty((num_blocks, PAGE, D_LATENT + D_ROPE), dtype=torch.bfloat16, device=device)
    return torch.full((num_blocks, PAGE, D_LATENT + D_ROPE), fill, dtype=torch.bfloat16, device=device)


Q8_ROW = 608  # bytes of an 8-bit cache row (include/xmla.h)


def new_pool_q8(num_blocks: int, device) -> torch.Tensor:
    return torch.zeros((num_blocks, PAGE, Q8_ROW), dtype=torch.uint8, device=device)


def rope_rows(cfg, x: torch.Tensor, positions: torch.Tensor, stream=None) -> None:
    """Rotate, in place, the rope part of q [R, H, 192] or of k_pe [T, 64]."""
    if x.dim() == 3:
        R, H, D = x.shape
        xmla.xmla_rope_yarn(cfg, x, R, H, D, H * D, D_NOPE, positions, stream)
    else:
        T, D = x.shape
        xmla.xmla_rope_yarn(cfg, x, T, 1, D, D, 0, positions, stream)


@dataclass
class NewTokens:
    """The q_len newest tokens of every sequence: what one decode step appends."""

    c_kv: torch.Tensor       # [B*q_len, 512] bf16
    k_pe: torch.Tensor       # [B*q_len, 64] bf16, not rotated
    positions: torch.Tensor  # [B*q_len] int64
    seq_ids: torch.Tensor    # [B*q_len] int32


def split_prefix(wl: Workload, inp: LayerInputs) -> tuple[LayerInputs, NewTokens]:
    """Split a layer's token rows into the cached prefix and the step's new tokens."""
    T = inp.c_kv.shape[0]
    dev = inp.c_kv.device
    new_rows = torch.tensor(new_token_rows(wl, inp.offsets), dtype=torch.int64, device=dev)
    keep = torch.ones(T, dtype=torch.bool, device=dev)
    keep[new_rows] = False
    prefix = LayerInputs(q=inp.q, c_kv=inp.c_kv[keep], k_pe=inp.k_pe[keep], W_UK=inp.W_UK,
                         W_UV=inp.W_UV, block_table=inp.block_table, seqlens=inp.seqlens,
                         seq_ids=inp.seq_ids[keep], positions=inp.positions[keep],
                         num_blocks=inp.num_blocks, offsets=inp.offsets)
    new = NewTokens(c_kv=inp.c_kv[new_rows].contiguous(), k_pe=inp.k_pe[new_rows].contiguous(),
                    positions=inp.positions[new_rows].contiguous(),
                    seq_ids=inp.seq_ids[new_rows].contiguous())
    return prefix, new


def build_layer(cfg, wl: Workload, inp: LayerInputs, device, chunk: int = 1 << 20,
                pool_fill: float | None = 0.0, status: torch.Tensor | None = None,
                cache: str = "bf16") -> LayerState:
    """Upload one layer's inputs and fill its paged cache with every token of
    every sequence (RoPE on k_pe, then append), in chunks of `chunk` tokens.
    cache="q8": the 8-bit pool, filled through xmla_cache_append_q8."""
    q8 = cache == "q8"
    pool = new_pool_q8(inp.num_blocks, device) if q8 else new_pool(inp.num_blocks, device, pool_fill)
    append = xmla.xmla_cache_append_q8 if q8 else xmla.xmla_cache_append
    bt = inp.block_table.to(device)
    T = inp.c_kv.shape[0]
    for t0 in range(0, T, chunk):
        t1 = min(T, t0 + chunk)
        c = inp.c_kv[t0:t1].to(device, non_blocking=True)
        k = inp.k_pe[t0:t1].to(device, non_blocking=True).contiguous()
        pos = inp.positions[t0:t1].to(device)
        sid = inp.seq_ids[t0:t1].to(device)
        append(pool, inp.num_blocks, bt, bt.shape[1], wl.batch, sid, pos, c, k, cfg, t1 - t0,
               status)
    return LayerState(pool=pool, block_table=bt, seqlens=inp.seqlens.to(device),
                      W_UK=inp.W_UK.to(device), W_UV=inp.W_UV.to(device),
                      num_blocks=inp.num_blocks, max_blocks=bt.shape[1], cache=cache)


class Decoder:
    """Workspace and output buffers for xmla_decode at fixed sizes."""

    def __init__(self, batch: int, q_len: int, max_seqlen: int, device, num_splits: int = 0,
                 cache: str = "bf16"):
        self.batch, self.q_len, self.max_seqlen = batch, q_len, max_seqlen
        self.num_splits = num_splits
        self.cache = cache
        self.sms = num_sms(device)
        ws = xmla.xmla_decode_q8_workspace_size if cache == "q8" else xmla.xmla_decode_workspace_size
        self.ws_bytes = ws(batch, q_len, max_seqlen, self.sms, num_splits)
        if self.ws_bytes == 0:
            raise ValueError("unsupported decode sizes")
        self.workspace = torch.empty(self.ws_bytes, dtype=torch.uint8, device=device)
        self.out = torch.empty((batch, q_len, N_HEADS, D_V), dtype=torch.bfloat16, device=device)
        self.status = torch.zeros(1, dtype=torch.int32, device=device)

    @property
    def splits(self) -> int:
        f = xmla.xmla_decode_q8_num_splits if self.cache == "q8" else xmla.xmla_decode_num_splits
        return f(self.batch, self.q_len, self.max_seqlen, self.sms, self.num_splits)

    def decode(self, cfg, st: LayerState, q: torch.Tensor, softmax_scale: float, out=None,
               stream=None, events=None) -> torch.Tensor:
        """xmla_decode on raw q (q_pe rotated inside); `events` = (start, stop) CUDA
        events recorded around the split-K attention kernel (xmla_decode_profiled)."""
        out = self.out if out is None else out
        ev = events or (None, None)
        f = xmla.xmla_decode_q8_profiled if st.cache == "q8" else xmla.xmla_decode_profiled
        f(cfg, q, st.W_UK, st.W_UV, st.pool, st.num_blocks, st.block_table, st.max_blocks,
          st.seqlens, self.batch, self.q_len, self.max_seqlen, softmax_scale, self.num_splits,
          self.workspace, self.ws_bytes, self.status, out, stream, ev[0], ev[1])
        return out

    def step(self, cfg, st: LayerState, q: torch.Tensor, c_new: torch.Tensor,
             k_new: torch.Tensor, new_pos: torch.Tensor, new_seq: torch.Tensor,
             softmax_scale: float, out=None, stream=None, events=None,
             fused: bool = True) -> torch.Tensor:
        """One decode step on raw q: the q_len newest tokens (c_new, k_new raw)
        are appended with their rope keys rotated, then the layer attends.
        fused=True uses xmla_decode_step (append inside the first kernel);
        fused=False issues xmla_cache_append and then xmla_decode_profiled.  On the
        8-bit cache the append is always its own call (xmla_cache_append_q8)."""
        out = self.out if out is None else out
        if not fused or st.cache == "q8":
            append = xmla.xmla_cache_append_q8 if st.cache == "q8" else xmla.xmla_cache_append
            append(st.pool, st.num_blocks, st.block_table, st.max_blocks, self.batch, new_seq,
                   new_pos, c_new, k_new, cfg, c_new.shape[0], self.status, stream)
            return self.decode(cfg, st, q, softmax_scale, out, stream, events)
        ev = events or (None, None)
        xmla.xmla_decode_step(cfg, q, st.W_UK, st.W_UV, st.pool, st.num_blocks, st.block_table,
                              st.max_blocks, st.seqlens, self.batch, self.q_len, self.max_seqlen,
                              new_seq, new_pos, c_new, k_new, c_new.shape[0], softmax_scale,
                              self.num_splits, self.workspace, self.ws_bytes, self.status, out,
                              stream, ev[0], ev[1])
        return out

    def step_from_hidden(self, cfg, st: LayerState, q: torch.Tensor, hidden: torch.Tensor,
                         W_kva: torch.Tensor, new_pos: torch.Tensor, new_seq: torch.Tensor,
                         softmax_scale: float, out=None, stream=None, events=None,
                         bias: torch.Tensor | None = None) -> torch.Tensor:
        """One decode step from the new tokens' hidden states: their cache rows
        are produced (kv_a_proj_with_mqa, RoPE, append), then the layer attends."""
        out = self.out if out is None else out
        ev = events or (None, None)
        xmla.xmla_decode_step_from_hidden(cfg, q, st.W_UK, st.W_UV, hidden, W_kva, bias, st.pool,
                                          st.num_blocks, st.block_table, st.max_blocks,
                                          st.seqlens, self.batch, self.q_len, self.max_seqlen,
                                          new_seq, new_pos, hidden.shape[0], softmax_scale,
                                          self.num_splits, self.workspace, self.ws_bytes,
                                          self.status, out, stream, ev[0], ev[1])
        return out

    def check_status(self) -> int:
        return int(self.status.item())
