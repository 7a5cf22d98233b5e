"""Seeded synthetic inputs for MLA latent-KV decode.

This module only draws random tensors and builds block tables; it holds none
of the attention, RoPE or cache arithmetic.  Both the CUDA path and the CPU
oracle consume exactly the tensors it returns.

Value distributions: q_nope, q_pe, c_kv and k_pe are N(0, 1); W_UK and W_UV are
N(0, 1/512) (variance 1/512).  Every tensor is sampled in float32 from a
seeded torch generator on the requested device and rounded to bf16 (round to
nearest even).  Sequence s of a workload owns ceil(N_s / 64) cache blocks; in
the paged workloads the blocks of all sequences are a seeded random
permutation of the pool, in the contiguous workload block i of the single
sequence is pool block i.

The five workloads follow the Xing4.0-29B-A4B attention shape (32 heads,
latent 512 + rope 64 per token, nope 128, v 128):
  decode_4k       B=1, q_len=1, N=4096, contiguous cache, one layer
  decode_256k     B=1, q_len=1, N=262144, shuffled 64-token pages, one layer
  step_40l_b32    40 layers, B=32, q_len=1, N_s ~ U[8192, 65536], shuffled pages
  verify_q4_b8    B=8, q_len=4 (causal among the 4 new tokens), N=131072, shuffled
  decode_512k_b4  B=4, q_len=1, N=524288 (positions past 262144), shuffled
and one more, outside those five:
  prefill_4k      B=1, a 4096-token prompt attended as one chunk (q_len=4096, N=4096,
                  causal), shuffled pages
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch

N_HEADS = 32
D_NOPE = 128
D_ROPE = 64
D_LATENT = 512
D_V = 128
PAGE = 64


@dataclass
class Workload:
    name: str
    batch: int
    q_len: int
    seqlens: list[int]
    layers: int = 1
    contiguous: bool = False
    seed: int = 1234
    heads: int = N_HEADS

    @property
    def tokens(self) -> int:
        return int(sum(self.seqlens))

    @property
    def max_seqlen(self) -> int:
        return int(max(self.seqlens))

    @property
    def max_blocks(self) -> int:
        return (self.max_seqlen + PAGE - 1) // PAGE

    @property
    def num_blocks(self) -> int:
        return int(sum((n + PAGE - 1) // PAGE for n in self.seqlens))


WORKLOAD_NAMES = ["decode_4k", "decode_256k", "step_40l_b32", "verify_q4_b8", "decode_512k_b4"]
EXTRA_WORKLOADS = ["prefill_4k"]


def workload(index_or_name) -> Workload:
    """The five seeded workloads, by index 0..4 or by name, and the extra ones by name."""
    if index_or_name == "prefill_4k":
        return Workload("prefill_4k", 1, 4096, [4096], seed=1234 + 5)
    idx = WORKLOAD_NAMES.index(index_or_name) if isinstance(index_or_name, str) else int(index_or_name)
    seed = 1234 + idx
    if idx == 0:
        return Workload("decode_4k", 1, 1, [4096], contiguous=True, seed=seed)
    if idx == 1:
        return Workload("decode_256k", 1, 1, [262144], seed=seed)
    if idx == 2:
        g = torch.Generator(device="cpu").manual_seed(seed)
        lens = torch.randint(8192, 65536 + 1, (32,), generator=g).tolist()
        return Workload("step_40l_b32", 32, 1, lens, layers=40, seed=seed)
    if idx == 3:
        return Workload("verify_q4_b8", 8, 4, [131072] * 8, seed=seed)
    if idx == 4:
        return Workload("decode_512k_b4", 4, 1, [524288] * 4, seed=seed)
    raise ValueError(f"unknown workload {index_or_name!r}")


def custom(batch: int, q_len: int, seqlens, *, contiguous: bool = False, seed: int = 7,
           heads: int = N_HEADS, name: str = "custom", layers: int = 1) -> Workload:
    return Workload(name, batch, q_len, list(int(n) for n in seqlens), layers=layers,
                    contiguous=contiguous, seed=seed, heads=heads)


_TENSOR_IDS = {"q": 1, "c_kv": 2, "k_pe": 3, "W_UK": 4, "W_UV": 5, "blocks": 6, "hidden": 7,
               "W_kva": 8}


def _gen(wl: Workload, layer: int, what: str, device) -> torch.Generator:
    s = (wl.seed * 1_000_003 + layer * 10_007 + _TENSOR_IDS[what] * 101) & 0x7FFF_FFFF_FFFF
    return torch.Generator(device=device).manual_seed(s)


def _normal_bf16(shape, std: float, g: torch.Generator, device) -> torch.Tensor:
    x = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    return x.to(torch.bfloat16)


@dataclass
class LayerInputs:
    """One layer's inputs.  Token rows of all sequences are concatenated in
    sequence order; token i of sequence s sits at position i."""

    q: torch.Tensor            # [B, q_len, H, 192] bf16 (q_pe not rotated)
    c_kv: torch.Tensor         # [T, 512] bf16
    k_pe: torch.Tensor         # [T, 64] bf16 (not rotated)
    W_UK: torch.Tensor         # [H, 128, 512] bf16
    W_UV: torch.Tensor         # [H, 512, 128] bf16
    block_table: torch.Tensor  # [B, max_blocks] int32
    seqlens: torch.Tensor      # [B] int32
    seq_ids: torch.Tensor      # [T] int32
    positions: torch.Tensor    # [T] int64
    num_blocks: int
    offsets: list[int] = field(default_factory=list)  # first token row of each sequence


def block_table(wl: Workload, layer: int, device="cpu") -> torch.Tensor:
    nb = wl.num_blocks
    if wl.contiguous:
        perm = torch.arange(nb, dtype=torch.int64)
    else:
        perm = torch.randperm(nb, generator=_gen(wl, layer, "blocks", "cpu"))
    bt = torch.full((wl.batch, wl.max_blocks), -1, dtype=torch.int32)
    k = 0
    for s, n in enumerate(wl.seqlens):
        nbs = (n + PAGE - 1) // PAGE
        bt[s, :nbs] = perm[k:k + nbs].to(torch.int32)
        k += nbs
    return bt.to(device)


def token_index(wl: Workload, device="cpu"):
    """(seq_ids [T] int32, positions [T] int64, offsets) of the concatenated token rows."""
    seq_ids = torch.cat([torch.full((n,), s, dtype=torch.int32) for s, n in enumerate(wl.seqlens)])
    positions = torch.cat([torch.arange(n, dtype=torch.int64) for n in wl.seqlens])
    offsets = [0]
    for n in wl.seqlens[:-1]:
        offsets.append(offsets[-1] + n)
    return seq_ids.to(device), positions.to(device), offsets


def layer_inputs(wl: Workload, layer: int = 0, device="cpu") -> LayerInputs:
    H = wl.heads
    T = wl.tokens
    w_std = D_LATENT ** -0.5
    q = _normal_bf16((wl.batch, wl.q_len, H, D_NOPE + D_ROPE), 1.0, _gen(wl, layer, "q", device), device)
    c_kv = _normal_bf16((T, D_LATENT), 1.0, _gen(wl, layer, "c_kv", device), device)
    k_pe = _normal_bf16((T, D_ROPE), 1.0, _gen(wl, layer, "k_pe", device), device)
    W_UK = _normal_bf16((H, D_NOPE, D_LATENT), w_std, _gen(wl, layer, "W_UK", device), device)
    W_UV = _normal_bf16((H, D_LATENT, D_V), w_std, _gen(wl, layer, "W_UV", device), device)
    seq_ids, positions, offsets = token_index(wl, device)
    return LayerInputs(q=q, c_kv=c_kv, k_pe=k_pe, W_UK=W_UK, W_UV=W_UV,
                       block_table=block_table(wl, layer, device),
                       seqlens=torch.tensor(wl.seqlens, dtype=torch.int32, device=device),
                       seq_ids=seq_ids, positions=positions, num_blocks=wl.num_blocks,
                       offsets=offsets)


def new_token_rows(wl: Workload, offsets) -> list[int]:
    """Row indices (into the concatenated token rows) of each sequence's q_len
    newest tokens: the ones a decode step appends before attending."""
    rows = []
    for s, n in enumerate(wl.seqlens):
        rows.extend(range(offsets[s] + n - wl.q_len, offsets[s] + n))
    return rows


HIDDEN = 3584  # model hidden size: input width of kv_a_proj_with_mqa


def producer_inputs(wl: Workload, layer: int = 0, device="cpu"):
    """Hidden states of each sequence's q_len new tokens [B*q_len, 3584] (N(0,1))
    and the layer's kv_a_proj_with_mqa weight [576, 3584] (N(0, 1/3584)), bf16."""
    hidden = _normal_bf16((wl.batch * wl.q_len, HIDDEN), 1.0, _gen(wl, layer, "hidden", device),
                          device)
    W_kva = _normal_bf16((D_LATENT + D_ROPE, HIDDEN), HIDDEN ** -0.5,
                         _gen(wl, layer, "W_kva", device), device)
    return hidden, W_kva
