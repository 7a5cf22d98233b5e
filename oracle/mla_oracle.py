"""fp64 CPU oracle for MLA latent-KV decode with YaRN RoPE.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import, call or
execute this module; only the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` use it.  It shares no code, table or constant
generator with the CUDA library.

Sources (web pages, cited by title and section):
  [P1] "256K 长上下文真能本地用：Xing4.0 原生长上下文的工程代价拆解"
       (lpnh.cn/news/2764750), section 一 "256K的规格真相" (the config.json
       excerpt: rope_scaling = yarn, factor 64, original 4096, beta_fast 32,
       beta_slow 1, mscale = mscale_all_dim = 1.0, kv_lora_rank 512,
       v_head_dim 128, attention_bias false; "attention logit 缩放") and
       section 二 "KV Cache 显存账本" (32 heads, qk_nope 128 + qk_rope 64).
  [P5] "mHC+MLA+MTP 是什么？拆开给 Agent 用的百亿 MoE"
       (hotelren.com/news/5507480), section "MLA：256K 上下文的'内存革命'"
       (the Xing4_0Attention field list: kv_a_proj_with_mqa -> 512 + 64,
       kv_b_proj: 512 -> heads*(128 + 128); K and V are expanded from the
       latent by kv_b_proj at attention time; yarn_get_mscale corrects the
       attention scale).

Where the pages are silent the oracle takes these readings (each is listed
with its reason in the design notes of the repository):
  * rope_theta is not printed; it is a parameter, default 10000.
  * The YaRN frequency construction is not printed; the oracle follows the
    "NTK-by-parts" interpolation of the YaRN paper (Peng, Quesnelle, Fan,
    Shippole 2023, section 3.2): dimensions that turn more than beta_fast
    times over the original context keep their frequency, dimensions that
    turn fewer than beta_slow times are divided by the scale factor, and a
    linear ramp blends the band between.  The band edges are the
    correction dimensions rounded outward (floor / ceil) and clipped.
  * RoPE pairs dimension i with i + 32 of the 64-dim rope part (rotate-half).
  * cos/sin carry the factor mscale(s, mscale) / mscale(s, mscale_all_dim);
    the softmax scale is (qk_nope + qk_rope)^-1/2 * mscale(s, mscale_all_dim)^2.
  * kv_b_proj output rows [256h, 256h+128) are head h's K_nope rows (W_UK[h],
    shape [128, 512]) and rows [256h+128, 256h+256) its V rows; W_UV[h] is
    their transpose, shape [512, 128].  No bias (attention_bias false).
  * kv_a_proj_with_mqa ([P5] MLA section: Linear(hidden_size, 512 + 64);
    hidden_size 3584 from the model summary page "Xing4.0" (alphasignal.ai),
    architecture paragraph) has no bias (attention_bias false) and no norm
    is printed between it and the cache: output columns [0, 512) are c_kv,
    [512, 576) the raw rope key, each rounded to bf16 as a bf16 Linear does
    before RoPE and caching.
  * A context of N tokens holds positions 0..N-1 and includes the q_len new
    tokens, which are its last q_len entries; query j sits at position
    N - q_len + j and sees tokens t <= N - q_len + j.

All arithmetic is float64 on the values it is given (bf16 inputs are widened
exactly by the caller).  Library primitives used: numpy matmul, exp, sin, cos.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np

# Model shape, [P5] MLA section field list and [P1] section 二.
N_HEADS = 32
D_NOPE = 128
D_ROPE = 64
D_LATENT = 512
D_V = 128
PAGE = 64  # tokens per cache block (paged-cache granularity of the decode path)


@dataclass(frozen=True)
class YarnConfig:
    """rope_scaling block of [P1] section 一; rope_theta is not on the pages."""

    rope_theta: float = 10000.0
    factor: float = 64.0
    original_max_position_embeddings: int = 4096
    beta_fast: float = 32.0
    beta_slow: float = 1.0
    mscale: float = 1.0
    mscale_all_dim: float = 1.0
    rotary_dim: int = D_ROPE


def yarn_get_mscale(scale: float, mscale: float) -> float:
    """Attention-magnitude correction named yarn_get_mscale in [P5] (MLA section).

    YaRN (Peng et al. 2023, section 3.4) scales attention by 0.1 ln(s) + 1 for a
    context extension factor s > 1; the mscale field multiplies the log term.
    """
    if scale <= 1.0:
        return 1.0
    return 0.1 * mscale * math.log(scale) + 1.0


def yarn_correction_dim(num_rotations: float, dim: int, base: float, max_pos: int) -> float:
    """Dimension index (in units of rotary pairs scaled to dim) whose wavelength
    turns exactly ``num_rotations`` times over ``max_pos`` positions.

    Pair i has frequency base^(-2i/dim), i.e. it turns max_pos*base^(-2i/dim)/(2 pi)
    times over the original context; solving for i gives this value.
    """
    return dim * math.log(max_pos / (num_rotations * 2.0 * math.pi)) / (2.0 * math.log(base))


def yarn_band(cfg: YarnConfig) -> tuple[float, float]:
    """Ramp edges (low, high) of the NTK-by-parts blend, rounded outward."""
    d = cfg.rotary_dim
    low = math.floor(yarn_correction_dim(cfg.beta_fast, d, cfg.rope_theta,
                                         cfg.original_max_position_embeddings))
    high = math.ceil(yarn_correction_dim(cfg.beta_slow, d, cfg.rope_theta,
                                         cfg.original_max_position_embeddings))
    low = max(low, 0)
    high = min(high, d - 1)
    if low == high:
        high = high + 0.001  # avoid a zero-width ramp
    return float(low), float(high)


def yarn_inv_freq(cfg: YarnConfig) -> np.ndarray:
    """float64 [rotary_dim/2] inverse frequencies after YaRN interpolation."""
    d = cfg.rotary_dim
    i = np.arange(d // 2, dtype=np.float64)
    base_freq = cfg.rope_theta ** (-(2.0 * i) / d)        # textbook RoPE
    if cfg.factor == 1.0:
        return base_freq
    low, high = yarn_band(cfg)
    ramp = np.clip((i - low) / (high - low), 0.0, 1.0)    # 0 keep, 1 interpolate
    return base_freq / cfg.factor * ramp + base_freq * (1.0 - ramp)


def cos_sin_factor(cfg: YarnConfig) -> float:
    """Magnitude applied to cos/sin: mscale(s, mscale) / mscale(s, mscale_all_dim)."""
    return yarn_get_mscale(cfg.factor, cfg.mscale) / yarn_get_mscale(cfg.factor, cfg.mscale_all_dim)


def softmax_scale(cfg: YarnConfig, qk_head_dim: int = D_NOPE + D_ROPE) -> float:
    """Logit scale: qk_head_dim^-1/2 times mscale(s, mscale_all_dim) squared.

    [P1] section 一 says the YaRN alignment includes an attention-logit scaling,
    and [P5] names yarn_get_mscale as the attention-scale correction.
    """
    m = yarn_get_mscale(cfg.factor, cfg.mscale_all_dim)
    return qk_head_dim ** -0.5 * m * m


def rope(x: np.ndarray, positions: np.ndarray, cfg: YarnConfig) -> np.ndarray:
    """Rotate the last axis (rotary_dim wide) of x at the given integer positions.

    x: [..., rotary_dim]; positions: broadcastable to x.shape[:-1] (int64).
    Pair (i, i + d/2) is rotated by angle position * inv_freq[i], computed in
    float64 on the exact integer position.
    """
    x = np.asarray(x, dtype=np.float64)
    half = cfg.rotary_dim // 2
    inv_freq = yarn_inv_freq(cfg)
    ang = np.asarray(positions, dtype=np.int64)[..., None].astype(np.float64) * inv_freq
    f = cos_sin_factor(cfg)
    c = np.cos(ang) * f
    s = np.sin(ang) * f
    x1 = x[..., :half]
    x2 = x[..., half:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


def _query_positions(seqlen: int, q_len: int) -> np.ndarray:
    return np.arange(seqlen - q_len, seqlen, dtype=np.int64)


def mla_attention_expanded(q: np.ndarray, c_kv: np.ndarray, k_pe: np.ndarray,
                           W_UK: np.ndarray, W_UV: np.ndarray,
                           cfg: YarnConfig) -> np.ndarray:
    """The definition: expand K and V per head from the latent, then attention.

    One sequence.  q: [q_len, H, D_NOPE + D_ROPE] (q_pe not yet rotated);
    c_kv: [N, 512]; k_pe: [N, 64] (not yet rotated; token t sits at position t);
    W_UK: [H, 128, 512]; W_UV: [H, 512, 128].  Returns [q_len, H, 128] float64.

    For each head h ([P5] MLA section: kv_b_proj expands K and V from the
    cached latent):  K_nope = c_kv W_UK[h]^T,  V = c_kv W_UV[h],
    K = [K_nope | rope(k_pe)],  Q = [q_nope | rope(q_pe)],
    P = softmax(scale * Q K^T) over the causally visible tokens,  out = P V.
    """
    q = np.asarray(q, dtype=np.float64)
    c_kv = np.asarray(c_kv, dtype=np.float64)
    k_pe = np.asarray(k_pe, dtype=np.float64)
    W_UK = np.asarray(W_UK, dtype=np.float64)
    W_UV = np.asarray(W_UV, dtype=np.float64)
    q_len, H, _ = q.shape
    N = c_kv.shape[0]
    scale = softmax_scale(cfg, q.shape[-1])
    qpos = _query_positions(N, q_len)
    k_rot = rope(k_pe, np.arange(N, dtype=np.int64), cfg)              # [N, 64]
    q_nope = q[..., :D_NOPE]
    q_rot = rope(q[..., D_NOPE:], qpos[:, None], cfg)                  # [q_len, H, 64]
    visible = np.arange(N)[None, :] <= qpos[:, None]                   # [q_len, N]
    out = np.empty((q_len, H, W_UV.shape[-1]), dtype=np.float64)
    for h in range(H):
        K_nope = c_kv @ W_UK[h].T                                       # [N, 128]
        V = c_kv @ W_UV[h]                                              # [N, 128]
        K = np.concatenate([K_nope, k_rot], axis=1)                     # [N, 192]
        Q = np.concatenate([q_nope[:, h, :], q_rot[:, h, :]], axis=1)   # [q_len, 192]
        S = scale * (Q @ K.T)                                           # [q_len, N]
        S = np.where(visible, S, -np.inf)
        S = S - S.max(axis=1, keepdims=True)
        P = np.exp(S)
        P = P / P.sum(axis=1, keepdims=True)
        out[:, h, :] = P @ V
    return out


def mla_attention_probs(q: np.ndarray, c_kv: np.ndarray, k_pe: np.ndarray,
                        W_UK: np.ndarray, cfg: YarnConfig) -> np.ndarray:
    """Softmax probabilities [q_len, H, N] of the expanded definition."""
    q = np.asarray(q, dtype=np.float64)
    c_kv = np.asarray(c_kv, dtype=np.float64)
    W_UK = np.asarray(W_UK, dtype=np.float64)
    q_len, H, _ = q.shape
    N = c_kv.shape[0]
    scale = softmax_scale(cfg, q.shape[-1])
    qpos = _query_positions(N, q_len)
    k_rot = rope(k_pe, np.arange(N, dtype=np.int64), cfg)
    q_rot = rope(q[..., D_NOPE:], qpos[:, None], cfg)
    visible = np.arange(N)[None, :] <= qpos[:, None]
    probs = np.empty((q_len, H, N), dtype=np.float64)
    for h in range(H):
        K = np.concatenate([c_kv @ W_UK[h].T, k_rot], axis=1)
        Q = np.concatenate([q[:, h, :D_NOPE], q_rot[:, h, :]], axis=1)
        S = np.where(visible, scale * (Q @ K.T), -np.inf)
        S = S - S.max(axis=1, keepdims=True)
        P = np.exp(S)
        probs[:, h, :] = P / P.sum(axis=1, keepdims=True)
    return probs


def mla_attention_absorbed(q: np.ndarray, c_kv: np.ndarray, k_pe_rot: np.ndarray,
                           W_UK: np.ndarray, W_UV: np.ndarray,
                           cfg: YarnConfig) -> np.ndarray:
    """Weight-absorbed form of the same attention (one sequence).

    Moves W_UK onto the query and W_UV after the probability-weighted latent
    sum:  q_lat = W_UK[h]^T q_nope,  S = scale (q_lat . c_kv + rope(q_pe) . k_pe_rot),
    o_lat = sum_t P c_kv[t],  out = W_UV[h]^T o_lat.  Here k_pe_rot is the
    already-rotated cached rope key (as the latent cache stores it).
    Returns [q_len, H, 128] float64.
    """
    q = np.asarray(q, dtype=np.float64)
    c_kv = np.asarray(c_kv, dtype=np.float64)
    k_pe_rot = np.asarray(k_pe_rot, dtype=np.float64)
    W_UK = np.asarray(W_UK, dtype=np.float64)
    W_UV = np.asarray(W_UV, dtype=np.float64)
    q_len, H, _ = q.shape
    N = c_kv.shape[0]
    scale = softmax_scale(cfg, q.shape[-1])
    qpos = _query_positions(N, q_len)
    q_rot = rope(q[..., D_NOPE:], qpos[:, None], cfg)                       # [q_len, H, 64]
    q_lat = np.einsum("jhd,hdc->jhc", q[..., :D_NOPE], W_UK)                # [q_len, H, 512]
    S = scale * (q_lat.reshape(q_len * H, -1) @ c_kv.T
                 + q_rot.reshape(q_len * H, -1) @ k_pe_rot.T)               # [q_len*H, N]
    visible = np.repeat(np.arange(N)[None, :] <= qpos[:, None], H, axis=0)
    S = np.where(visible, S, -np.inf)
    S = S - S.max(axis=1, keepdims=True)
    P = np.exp(S)
    P = P / P.sum(axis=1, keepdims=True)
    o_lat = (P @ c_kv).reshape(q_len, H, -1)                                # [q_len, H, 512]
    return np.einsum("jhc,hcv->jhv", o_lat, W_UV)


def attention_partial(q: np.ndarray, c_kv: np.ndarray, k_pe_rot: np.ndarray,
                      W_UK: np.ndarray, cfg: YarnConfig, seqlen: int, t_lo: int,
                      t_hi: int) -> tuple[np.ndarray, np.ndarray, np.ndarray]:
    """The absorbed attention of one sequence over its cached tokens [t_lo, t_hi) only.

    [P5] MLA section: the output is a softmax-weighted sum over the cached
    latent rows; restricted to a subset of tokens it is described exactly by
    (m, l, O): m the largest visible score of the subset, l = sum exp(S - m),
    O = sum exp(S - m) c_kv[t] (natural-log units, scores S as in
    mla_attention_absorbed).  q: [q_len, H, 192] (q_pe not rotated); c_kv,
    k_pe_rot: rows [t_lo, t_hi) of the sequence ([t_hi - t_lo, 512] / [.., 64]);
    seqlen: the sequence's full length (query j at seqlen - q_len + j).
    Rows that see no token of the subset get m = -inf, l = 0, O = 0.
    Returns m [q_len, H], l [q_len, H], O [q_len, H, 512].
    """
    q = np.asarray(q, dtype=np.float64)
    c_kv = np.asarray(c_kv, dtype=np.float64)
    k_pe_rot = np.asarray(k_pe_rot, dtype=np.float64)
    W_UK = np.asarray(W_UK, dtype=np.float64)
    q_len, H, _ = q.shape
    scale = softmax_scale(cfg, q.shape[-1])
    qpos = _query_positions(seqlen, q_len)
    q_rot = rope(q[..., D_NOPE:], qpos[:, None], cfg)
    q_lat = np.einsum("jhd,hdc->jhc", q[..., :D_NOPE], W_UK)
    S = scale * (q_lat.reshape(q_len * H, -1) @ c_kv.T
                 + q_rot.reshape(q_len * H, -1) @ k_pe_rot.T)        # [q_len*H, n]
    tpos = np.arange(t_lo, t_hi)
    visible = np.repeat(tpos[None, :] <= qpos[:, None], H, axis=0)
    S = np.where(visible, S, -np.inf)
    m = S.max(axis=1) if S.shape[1] > 0 else np.full(q_len * H, -np.inf)
    E = np.where(visible, np.exp(S - np.where(np.isfinite(m), m, 0.0)[:, None]), 0.0)
    l = E.sum(axis=1)
    O = E @ c_kv
    return m.reshape(q_len, H), l.reshape(q_len, H), O.reshape(q_len, H, -1)


def merge_partials(parts) -> tuple[np.ndarray, np.ndarray, np.ndarray]:
    """Exact merge of partials (m, l, O) of disjoint token subsets of one sequence.

    With M = max m_i over parts that saw a token: l = sum exp(m_i - M) l_i and
    O = sum exp(m_i - M) O_i (the log-sum-exp combination of softmax sums).
    """
    parts = list(parts)
    ms = np.stack([np.asarray(p[0], dtype=np.float64) for p in parts])
    ls = np.stack([np.asarray(p[1], dtype=np.float64) for p in parts])
    Os = np.stack([np.asarray(p[2], dtype=np.float64) for p in parts])
    seen = ls > 0
    M = np.where(seen, ms, -np.inf).max(axis=0)
    w = np.where(seen, np.exp(np.where(seen, ms, 0.0) - np.where(np.isfinite(M), M, 0.0)), 0.0)
    return M, (w * ls).sum(axis=0), (w[..., None] * Os).sum(axis=0)


def finish_partial(m: np.ndarray, l: np.ndarray, O: np.ndarray, W_UV: np.ndarray) -> np.ndarray:
    """Output of a complete partial: out[j, h] = W_UV[h]^T (O[j, h] / l[j, h]).
    Returns [q_len, H, 128]; rows with l = 0 give 0."""
    o_lat = np.where(l[..., None] > 0, O / np.where(l > 0, l, 1.0)[..., None], 0.0)
    return np.einsum("jhc,hcv->jhv", o_lat, np.asarray(W_UV, dtype=np.float64))


HIDDEN = 3584  # model hidden size (the summary page's architecture paragraph)


def kv_a_projection(hidden: np.ndarray, W_kva: np.ndarray,
                    bias: np.ndarray | None = None) -> tuple[np.ndarray, np.ndarray]:
    """kv_a_proj_with_mqa of token hidden states, before any rounding.

    [P5] MLA section: kv_a_proj_with_mqa = Linear(hidden_size,
    kv_lora_rank + qk_rope_head_dim) compresses each token into the 512-dim
    latent and the 64-dim (not yet rotated) rope key.  hidden: [T, HIDDEN];
    W_kva: [576, HIDDEN] (Linear weight layout: output x input); bias: [576]
    or None.  Returns (c_kv [T, 512], k_pe [T, 64]) in float64.
    """
    out = np.asarray(hidden, dtype=np.float64) @ np.asarray(W_kva, dtype=np.float64).T
    if bias is not None:
        out = out + np.asarray(bias, dtype=np.float64)
    return out[:, :D_LATENT], out[:, D_LATENT:]


def cache_append(pool_u16: np.ndarray, block_table: np.ndarray, seq_ids: np.ndarray,
                 positions: np.ndarray, c_kv_u16: np.ndarray, k_pe_rot_u16: np.ndarray) -> None:
    """Bit copy of token rows [c_kv | k_pe_rot] into a paged pool (in place).

    pool_u16: [num_blocks, PAGE, 576] uint16 (bf16 bit patterns);
    block_table: [B, max_blocks] int; token i of sequence seq_ids[i] at
    position positions[i] goes to block block_table[seq, pos // PAGE], row
    pos % PAGE.  [P1] section 二: the latent cache holds, per token and layer,
    the compressed latent; [P5]: the latent plus the 64-dim rope key.
    """
    for i in range(len(positions)):
        b = int(seq_ids[i])
        p = int(positions[i])
        blk = int(block_table[b, p // PAGE])
        pool_u16[blk, p % PAGE, :D_LATENT] = c_kv_u16[i]
        pool_u16[blk, p % PAGE, D_LATENT:] = k_pe_rot_u16[i]


def gather_sequence(pool: np.ndarray, block_table_row: np.ndarray, seqlen: int) -> np.ndarray:
    """Logical token rows [seqlen, 576] of one sequence, read through its block table."""
    rows = [pool[int(block_table_row[t // PAGE]), t % PAGE] for t in range(seqlen)]
    return np.stack(rows, axis=0) if rows else np.zeros((0, pool.shape[-1]), dtype=pool.dtype)


def mla_decode_from_pool(q: np.ndarray, pool: np.ndarray, block_table: np.ndarray,
                         seqlens: np.ndarray, W_UK: np.ndarray, W_UV: np.ndarray,
                         cfg: YarnConfig) -> np.ndarray:
    """Absorbed-form decode of a batch read through the paged cache.

    q: [B, q_len, H, 192] (q_pe not rotated); pool: [num_blocks, PAGE, 576]
    holding [c_kv | rotated k_pe] as float values; block_table: [B, max_blocks];
    seqlens: [B] (each includes its q_len new tokens).  Returns [B, q_len, H, 128].
    """
    B = q.shape[0]
    out = np.empty(q.shape[:3] + (W_UV.shape[-1],), dtype=np.float64)
    for b in range(B):
        rows = gather_sequence(pool, block_table[b], int(seqlens[b])).astype(np.float64)
        out[b] = mla_attention_absorbed(q[b], rows[:, :D_LATENT], rows[:, D_LATENT:],
                                        W_UK, W_UV, cfg)
    return out


# ---------------------------------------------------------------- 8-bit latent cache
#
# [P1] section 三, 方案 A: a q8_0 KV cache ("--cache-type-k q8_0") halves the
# bf16 cache bytes at a small precision cost.  The pages name the format only:
# 8-bit codes with one scale per block of 32 values.  Reading taken here: the
# 576 values of a cache row ([c_kv | rotated k_pe]) in 18 blocks of 32; each
# block keeps a power-of-two scale 2^e, e the smallest integer with
# 127 * 2^e >= the block's largest magnitude, clamped to [Q8_EMIN, Q8_EMAX];
# codes are x / 2^e rounded to nearest (ties to even) and clamped to
# [-127, 127].  A power of two (rather than q8_0's free fp16 scale) keeps every
# dequantised value code * 2^e exact in fp16 and bf16, so the cache holds
# exactly the values the attention consumes.

Q8_BLOCK = 32                # values per scale block
Q8_BLOCKS = (D_LATENT + D_ROPE) // Q8_BLOCK   # 18 blocks per cache row
Q8_EMIN, Q8_EMAX = -14, 8    # scale exponent range


def q8_block_exponent(amax: np.ndarray) -> np.ndarray:
    """Smallest e with 127 * 2^e >= amax, clamped to [Q8_EMIN, Q8_EMAX].

    Exact: with amax = m * 2^k (m in [0.5, 1)), 127 * 2^(k-7) = (127/128) 2^k is
    enough iff m <= 127/128, and 127 * 2^(k-6) > 2^k always is.
    """
    amax = np.asarray(amax, dtype=np.float64)
    m, k = np.frexp(amax)
    e = np.where(m > 127.0 / 128.0, k - 6, k - 7)
    e = np.where(amax > 0, e, Q8_EMIN)
    return np.clip(e, Q8_EMIN, Q8_EMAX).astype(np.int64)


def q8_quantize(rows: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """Quantise cache rows [..., 576] -> (codes int8 [..., 576], exps int8 [..., 18])."""
    x = np.asarray(rows, dtype=np.float64)
    xb = x.reshape(x.shape[:-1] + (Q8_BLOCKS, Q8_BLOCK))
    e = q8_block_exponent(np.max(np.abs(xb), axis=-1))
    codes = np.clip(np.rint(xb / np.exp2(e.astype(np.float64))[..., None]), -127, 127)
    return codes.reshape(x.shape).astype(np.int8), e.astype(np.int8)


def q8_dequantize(codes: np.ndarray, exps: np.ndarray) -> np.ndarray:
    """Values code * 2^e of quantised rows, float64 [..., 576]."""
    c = np.asarray(codes, dtype=np.float64)
    cb = c.reshape(c.shape[:-1] + (Q8_BLOCKS, Q8_BLOCK))
    scale = np.exp2(np.asarray(exps, dtype=np.float64))[..., None]
    return (cb * scale).reshape(c.shape)
