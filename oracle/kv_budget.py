"""KV-cache size arithmetic of the pages (TEST INFRASTRUCTURE ONLY).

[P1] "256K 长上下文真能本地用：Xing4.0 原生长上下文的工程代价拆解", section 二
"KV Cache 显存账本": per token and layer the MLA cache of that estimate holds the
512-dim latent plus the 128-dim V (640 bf16 = 1280 B; x40 layers = 51200 B);
the MHA comparison stores K and V for 32 heads x 192 dims.  Its table rounds
half up to one decimal (to integers at three digits).  The MLA column counts
K as 1024 and reports GiB; the MHA column counts K as 1000 up to 128K and as
1024 at 256K, also in GiB -- each column is reproduced in its own convention.

The decode path of this repository caches [c_kv 512 | k_pe 64] = 576 bf16
per token and layer ([P5] MLA section: the latent plus the 64-dim rope key).

Other pages give the same arithmetic for other models and are used as extra
checks of the generic formula:
  [P2] Swift-Qwen3.8-27B GGUF page: 16 layers x 4 KV heads x 256 x 2 x 2 B.
  [P3] "别把上下文开满：3.0 Flash 256K 最稳背后的设置避坑": 18 layers x 4 heads
       x 2 x 256 x 2 B, GB in decimal units with K = 1024.
"""
from __future__ import annotations

from decimal import ROUND_HALF_UP, Decimal

GiB = 1024 ** 3
GB = 1000 ** 3


def kv_bytes_per_token(elems_per_layer: int, layers: int, bytes_per_elem: int = 2) -> int:
    return elems_per_layer * layers * bytes_per_elem


def mla_elems_page_estimate(kv_lora_rank: int = 512, v_head_dim: int = 128) -> int:
    """[P1] section 二: latent plus decompressed V per token and layer."""
    return kv_lora_rank + v_head_dim


def mla_elems_latent_rope(kv_lora_rank: int = 512, qk_rope_head_dim: int = 64) -> int:
    """The cache this repository's decode path reads: [c_kv | k_pe]."""
    return kv_lora_rank + qk_rope_head_dim


def mha_elems(heads: int = 32, head_dim: int = 128 + 64) -> int:
    """[P1] section 二 MHA comparison: K and V for every head, 192 dims each."""
    return heads * head_dim * 2


def gqa_elems(kv_heads: int, head_dim: int) -> int:
    return kv_heads * head_dim * 2


def cache_bytes(tokens: int, per_token_bytes: int) -> int:
    return tokens * per_token_bytes


def round_half_up(x: float, digits: int) -> float:
    q = Decimal(1).scaleb(-digits)
    return float(Decimal(repr(x)).quantize(q, rounding=ROUND_HALF_UP))


def as_units(n_bytes: int, unit: int, digits: int) -> float:
    return round_half_up(n_bytes / unit, digits)


def tokens_fitting(budget_bytes: float, per_token_bytes: int) -> int:
    """Whole tokens of cache that fit in a byte budget."""
    return int(budget_bytes // per_token_bytes)
