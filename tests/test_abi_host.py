"""Host-side checks of libxmla that need no GPU: it loads, exports every
symbol include/xmla.h declares, and its host logic (YaRN table, scale,
workspace plan, argument validation) behaves as documented."""
import ctypes
import os
import re

import numpy as np
import pytest

from mla_latent_kv_yarn_b200 import build as xbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def x():
    xbuild.build()
    from mla_latent_kv_yarn_b200 import xmla
    return xmla


def _declared_functions():
    src = open(os.path.join(ROOT, "include", "xmla.h"), encoding="utf-8").read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(xmla_[a-z0-9_]+)\s*\(", src)))


def test_library_exports_every_declared_symbol(x):
    declared = _declared_functions()
    assert "xmla_decode" in declared and "xmla_cache_append" in declared
    L = x.lib()
    for name in declared:
        assert hasattr(L, name), name
    assert sorted(x.EXPORTS) == declared


def test_default_config_and_scale(x):
    cfg = x.xmla_yarn_default()
    assert (cfg.rope_theta, cfg.factor, cfg.original_max_position_embeddings) == (10000.0, 64.0, 4096)
    assert (cfg.beta_fast, cfg.beta_slow, cfg.mscale, cfg.mscale_all_dim, cfg.rotary_dim) == \
        (32.0, 1.0, 1.0, 1.0, 64)
    assert x.xmla_softmax_scale(cfg, 192) == pytest.approx(0.14467962580268923, rel=1e-15)


@pytest.mark.parametrize("theta,factor", [(1e4, 64.0), (1e7, 64.0), (1e4, 1.0), (5e5, 32.0)])
def test_yarn_table_matches_oracle(x, theta, factor):
    from oracle import mla_oracle as om
    cfg = x.xmla_yarn_default()
    cfg.rope_theta = theta
    cfg.factor = factor
    got = np.array(x.xmla_yarn_inv_freq(cfg))
    want = om.yarn_inv_freq(om.YarnConfig(rope_theta=theta, factor=factor))
    assert np.allclose(got, want, rtol=1e-14, atol=0)


def test_workspace_plan(x):
    # 256K context, batch 1, 148 SMs: one split per SM (at least two pages each)
    assert x.xmla_decode_num_splits(1, 1, 262144, 148) == 148
    assert x.xmla_decode_num_splits(1, 1, 128, 148) == 1          # two pages -> one split
    assert x.xmla_decode_num_splits(4, 1, 524288, 148) == 37
    assert x.xmla_decode_num_splits(8, 4, 131072, 148) == 9       # 16 (seq, row group) units
    assert x.xmla_decode_num_splits(1, 1, 4096, 148, 5) == 5      # forced
    ws = x.xmla_decode_workspace_size(1, 1, 262144, 148)
    # q_ext (32 x 576 bf16) + partial O (148 x 32 x 512 fp32) + (m, l), 1 KiB aligned pieces
    assert ws >= 148 * 32 * 512 * 4 + 148 * 32 * 8 + 32 * 576 * 2
    assert ws % 1024 == 0
    assert x.xmla_decode_workspace_size(1, 65537, 70000, 148) == 0  # q_len > 65536
    assert x.xmla_decode_workspace_size(1, 4096, 4096, 148) > 0     # a prefill chunk
    assert x.xmla_decode_workspace_size(0, 1, 4096, 148) == 0
    assert x.xmla_decode_workspace_size(1, 4, 3, 148) == 0         # max_seqlen < q_len
    # the 8-bit cache: 32 rows per CTA at any q_len <= 8, one f16 query row each
    assert x.xmla_decode_q8_num_splits(1, 1, 262144, 148) == 148
    assert x.xmla_decode_q8_num_splits(8, 4, 131072, 148) == 4     # 32 (seq, query) units
    assert x.xmla_decode_q8_workspace_size(1, 1, 262144, 148) == ws
    assert x.xmla_decode_q8_workspace_size(1, 8, 4096, 148) > 0
    assert x.xmla_decode_q8_workspace_size(1, 9, 4096, 148) == 0   # q_len > 8


def test_argument_validation_without_gpu(x):
    L = x.lib()
    cfg = x.xmla_yarn_default()
    # null data pointers are rejected before any CUDA call
    st = L.xmla_decode(ctypes.byref(cfg), None, None, None, None, 1, None, 1, None, 1, 1, 64, 0.1,
                       0, None, 0, None, None, None)
    assert st == 1
    st = L.xmla_decode(None, None, None, None, None, 1, None, 1, None, 1, 1, 64, 0.1, 0, None, 0,
                       None, None, None)
    assert st == 1
    assert L.xmla_rope_yarn(ctypes.byref(cfg), None, 5, 1, 64, 64, 0, None, None) == 1
    assert L.xmla_rope_yarn(ctypes.byref(cfg), None, 0, 1, 64, 64, 0, None, None) == 0  # no-op
    bad = x.xmla_yarn_default()
    bad.rotary_dim = 32
    assert L.xmla_rope_yarn(ctypes.byref(bad), None, 1, 1, 64, 64, 0, None, None) == 2
    assert L.xmla_cache_append(None, 4, None, 1, 1, None, None, None, None, None, 0, None, None) == 0
    assert L.xmla_cache_append(None, 4, None, 1, 1, None, None, None, None, None, 3, None, None) == 1
    assert L.xmla_cache_append_q8(None, 4, None, 1, 1, None, None, None, None, None, 0, None,
                                  None) == 0
    assert L.xmla_cache_append_q8(None, 4, None, 1, 1, None, None, None, None, None, 3, None,
                                  None) == 1
    st = L.xmla_decode_q8(ctypes.byref(cfg), None, None, None, None, 1, None, 1, None, 1, 1, 64,
                          0.1, 0, None, 0, None, None, None)
    assert st == 1
    assert L.xmla_selftest_wait_timeout(None, 1000, None) == 1
    for code in range(8):
        assert x.xmla_status_string(code)


def test_row_counts_beyond_int32_are_rejected(x):
    L = x.lib()
    # batch * q_len * 32 (query rows times heads) must stay below 2^31
    assert x.xmla_decode_workspace_size(1 << 16, 1024, 65536, 148) == 0   # 2^31 exactly
    assert x.xmla_decode_workspace_size((1 << 16) - 1, 1024, 65536, 148) > 0
    assert x.xmla_decode_q8_workspace_size(1 << 28, 8, 4096, 148) == 0
    # the shard combine checks the same bound before touching any pointer
    fake = ctypes.c_void_p(256)
    assert L.xmla_combine_shards(fake, 2, fake, 1 << 16, 1024, fake, None) == 2


def test_prompt_chunk_workspace_covers_the_non_absorbed_path(x):
    # From 64 new tokens a chunk runs the non-absorbed form: the workspace holds
    # the fp16 queries [rows, 32, 192], K_nope and V [B * s_pad, 32, 128] each and
    # the rope key [B * s_pad, 64] (s_pad = max_seqlen rounded up to 128), each
    # piece 1 KiB aligned.  Below 64 tokens the absorbed form's smaller plan.
    def prefill_bytes(batch, q_len, max_seqlen):
        up = lambda v: (v + 1023) // 1024 * 1024
        s_pad = (max_seqlen + 127) // 128 * 128
        kx = up(batch * q_len * 32 * 192 * 2)
        vx = up(kx + batch * s_pad * 32 * 128 * 2)
        kp = up(vx + batch * s_pad * 32 * 128 * 2)
        return up(kp + batch * s_pad * 64 * 2)
    for batch, q_len, n in [(1, 64, 4096), (1, 4096, 4096), (3, 100, 5000), (2, 128, 129)]:
        assert x.xmla_decode_workspace_size(batch, q_len, n, 148) >= prefill_bytes(batch, q_len, n)
    # one token fewer: the absorbed plan, which needs no expanded K/V
    assert x.xmla_decode_workspace_size(1, 63, 4096, 148) < prefill_bytes(1, 64, 4096)
