"""Parity of the sequence-parallel decode (xmla_decode_shard on every rank's
pages, gather, xmla_combine_shards) with the fp64 oracle.  The G ranks are
emulated one after another on one GPU: each shard runs on a pool holding
only its pages, and their partials are stacked in rank order as the
all-gather would leave them."""
import math

import numpy as np
import pytest
import torch

from mla_latent_kv_yarn_b200 import seq_parallel as sp
from mla_latent_kv_yarn_b200 import session, workloads, xmla
from oracle import mla_oracle as om

import gpu_cases as gc

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from mla_latent_kv_yarn_b200 import build
    build.build()
    torch.cuda.init()


def _run_shards(wl, inp, cfg, world, num_splits=0):
    dev = torch.device("cuda")
    st = session.build_layer(cfg, wl, inp, dev)
    q = inp.q.to(dev)
    scale = xmla.xmla_softmax_scale(cfg, 192)
    shards, partials = [], []
    for r in range(world):
        sh = sp.ShardDecoder(wl.batch, wl.q_len, wl.max_seqlen, world, r, dev, num_splits)
        st_r = sp.shard_layer(st, sh.page_lo, sh.page_hi)
        sh.decode_shard(cfg, st_r, q, scale)
        torch.cuda.synchronize()
        assert int(sh.status.item()) == 0
        shards.append(sh)
        partials.append(sh.partial.clone())
    sh0 = shards[0]
    sh0.gathered.copy_(torch.cat(partials))
    out = sh0.combine(st.W_UV).clone()
    torch.cuda.synchronize()
    return out, shards, partials, st


CASES = [
    # batch, q_len, seqlens, world
    (1, 1, [20000], 2),
    (1, 1, [20000], 3),
    (1, 1, [4096], 8),
    (2, 2, [1500, 900], 2),
    (3, 1, [777, 64, 2049], 4),
    (1, 4, [5000], 2),
    (1, 1, [100], 3),        # more ranks than pages: the last rank sees nothing
    (2, 8, [700, 130], 3),
]


@pytest.mark.parametrize("batch,q_len,seqlens,world", CASES)
def test_shards_merge_to_the_expanded_oracle(batch, q_len, seqlens, world):
    wl = workloads.custom(batch, q_len, seqlens, seed=31 + sum(seqlens) + world)
    cfg, ocfg = gc.cfgs()
    inp = workloads.layer_inputs(wl, 0, "cpu")
    out, _, _, _ = _run_shards(wl, inp, cfg, world)
    gc.assert_close(out, gc.oracle_out(wl, inp, ocfg), f"{batch}x{q_len} {seqlens} G={world}")


@pytest.mark.parametrize("batch,q_len,seqlens,world", [(2, 2, [1500, 900], 3), (1, 1, [100], 3)])
def test_each_shard_partial_matches_the_oracle_partial(batch, q_len, seqlens, world):
    """Per rank and row: the log-sum-exp (M + log2 L, natural units after the
    log2 e factor) and the normalised latent O / L of the rank's pages."""
    wl = workloads.custom(batch, q_len, seqlens, seed=77 + world)
    cfg, ocfg = gc.cfgs()
    inp = workloads.layer_inputs(wl, 0, "cpu")
    _, shards, partials, _ = _run_shards(wl, inp, cfg, world)
    wk = gc.f64(inp.W_UK)
    for sh, part in zip(shards, partials):
        O, ML = sp.partial_views(part, batch, q_len)
        O, ML = gc.f64(O), gc.f64(ML)
        for b in range(batch):
            n, o = wl.seqlens[b], inp.offsets[b]
            t_lo, t_hi = min(n, 64 * sh.page_lo), min(n, 64 * sh.page_hi)
            c = gc.f64(inp.c_kv[o + t_lo:o + t_hi])
            k_rot = om.rope(gc.f64(inp.k_pe[o:o + n]), np.arange(n), ocfg)[t_lo:t_hi]
            m, l, ow = om.attention_partial(gc.f64(inp.q[b]), c, k_rot, wk, ocfg, n, t_lo, t_hi)
            rows = slice(b * q_len * 32, (b + 1) * q_len * 32)
            Lg, Mg = ML[rows, 1], ML[rows, 0]
            seen = l.reshape(-1) > 0
            assert np.array_equal(Lg > 0, seen)                  # the same rows saw tokens
            assert np.all(Mg[~seen] == -np.inf) and np.all(O[rows][~seen] == 0)
            if not seen.any():
                continue
            lse_g = (Mg[seen] + np.log2(Lg[seen])) * math.log(2.0)
            lse_w = (m.reshape(-1) + np.log(l.reshape(-1)))[seen]
            assert np.abs(lse_g - lse_w).max() < 2e-2
            og = O[rows][seen] / Lg[seen, None]
            ow_n = ow.reshape(-1, 512)[seen] / l.reshape(-1)[seen, None]
            assert np.linalg.norm(og - ow_n) / np.linalg.norm(ow_n) < 1e-2


def test_one_shard_equals_the_plain_decode_closely():
    """G = 1: the shard covers every page; after the extra merge the result
    stays within bf16 rounding of xmla_decode's."""
    wl = workloads.custom(2, 2, [1500, 900], seed=5)
    cfg, ocfg = gc.cfgs()
    inp = workloads.layer_inputs(wl, 0, "cpu")
    out, _, _, st = _run_shards(wl, inp, cfg, 1)
    dev = torch.device("cuda")
    dec = session.Decoder(wl.batch, wl.q_len, wl.max_seqlen, dev)
    ref = dec.decode(cfg, st, inp.q.to(dev), xmla.xmla_softmax_scale(cfg, 192)).clone()
    torch.cuda.synchronize()
    d = (out.float() - ref.float()).abs()
    assert float(d.max()) <= 2.0 ** -7 * float(ref.float().abs().max())
    gc.assert_close(out, gc.oracle_out(wl, inp, ocfg), "G=1")


def test_combine_shards_rejects_bad_arguments():
    dev = torch.device("cuda")
    W = torch.zeros((32, 512, 128), dtype=torch.bfloat16, device=dev)
    buf = torch.zeros(2 * xmla.xmla_shard_partial_floats(1, 1), dtype=torch.float32, device=dev)
    out = torch.empty((1, 1, 32, 128), dtype=torch.bfloat16, device=dev)
    for args, code in [((buf, 0, W, 1, 1, out), "XMLA_ERR_SHAPE"),
                       ((buf, 2, W, 1, 65537, out), "XMLA_ERR_SHAPE"),
                       ((buf[1:], 2, W, 1, 1, out), "XMLA_ERR_INVALID_ARG")]:
        with pytest.raises(xmla.XmlaError, match=code):
            xmla.xmla_combine_shards(*args)
