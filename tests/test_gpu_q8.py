"""Parity of the 8-bit latent cache path with the oracle: the quantising append
(bit-exact codes and exponents) and the decode over the 8-bit pool (output
within the decode tolerance of the fp64 attention over the dequantised rows)."""
import numpy as np
import pytest
import torch

from mla_latent_kv_yarn_b200 import session, workloads, xmla
from oracle import mla_oracle as om

import gpu_cases as gc

pytestmark = pytest.mark.gpu


def _bf16_rne(x: np.ndarray) -> np.ndarray:
    """float64 -> the nearest bf16 value (8 significant bits, ties to even)."""
    m, e = np.frexp(np.asarray(x, dtype=np.float64))
    return np.ldexp(np.rint(m * 256.0) / 256.0, e)


def _oracle_rows(c_kv: np.ndarray, k_pe: np.ndarray, positions, ocfg, rotate=True):
    """The oracle's quantised cache rows of tokens (c_kv, raw k_pe) at positions."""
    k = _bf16_rne(om.rope(k_pe, np.asarray(positions), ocfg)) if rotate else k_pe
    return om.q8_quantize(np.concatenate([c_kv, k], axis=1))


def _read_rows(pool: torch.Tensor, bt: np.ndarray, seq_ids, positions):
    rows = torch.stack([pool[int(bt[s, p // 64]), p % 64] for s, p in zip(seq_ids, positions)])
    rows = rows.cpu()
    return (rows[:, :576].view(torch.int8).numpy(), rows[:, 576:594].view(torch.int8).numpy(),
            rows[:, 594:].numpy())


@pytest.mark.parametrize("rotate", [True, False])
def test_q8_append_matches_the_oracle_quantisation(rotate):
    cfg, ocfg = gc.cfgs()
    g = torch.Generator().manual_seed(31 + rotate)
    T, B, max_blocks = 300, 2, 4
    c = torch.randn((T, 512), generator=g) * torch.exp2(
        torch.randint(-8, 9, (T, 1), generator=g).float())
    c = c.to(torch.bfloat16)
    k = (torch.randn((T, 64), generator=g) * 3).to(torch.bfloat16)
    seq = torch.randint(0, B, (T,), generator=g).to(torch.int32)
    pos = torch.randperm(B * max_blocks * 64, generator=g)[:T] % (max_blocks * 64)
    # one cache slot per row
    key = seq.long() * 10_000 + pos
    _, first = np.unique(key.numpy(), return_index=True)
    sel = torch.as_tensor(np.sort(first))
    c, k, seq, pos = c[sel].contiguous(), k[sel].contiguous(), seq[sel], pos[sel].to(torch.int64)
    T = c.shape[0]
    c[0, :32] = 0                       # an all-zero block
    c[1, 32:64] = 1e-6                  # below the smallest exponent's range
    c[2, 64:96] = 5e4                   # above the largest: saturates
    nblk = B * max_blocks + 3
    bt = torch.randperm(nblk, generator=g)[:B * max_blocks].view(B, max_blocks).to(torch.int32)
    pool = torch.full((nblk, 64, 608), 0x5a, dtype=torch.uint8, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    xmla.xmla_cache_append_q8(pool, nblk, bt.cuda(), max_blocks, B, seq.cuda(), pos.cuda(),
                              c.cuda(), k.cuda(), cfg if rotate else None, T, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    codes, exps, pad = _read_rows(pool, bt.numpy(), seq.tolist(), pos.tolist())
    want_c, want_e = _oracle_rows(gc.f64(c), gc.f64(k), pos.numpy(), ocfg, rotate)
    assert np.array_equal(exps, want_e)
    assert np.array_equal(codes, want_c)
    assert not pad.any()
    assert exps[0, 0] == om.Q8_EMIN and not codes[0, :32].any()
    assert exps[2, 2] == om.Q8_EMAX and np.all(np.abs(codes[2, 64:96]) == 127)


def test_q8_append_reports_rows_out_of_range():
    cfg, _ = gc.cfgs()
    pool = torch.zeros((2, 64, 608), dtype=torch.uint8, device="cuda")
    bt = torch.tensor([[0, 1]], dtype=torch.int32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    c = torch.ones((2, 512), dtype=torch.bfloat16, device="cuda")
    k = torch.ones((2, 64), dtype=torch.bfloat16, device="cuda")
    pos = torch.tensor([5, 128], dtype=torch.int64, device="cuda")   # 128: past the table
    sid = torch.zeros(2, dtype=torch.int32, device="cuda")
    xmla.xmla_cache_append_q8(pool, 2, bt, 2, 1, sid, pos, c, k, cfg, 2, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 5
    # the valid row went in: latent blocks of ones have e = -6 and codes 64
    row = pool[0, 5].cpu()
    assert row[:512].view(torch.int8).eq(64).all()
    assert row[576:592].view(torch.int8).eq(-6).all()


def _oracle_q8(wl, inp, ocfg, seqs=None):
    res = {}
    wk, wv = gc.f64(inp.W_UK), gc.f64(inp.W_UV)
    for b in (range(wl.batch) if seqs is None else seqs):
        o, n = inp.offsets[b], wl.seqlens[b]
        codes, exps = _oracle_rows(gc.f64(inp.c_kv[o:o + n]), gc.f64(inp.k_pe[o:o + n]),
                                   np.arange(n), ocfg)
        rows = om.q8_dequantize(codes, exps)
        res[b] = om.mla_attention_absorbed(gc.f64(inp.q[b]), rows[:, :512], rows[:, 512:], wk, wv,
                                           ocfg)
    return res


Q8_CASES = [
    # batch, q_len, seqlens
    (1, 1, [1]),
    (1, 1, [64]),
    (1, 1, [65]),
    (1, 1, [4096]),
    (1, 1, [20000]),
    (1, 8, [1200]),
    (2, 4, [300, 5000]),
    (3, 2, [4000, 90, 1500]),          # several sequences: the length-aware plan
    (4, 1, [10, 700, 64, 3000]),
]


@pytest.mark.parametrize("batch,q_len,seqlens", Q8_CASES)
def test_q8_decode_matches_the_oracle(batch, q_len, seqlens):
    wl = workloads.custom(batch, q_len, seqlens, seed=800 + q_len + sum(seqlens))
    cfg, ocfg = gc.cfgs()
    inp = workloads.layer_inputs(wl, 0, "cpu")
    out, dec, _ = gc.gpu_step(wl, inp, cfg, cache="q8")
    assert dec.check_status() == 0
    gc.assert_close(out, _oracle_q8(wl, inp, ocfg), f"q8 {batch} {q_len} {seqlens}")


@pytest.mark.parametrize("magnitude", [2.0 ** -12, 4096.0])
def test_q8_decode_with_small_and_large_cache_values(magnitude):
    # block exponents at the bottom of the range and above 5 (the converters'
    # general path): the latent and rope values scaled by a power of two
    wl = workloads.custom(2, 2, [700, 130], seed=826)
    cfg, ocfg = gc.cfgs()
    inp = workloads.layer_inputs(wl, 0, "cpu")
    inp.c_kv.mul_(magnitude)
    inp.k_pe.mul_(magnitude)
    out, dec, _ = gc.gpu_step(wl, inp, cfg, cache="q8")
    assert dec.check_status() == 0
    gc.assert_close(out, _oracle_q8(wl, inp, ocfg), f"q8 values x {magnitude}")


def test_q8_split_count_only_changes_rounding():
    wl = workloads.custom(1, 1, [9000], seed=823)
    cfg, ocfg = gc.cfgs()
    inp = workloads.layer_inputs(wl, 0, "cpu")
    ref = _oracle_q8(wl, inp, ocfg)
    for ns in (1, 7, 70):
        out, dec, _ = gc.gpu_step(wl, inp, cfg, cache="q8", num_splits=ns)
        assert dec.check_status() == 0
        gc.assert_close(out, ref, f"q8 splits {ns}")


def test_q8_decode_is_deterministic():
    wl = workloads.custom(3, 2, [4000, 90, 1500], seed=77)
    cfg, _ = gc.cfgs()
    inp = workloads.layer_inputs(wl, 0, "cpu")
    a, dec, st = gc.gpu_step(wl, inp, cfg, cache="q8")
    q = inp.q.cuda().clone()
    b = dec.decode(cfg, st, q, xmla.xmla_softmax_scale(cfg)).clone()
    torch.cuda.synchronize()
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_q8_rejects_long_query_chunks():
    cfg, _ = gc.cfgs()
    assert xmla.xmla_decode_q8_workspace_size(1, 9, 100, 148) == 0
    wl = workloads.custom(1, 1, [256], seed=26)
    inp = workloads.layer_inputs(wl, 0, "cpu")
    _, dec, st = gc.gpu_step(wl, inp, cfg, cache="q8")
    q = torch.zeros((1, 9, 32, 192), dtype=torch.bfloat16, device="cuda")
    out = torch.empty((1, 9, 32, 128), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(xmla.XmlaError) as e:
        xmla.xmla_decode_q8(cfg, q, st.W_UK, st.W_UV, st.pool, st.num_blocks, st.block_table,
                            st.max_blocks, st.seqlens, 1, 9, 256, 0.1, 0, dec.workspace,
                            dec.ws_bytes, dec.status, out)
    assert e.value.status == 2


def test_q8_workload_decode_256k():
    wl = workloads.workload("decode_256k")
    cfg, ocfg = gc.cfgs()
    inp = workloads.layer_inputs(wl, 0, "cuda")
    out, dec, _ = gc.gpu_step(wl, inp, cfg, cache="q8")
    assert dec.check_status() == 0
    gc.assert_close(out, _oracle_q8(wl, inp, ocfg), "q8 decode_256k", plain_max_abs=True)


def test_q8_workload_step_40l_b32_layer0_sampled():
    wl = workloads.workload("step_40l_b32")
    cfg, ocfg = gc.cfgs()
    inp = workloads.layer_inputs(wl, 0, "cuda")
    out, dec, _ = gc.gpu_step(wl, inp, cfg, cache="q8")
    assert dec.check_status() == 0
    seqs = [int(np.argmax(wl.seqlens)), int(np.argmin(wl.seqlens)), 5]
    gc.assert_close(out, _oracle_q8(wl, inp, ocfg, seqs), "q8 step_40l_b32 layer 0",
                    plain_max_abs=True)


def test_q8_bad_block_id_is_reported_not_faulted():
    wl = workloads.custom(1, 1, [200], seed=824)
    cfg, _ = gc.cfgs()
    inp = workloads.layer_inputs(wl, 0, "cpu")
    _, dec, st = gc.gpu_step(wl, inp, cfg, cache="q8")
    st.block_table[0, 1] = st.num_blocks + 7          # points outside the pool
    dec.status.zero_()
    out = dec.decode(cfg, st, inp.q.cuda().clone(), 0.1)
    torch.cuda.synchronize()
    assert dec.check_status() == 5
    assert torch.isfinite(out.float()).all()


def test_q8_sequence_longer_than_max_seqlen_is_reported():
    wl = workloads.custom(1, 1, [200], seed=825)
    cfg, _ = gc.cfgs()
    inp = workloads.layer_inputs(wl, 0, "cpu")
    _, dec, st = gc.gpu_step(wl, inp, cfg, cache="q8")
    st.seqlens[0] = 10_000                            # > max_seqlen given to the plan (200)
    dec.status.zero_()
    out = dec.decode(cfg, st, inp.q.cuda().clone(), 0.1)
    torch.cuda.synchronize()
    assert dec.check_status() == 5
    assert torch.isfinite(out.float()).all()
