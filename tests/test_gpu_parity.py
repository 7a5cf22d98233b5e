"""Parity of the CUDA path (through the C ABI) with the fp64 oracle."""
import math

import numpy as np
import pytest
import torch

from mla_latent_kv_yarn_b200 import session, workloads, xmla
from oracle import mla_oracle as om

import gpu_cases as gc

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from mla_latent_kv_yarn_b200 import build
    build.build()
    torch.cuda.init()


# ------------------------------------------------------------------ RoPE

def _half_ulp_bf16(v: np.ndarray) -> np.ndarray:
    a = np.maximum(np.abs(v), 1e-30)
    return np.exp2(np.floor(np.log2(a)) - 8.0)


@pytest.mark.parametrize("theta,factor,mscale,mscale_all", [
    (1e4, 64.0, 1.0, 1.0), (1e7, 64.0, 1.0, 1.0), (1e4, 1.0, 1.0, 1.0),
    (1e4, 64.0, 0.707, 1.0),   # cos/sin carry mscale(s, 0.707) / mscale(s, 1) = 0.9139...
    (1e4, 64.0, 1.0, 0.5),     # ... and mscale(s, 1) / mscale(s, 0.5) = 1.0941...
])
def test_rope_within_half_ulp_of_oracle(theta, factor, mscale, mscale_all):
    cfg, ocfg = gc.cfgs(theta)
    cfg.factor = factor
    cfg.mscale = mscale
    cfg.mscale_all_dim = mscale_all
    ocfg = om.YarnConfig(rope_theta=theta, factor=factor, mscale=mscale, mscale_all_dim=mscale_all)
    g = torch.Generator().manual_seed(5)
    R, H = 37, 32
    q = torch.randn((R, H, 192), generator=g).to(torch.bfloat16)
    k = torch.randn((R, 64), generator=g).to(torch.bfloat16)
    pos = torch.tensor([0, 1, 63, 64, 4095, 4096, 262143, 262144, 524287] +
                       torch.randint(0, 524288, (R - 9,), generator=g).tolist(), dtype=torch.int64)
    qd, kd, pd = q.cuda(), k.cuda(), pos.cuda()
    session.rope_rows(cfg, qd, pd)
    session.rope_rows(cfg, kd, pd)
    torch.cuda.synchronize()
    want_q = om.rope(gc.f64(q)[..., 128:], pos.numpy()[:, None], ocfg)
    want_k = om.rope(gc.f64(k), pos.numpy(), ocfg)
    got_q, got_k = gc.f64(qd), gc.f64(kd)
    assert np.array_equal(got_q[..., :128], gc.f64(q)[..., :128])   # nope part untouched
    assert np.all(np.abs(got_q[..., 128:] - want_q) <= _half_ulp_bf16(want_q) * (1 + 1e-6))
    assert np.all(np.abs(got_k - want_k) <= _half_ulp_bf16(want_k) * (1 + 1e-6))


# ------------------------------------------------------------------ cache append

def test_cache_append_is_a_bit_exact_scatter():
    wl = workloads.custom(3, 1, [130, 64, 7], seed=3)
    bt = workloads.block_table(wl, 0)
    sid, pos, _ = workloads.token_index(wl)
    T = wl.tokens
    g = torch.Generator().manual_seed(9)
    c_bits = torch.randint(-32768, 32767, (T, 512), generator=g, dtype=torch.int16)
    k_bits = torch.randint(-32768, 32767, (T, 64), generator=g, dtype=torch.int16)
    pool0 = torch.randint(-32768, 32767, (wl.num_blocks + 2, 64, 576), generator=g, dtype=torch.int16)
    pool = pool0.cuda()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    xmla.xmla_cache_append(pool, pool.shape[0], bt.cuda(), bt.shape[1], 3, sid.cuda(), pos.cuda(),
                           c_bits.cuda(), k_bits.cuda(), None, T, status)
    torch.cuda.synchronize()
    want = pool0.numpy().view(np.uint16).copy()
    om.cache_append(want, bt.numpy(), sid.numpy(), pos.numpy(), c_bits.numpy().view(np.uint16),
                    k_bits.numpy().view(np.uint16))
    assert np.array_equal(pool.cpu().numpy().view(np.uint16), want)
    assert int(status.item()) == 0


def test_cache_append_skips_out_of_range_rows():
    bt = torch.tensor([[1, 0], [2, 5]], dtype=torch.int32)          # block 5 is outside a 3-block pool
    sid = torch.tensor([0, 1, 1, 2, 0], dtype=torch.int32)         # seq 2 does not exist
    pos = torch.tensor([3, 10, 70, 0, 200], dtype=torch.int64)      # 200 is past max_blocks*64
    c = torch.ones((5, 512), dtype=torch.bfloat16)
    k = torch.ones((5, 64), dtype=torch.bfloat16)
    pool = torch.zeros((3, 64, 576), dtype=torch.bfloat16, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    xmla.xmla_cache_append(pool, 3, bt.cuda(), 2, 2, sid.cuda(), pos.cuda(), c.cuda(), k.cuda(), None,
                           5, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 5
    p = pool.cpu().float()
    assert torch.all(p[1, 3] == 1) and torch.all(p[2, 10] == 1)    # the two valid rows landed
    assert float(p.sum()) == 2 * 576


def test_cache_append_with_rope_rotates_the_key_and_copies_the_latent():
    cfg, ocfg = gc.cfgs()
    g = torch.Generator().manual_seed(12)
    # distinct positions, some far past the original context (float64 angle matters there)
    pos = torch.cat([torch.tensor([0, 1, 63, 4095, 262143, 262144, 524287]),
                     torch.randperm(524287, generator=g)[:293] + 1]).unique()
    T = pos.numel()
    c = torch.randn((T, 512), generator=g).to(torch.bfloat16)
    k = torch.randn((T, 64), generator=g).to(torch.bfloat16)
    logical = torch.unique(pos // 64)
    bt = torch.zeros((1, 524288 // 64), dtype=torch.int32)
    bt[0, logical] = torch.arange(logical.numel(), dtype=torch.int32)
    nblk = logical.numel()
    pool = torch.zeros((nblk, 64, 576), dtype=torch.bfloat16, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    sid = torch.zeros(T, dtype=torch.int32)
    xmla.xmla_cache_append(pool, nblk, bt.cuda(), bt.shape[1], 1, sid.cuda(), pos.cuda(), c.cuda(),
                           k.cuda(), cfg, T, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    got = pool.cpu()
    rows = got[bt[0, pos // 64].long(), (pos % 64).long()]
    assert torch.equal(rows[:, :512].view(torch.int16), c.view(torch.int16))
    want = om.rope(gc.f64(k), pos.numpy(), ocfg)
    assert np.all(np.abs(gc.f64(rows[:, 512:]) - want) <= _half_ulp_bf16(want) * (1 + 1e-6))


# ------------------------------------------------------------------ decode, small cases

SMALL = [
    # batch, q_len, seqlens, num_splits
    (1, 1, [1], 0),
    (1, 1, [64], 0),
    (1, 1, [65], 0),
    (4, 1, [8, 16, 24, 40], 0),
    (2, 1, [1000, 130], 0),
    (3, 1, [777, 64, 2049], 3),
    (1, 1, [5000], 1),
    (1, 1, [300], 16),
    (2, 2, [129, 70], 0),
    (2, 3, [500, 63], 2),
    (2, 4, [1000, 257], 0),
    (1, 8, [2000], 0),
    (1, 4, [4], 0),
    # more splits per combine group than it keeps in flight (merged online)
    (2, 8, [1500, 900], 0),
    (1, 1, [20000], 200),
]


@pytest.mark.parametrize("batch,q_len,seqlens,splits", SMALL)
def test_decode_matches_expanded_oracle(batch, q_len, seqlens, splits):
    wl = workloads.custom(batch, q_len, seqlens, seed=sum(seqlens) + q_len)
    cfg, ocfg = gc.cfgs()
    inp = workloads.layer_inputs(wl, 0, "cpu")
    out, dec, _ = gc.gpu_step(wl, inp, cfg, num_splits=splits)
    assert dec.check_status() == 0
    gc.assert_close(out, gc.oracle_out(wl, inp, ocfg), f"{batch}x{q_len} {seqlens} s={splits}")


@pytest.mark.parametrize("batch,q_len,seqlens", [(1, 1, [300]), (2, 4, [1000, 257]),
                                                 (4, 1, [8, 16, 24, 40])])
def test_fused_step_equals_append_then_decode(batch, q_len, seqlens):
    """xmla_decode_step runs the append inside the first kernel of the chain;
    its output and the cache it leaves must be bit-identical to
    xmla_cache_append followed by xmla_decode."""
    wl = workloads.custom(batch, q_len, seqlens, seed=7 + sum(seqlens))
    cfg, _ = gc.cfgs()
    inp = workloads.layer_inputs(wl, 0, "cpu")
    out_f, dec_f, st_f = gc.gpu_step(wl, inp, cfg, fused=True)
    out_u, dec_u, st_u = gc.gpu_step(wl, inp, cfg, fused=False)
    assert dec_f.check_status() == 0 and dec_u.check_status() == 0
    assert torch.equal(out_f.view(torch.int16), out_u.view(torch.int16))
    assert torch.equal(st_f.pool.view(torch.int16), st_u.pool.view(torch.int16))


def test_fused_step_with_no_new_rows_is_a_plain_decode():
    wl = workloads.custom(2, 2, [129, 70], seed=11)
    cfg, _ = gc.cfgs()
    inp = workloads.layer_inputs(wl, 0, "cpu")
    dev = torch.device("cuda")
    st = session.build_layer(cfg, wl, inp, dev)  # every token, new ones included
    dec = session.Decoder(wl.batch, wl.q_len, wl.max_seqlen, dev)
    q = inp.q.to(dev)
    scale = xmla.xmla_softmax_scale(cfg, 192)
    ref = dec.decode(cfg, st, q, scale).clone()
    empty_i32 = torch.empty(0, dtype=torch.int32, device=dev)
    empty_i64 = torch.empty(0, dtype=torch.int64, device=dev)
    empty_bf = torch.empty((0, 576), dtype=torch.bfloat16, device=dev)
    out = torch.empty_like(ref)
    xmla.xmla_decode_step(cfg, q, st.W_UK, st.W_UV, st.pool, st.num_blocks, st.block_table,
                          st.max_blocks, st.seqlens, wl.batch, wl.q_len, wl.max_seqlen, empty_i32,
                          empty_i64, empty_bf, empty_bf, 0, scale, 0, dec.workspace, dec.ws_bytes,
                          dec.status, out)
    torch.cuda.synchronize()
    assert dec.check_status() == 0
    assert torch.equal(out.view(torch.int16), ref.view(torch.int16))


def test_decode_ignores_garbage_past_sequence_end():
    """Cache rows past a sequence's end (inside its last block) hold NaN here."""
    wl = workloads.custom(2, 1, [100, 130], seed=21)
    cfg, ocfg = gc.cfgs()
    inp = workloads.layer_inputs(wl, 0, "cpu")
    out, dec, _ = gc.gpu_step(wl, inp, cfg, pool_fill=float("nan"))
    assert dec.check_status() == 0
    gc.assert_close(out, gc.oracle_out(wl, inp, ocfg), "nan tail")


def test_decode_theta_1e7():
    wl = workloads.custom(1, 2, [3000], seed=22)
    cfg, ocfg = gc.cfgs(1e7)
    inp = workloads.layer_inputs(wl, 0, "cpu")
    out, _, _ = gc.gpu_step(wl, inp, cfg)
    gc.assert_close(out, gc.oracle_out(wl, inp, ocfg), "theta 1e7")


# ------------------------------------------------------------------ length-aware split plan

# A batch of several sequences with automatic splits is planned on the device:
# the first kernel of the call gives each (sequence, row group) unit a share of
# the SM-count CTAs in proportion to its pages.  Lengths far apart put most
# CTAs on one sequence and one CTA on each short one.
PLAN_CASES = [
    # batch, q_len, seqlens
    (2, 1, [3000, 100]),
    (6, 1, [1, 64, 65, 2500, 700, 129]),
    (3, 4, [2200, 300, 4]),
    (5, 8, [1200, 70, 640, 65, 999]),
    (3, 8, [8, 8, 8]),                      # every query sees 1..8 tokens
]


def _plan_tables(dec: session.Decoder):
    """The work and unit tables the first kernel left in the decoder's
    workspace (layout of the library's workspace plan: q_ext -- two bf16 rows,
    hi and lo, per query row up to 4096 tokens --, split O, split (m, l), then
    the two tables)."""
    def up(x, a):
        return (x + a - 1) // a * a
    split = dec.max_seqlen <= 4096                  # hi/lo query up to 4096 tokens
    hilo_rows = split or dec.batch > 1              # a batch past 4096 tokens keeps both parts too
    nr = 32 if dec.q_len == 1 or split else 64
    groups = (dec.q_len * 32 + nr - 1) // nr
    items = dec.sms
    off_o = up(dec.batch * dec.q_len * 32 * 576 * 2 * (2 if hilo_rows else 1), 1024)
    off_ml = up(off_o + items * nr * 512 * 4, 1024)
    off_w = up(off_ml + items * nr * 2 * 4, 1024)
    off_u = up(off_w + items * 16, 256)
    ws = dec.workspace
    work = ws[off_w:off_w + items * 16].view(torch.int32).view(items, 4).cpu().numpy()
    unit = ws[off_u:off_u + dec.batch * groups * 8].view(torch.int32).view(-1, 2).cpu().numpy()
    return work, unit, groups


@pytest.mark.parametrize("batch,q_len,seqlens", PLAN_CASES)
def test_length_aware_plan_matches_expanded_oracle(batch, q_len, seqlens):
    wl = workloads.custom(batch, q_len, seqlens, seed=90 + sum(seqlens))
    cfg, ocfg = gc.cfgs()
    inp = workloads.layer_inputs(wl, 0, "cpu")
    out, dec, _ = gc.gpu_step(wl, inp, cfg)
    assert dec.check_status() == 0
    gc.assert_close(out, gc.oracle_out(wl, inp, ocfg), f"plan {batch}x{q_len} {seqlens}")


@pytest.mark.parametrize("batch,q_len,seed", [(40, 1, 1), (147, 1, 2), (20, 4, 3)])
def test_length_aware_plan_partitions_every_page_once(batch, q_len, seed):
    """The tables: every page of every unit in exactly one CTA's run, runs of a
    unit consecutive and in page order, no more CTAs than SMs, and the largest
    run the smallest that fits (found here by brute force); then the output
    against the (absorbed, pinned to the expanded) oracle."""
    rng = np.random.default_rng(seed)
    seqlens = [int(x) for x in rng.integers(q_len, 900, size=batch)]
    seqlens[0] = 4000       # one long sequence; up to 4096 tokens the query is split hi/lo
    wl = workloads.custom(batch, q_len, seqlens, seed=300 + seed)
    cfg, ocfg = gc.cfgs()
    inp = workloads.layer_inputs(wl, 0, "cpu")
    out, dec, _ = gc.gpu_step(wl, inp, cfg)
    assert dec.check_status() == 0
    work, unit, groups = _plan_tables(dec)
    C = dec.sms
    w = [(seqlens[u // groups] + 63) // 64 for u in range(batch * groups)]
    covered = 0
    for u, (first, ns) in enumerate(unit):
        assert ns >= 1
        runs = work[first:first + ns]
        assert (runs[:, 0] == u).all()
        assert runs[0, 1] == 0 and runs[-1, 2] == w[u]
        assert (runs[1:, 1] == runs[:-1, 2]).all() and (runs[:, 2] > runs[:, 1]).all()
        covered += ns
    assert covered <= C and (work[covered:, 0] == -1).all()
    assert (unit[:, 0] == np.cumsum([0] + list(unit[:-1, 1]))).all()   # unit after unit
    tot, wmax = sum(w), max(w)
    T = next(t for t in range(max(1, -(-tot // C), min(2, wmax)), wmax + 2)
             if sum(max(1, -(-x // t)) for x in w) <= C)
    assert int((work[:covered, 2] - work[:covered, 1]).max()) == T
    gc.assert_close(out, gc.oracle_out(wl, inp, ocfg, form="absorbed"), f"plan B={batch}")


@pytest.mark.parametrize("q_len,seed", [(1, 1), (1, 2), (1, 3), (2, 4), (4, 5), (8, 6)])
def test_short_contexts(q_len, seed):
    """Contexts of q_len to 200 tokens, where few tokens dominate and |out|
    reaches ~4: the score error of a bf16-rounded query (about 2^-9 relative)
    alone would exceed the bound on some of them (measured by emulating the
    kernel's roundings on the CPU: 2 in 60 random cases, worst 1.4e-2), so up
    to 4096 tokens the query goes to the QK product as hi + lo bf16 parts."""
    rng = np.random.default_rng(500 + seed)
    seqlens = [int(x) for x in rng.integers(q_len, 200, size=8)]
    wl = workloads.custom(8, q_len, seqlens, seed=600 + seed)
    cfg, ocfg = gc.cfgs()
    inp = workloads.layer_inputs(wl, 0, "cpu")
    out, dec, _ = gc.gpu_step(wl, inp, cfg)
    assert dec.check_status() == 0
    gc.assert_close(out, gc.oracle_out(wl, inp, ocfg), f"short {seqlens}")


# ------------------------------------------------------------------ prefill chunks

# A long q_len is a chunk of a prompt: the chunk's tokens are appended and each
# attends causally to the cache up to its own position (the first ones of a
# fresh prompt see a handful of tokens).
PREFILL_CASES = [
    # batch, q_len, seqlens, oracle form.  From 64 new tokens per sequence a chunk
    # runs the non-absorbed tensor-core path (K_nope and V expanded per head, fp16
    # products); shorter ones the absorbed split-K path.
    (1, 64, [64], "expanded"),             # a fresh 64-token prompt
    (1, 200, [1000], "expanded"),          # a chunk on an 800-token prefix
    (2, 130, [130, 700], "expanded"),      # one fresh prompt, one continued
    (1, 96, [4500], "absorbed"),           # a chunk past 4096 tokens
    (1, 1024, [1024], "absorbed"),
    (1, 256, [256], "expanded"),           # exactly two tiles of 128 queries
    (3, 128, [128, 1000, 300], "absorbed"),  # three sequences, different prefixes
    (1, 64, [9000], "absorbed"),           # 64 queries over 71 key tiles
    (2, 100, [100, 5000], "absorbed"),
    (1, 63, [700], "absorbed"),            # one below the tensor-core path: absorbed
    (1, 16, [3000], "absorbed"),           # several splits per unit: merged before W_UV
    (2, 12, [2000, 500], "absorbed"),      # length-aware plan, merged through the unit table
]


@pytest.mark.parametrize("batch,q_len,seqlens,form", PREFILL_CASES)
def test_prefill_chunk_matches_the_oracle(batch, q_len, seqlens, form):
    wl = workloads.custom(batch, q_len, seqlens, seed=400 + q_len + sum(seqlens))
    cfg, ocfg = gc.cfgs()
    inp = workloads.layer_inputs(wl, 0, "cpu")
    out, dec, _ = gc.gpu_step(wl, inp, cfg)
    assert dec.check_status() == 0
    gc.assert_close(out, gc.oracle_out(wl, inp, ocfg, form=form), f"prefill {q_len} {seqlens}",
                    plain_below=True)


@pytest.mark.parametrize("q_len,seqlens", [(70, [70]), (128, [200])])
def test_prefill_chunk_ignores_garbage_past_sequence_end(q_len, seqlens):
    """The pool rows past each sequence's end hold NaN: the expansion writes zeros
    for them, so a zero probability never meets a NaN value."""
    wl = workloads.custom(1, q_len, seqlens, seed=31 + q_len)
    cfg, ocfg = gc.cfgs()
    inp = workloads.layer_inputs(wl, 0, "cpu")
    out, dec, _ = gc.gpu_step(wl, inp, cfg, pool_fill=float("nan"))
    assert dec.check_status() == 0
    gc.assert_close(out, gc.oracle_out(wl, inp, ocfg), f"prefill nan tail {q_len} {seqlens}")


def test_prefill_chunk_plain_decode_call_equals_the_step():
    """xmla_decode on a cache that already holds the chunk (no append in the call)
    gives the step's output bit for bit."""
    wl = workloads.custom(2, 96, [300, 96], seed=5)
    cfg, _ = gc.cfgs()
    inp = workloads.layer_inputs(wl, 0, "cpu")
    out, dec, st = gc.gpu_step(wl, inp, cfg)
    again = dec.decode(cfg, st, inp.q.cuda(), xmla.xmla_softmax_scale(cfg)).clone()
    torch.cuda.synchronize()
    assert dec.check_status() == 0
    assert torch.equal(out.view(torch.int16), again.view(torch.int16))


def test_length_aware_plan_is_deterministic():
    wl = workloads.custom(3, 2, [4000, 90, 1500], seed=77)
    cfg, _ = gc.cfgs()
    inp = workloads.layer_inputs(wl, 0, "cpu")
    a, dec, st = gc.gpu_step(wl, inp, cfg)
    q = inp.q.cuda().clone()
    for _ in range(2):
        b = dec.decode(cfg, st, q, xmla.xmla_softmax_scale(cfg)).clone()
        torch.cuda.synchronize()
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def _host_mapped(t: torch.Tensor) -> bool:
    try:
        from cuda.bindings import runtime as rt
        err, dptr = rt.cudaHostGetDevicePointer(t.data_ptr(), 0)
        return int(err) == 0 and int(dptr) == t.data_ptr()
    except Exception:
        return False


def test_decode_step_buffers_in_mapped_host_memory():
    # a decode call (q_len <= 8) may take q and out in pinned host memory mapped into
    # the device: the same output as with device buffers
    wl = workloads.custom(2, 2, [300, 129], seed=27)
    cfg, _ = gc.cfgs()
    inp = workloads.layer_inputs(wl, 0, "cpu")
    _, dec, st = gc.gpu_step(wl, inp, cfg)
    q_h = inp.q.clone().pin_memory()
    out_h = torch.zeros((wl.batch, wl.q_len, 32, 128), dtype=torch.bfloat16).pin_memory()
    if not (_host_mapped(q_h) and _host_mapped(out_h)):
        pytest.skip("pinned host memory is not mapped into the device")
    scale = xmla.xmla_softmax_scale(cfg)
    want = dec.decode(cfg, st, inp.q.cuda(), scale).clone()
    dec.decode(cfg, st, q_h, scale, out=out_h)
    torch.cuda.synchronize()
    assert dec.check_status() == 0
    assert torch.equal(out_h.view(torch.int16), want.cpu().view(torch.int16))


def test_decode_is_deterministic_and_split_count_only_changes_rounding():
    wl = workloads.custom(1, 1, [9000], seed=23)
    cfg, ocfg = gc.cfgs()
    inp = workloads.layer_inputs(wl, 0, "cpu")
    a, dec, st = gc.gpu_step(wl, inp, cfg)
    q = inp.q.cuda().clone()
    b = dec.decode(cfg, st, q, xmla.xmla_softmax_scale(cfg)).clone()
    torch.cuda.synchronize()
    assert torch.equal(a, b)                                   # same split plan: bit-identical
    ref = gc.oracle_out(wl, inp, ocfg)
    for s in (1, 2, 7, 70):
        d = session.Decoder(1, 1, 9000, "cuda", s)
        gc.assert_close(d.decode(cfg, st, q, xmla.xmla_softmax_scale(cfg)), ref, f"splits={s}")


# ------------------------------------------------------------------ device-detected errors

def test_bad_block_id_is_reported_not_faulted():
    wl = workloads.custom(1, 1, [200], seed=24)
    cfg, _ = gc.cfgs()
    inp = workloads.layer_inputs(wl, 0, "cpu")
    _, dec, st = gc.gpu_step(wl, inp, cfg)
    st.block_table[0, 1] = st.num_blocks + 7          # points outside the pool
    dec.status.zero_()
    q = inp.q.cuda().clone()
    out = dec.decode(cfg, st, q, 0.1)
    torch.cuda.synchronize()
    assert dec.check_status() == 5
    assert torch.isfinite(out.float()).all()


def test_sequence_longer_than_max_seqlen_is_reported():
    wl = workloads.custom(1, 1, [200], seed=25)
    cfg, _ = gc.cfgs()
    inp = workloads.layer_inputs(wl, 0, "cpu")
    _, dec, st = gc.gpu_step(wl, inp, cfg)
    st.seqlens[0] = 10_000                            # > max_seqlen given to the plan (200)
    dec.status.zero_()
    dec.decode(cfg, st, inp.q.cuda().clone(), 0.1)
    torch.cuda.synchronize()
    assert dec.check_status() == 5


def test_bounded_wait_gives_up_and_reports_timeout():
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    xmla.xmla_selftest_wait_timeout(status, 2_000_000)      # 2 ms
    torch.cuda.synchronize()
    assert int(status.item()) == 6
    # the context is still usable
    assert float(torch.ones(4, device="cuda").sum()) == 4.0


def test_host_rejects_small_workspace():
    wl = workloads.custom(1, 1, [256], seed=26)
    cfg, _ = gc.cfgs()
    inp = workloads.layer_inputs(wl, 0, "cpu")
    _, dec, st = gc.gpu_step(wl, inp, cfg)
    with pytest.raises(xmla.XmlaError) as e:
        xmla.xmla_decode(cfg, inp.q.cuda(), st.W_UK, st.W_UV, st.pool, st.num_blocks, st.block_table,
                         st.max_blocks, st.seqlens, 1, 1, 256, 0.1, 0, dec.workspace,
                         dec.ws_bytes - 1024, dec.status, dec.out)
    assert e.value.status == 3


# ------------------------------------------------------------------ the five seeded workloads

def test_workload_decode_4k():
    wl = workloads.workload("decode_4k")
    cfg, ocfg = gc.cfgs()
    inp = workloads.layer_inputs(wl, 0, "cpu")
    out, dec, _ = gc.gpu_step(wl, inp, cfg)
    assert dec.check_status() == 0
    gc.assert_close(out, gc.oracle_out(wl, inp, ocfg, form="expanded"), "decode_4k", plain_max_abs=True)


def test_workload_decode_256k():
    wl = workloads.workload("decode_256k")
    cfg, ocfg = gc.cfgs()
    inp = workloads.layer_inputs(wl, 0, "cuda")
    out, dec, _ = gc.gpu_step(wl, inp, cfg)
    assert dec.check_status() == 0
    gc.assert_close(out, gc.oracle_out(wl, inp, ocfg, form="expanded"), "decode_256k", plain_max_abs=True)


def test_workload_verify_q4_b8():
    wl = workloads.workload("verify_q4_b8")
    cfg, ocfg = gc.cfgs()
    inp = workloads.layer_inputs(wl, 0, "cuda")
    out, dec, _ = gc.gpu_step(wl, inp, cfg)
    assert dec.check_status() == 0
    gc.assert_close(out, gc.oracle_out(wl, inp, ocfg, seqs=[0, 3, 7], form="absorbed"), "verify_q4_b8", plain_max_abs=True)


def test_workload_decode_512k_b4():
    wl = workloads.workload("decode_512k_b4")
    cfg, ocfg = gc.cfgs()
    inp = workloads.layer_inputs(wl, 0, "cuda")
    out, dec, _ = gc.gpu_step(wl, inp, cfg)
    assert dec.check_status() == 0
    gc.assert_close(out, gc.oracle_out(wl, inp, ocfg, seqs=[0, 3], form="absorbed"), "decode_512k_b4", plain_max_abs=True)


def test_workload_prefill_4k_sampled_queries():
    # query j of the chunk sits at position N - q_len + j and sees tokens 0..that
    # position, which is the one-query case over the first position + 1 tokens
    wl = workloads.workload("prefill_4k")
    cfg, ocfg = gc.cfgs()
    inp = workloads.layer_inputs(wl, 0, "cuda")
    out, dec, _ = gc.gpu_step(wl, inp, cfg)
    assert dec.check_status() == 0
    n, ql = wl.seqlens[0], wl.q_len
    js = [0, 1, 63, 64, 127, 1000, 2047, 2048, 3071, 4000, ql - 1]
    c, kp = gc.f64(inp.c_kv[:n]), gc.f64(inp.k_pe[:n])
    kp_rot = om.rope(kp, np.arange(n), ocfg)
    wk, wv = gc.f64(inp.W_UK), gc.f64(inp.W_UV)
    ref = []
    for j in js:
        t = n - ql + j + 1
        ref.append(om.mla_attention_absorbed(gc.f64(inp.q[0, j:j + 1]), c[:t], kp_rot[:t], wk, wv,
                                             ocfg)[0])
    gc.assert_close(out[:, js], {0: np.stack(ref)}, "prefill_4k sampled queries", plain_below=True)


@pytest.mark.parametrize("layer", [0, 39])
def test_workload_step_40l_b32_sampled_layers(layer):
    wl = workloads.workload("step_40l_b32")
    cfg, ocfg = gc.cfgs()
    inp = workloads.layer_inputs(wl, layer, "cuda")
    out, dec, _ = gc.gpu_step(wl, inp, cfg)
    assert dec.check_status() == 0
    seqs = [int(np.argmax(wl.seqlens)), int(np.argmin(wl.seqlens)), 5, 17]
    gc.assert_close(out, gc.oracle_out(wl, inp, ocfg, seqs=seqs, form="absorbed"),
                    f"step_40l_b32 layer {layer}", plain_max_abs=True)


# ------------------------------------------------------------------ cache producer (kv_a_proj_with_mqa)

def _bf16_ulp(v: np.ndarray) -> np.ndarray:
    a = np.maximum(np.abs(v), 2.0 ** -126)
    return np.exp2(np.floor(np.log2(a)) - 7.0)


def _produce(T, seed, bias=True, rope=True):
    cfg, ocfg = gc.cfgs()
    g = torch.Generator().manual_seed(seed)
    hidden = torch.randn((T, om.HIDDEN), generator=g).to(torch.bfloat16)
    W = (torch.randn((576, om.HIDDEN), generator=g) / om.HIDDEN ** 0.5).to(torch.bfloat16)
    b = (torch.randn(576, generator=g) * 0.5).to(torch.bfloat16) if bias else None
    pos = torch.randperm(262144, generator=g)[:T].to(torch.int64)
    pos[0] = 262143
    logical = torch.unique(pos // 64)
    bt = torch.full((1, 4096), -1, dtype=torch.int32)
    bt[0, logical] = torch.randperm(logical.numel(), generator=g).to(torch.int32)
    nblk = logical.numel()
    pool = torch.zeros((nblk, 64, 576), dtype=torch.bfloat16, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    sid = torch.zeros(T, dtype=torch.int32)
    xmla.xmla_kv_produce(hidden.cuda(), W.cuda(), None if b is None else b.cuda(), T,
                         cfg if rope else None, pool, nblk, bt.cuda(), 4096, 1, sid.cuda(),
                         pos.cuda(), status)
    torch.cuda.synchronize()
    rows = pool.cpu()[bt[0, pos // 64].long(), (pos % 64).long()]
    c, k = om.kv_a_projection(gc.f64(hidden), gc.f64(W), None if b is None else gc.f64(b))
    return int(status.item()), gc.f64(rows), c, k, pos, ocfg


@pytest.mark.parametrize("T,bias", [(1, False), (5, True), (33, False)])
def test_kv_produce_matches_the_projection_oracle(T, bias):
    """The latent is the bf16 rounding of the projection (within one bf16 step of
    the fp64 value, fp32 accumulation); the rope key is the rotation of the
    bf16-rounded raw key (within two steps: one from the input, the rotation's
    own rounding)."""
    st, rows, c, k, pos, ocfg = _produce(T, 40 + T, bias)
    assert st == 0
    assert np.all(np.abs(rows[:, :512] - c) <= _bf16_ulp(c) * (1 + 1e-6))
    k_bf16 = gc.f64(torch.from_numpy(k).to(torch.bfloat16))
    want = om.rope(k_bf16, pos.numpy(), ocfg)
    pair_mag = np.maximum(np.abs(np.concatenate([k_bf16[:, 32:], k_bf16[:, :32]], axis=1)),
                          np.abs(k_bf16))
    assert np.all(np.abs(rows[:, 512:] - want) <= 2 * _bf16_ulp(pair_mag) * (1 + 1e-6))


def test_kv_produce_without_rope_stores_the_raw_key():
    st, rows, c, k, _, _ = _produce(3, 77, bias=True, rope=False)
    assert st == 0
    assert np.all(np.abs(rows[:, 512:] - k) <= _bf16_ulp(k) * (1 + 1e-6))


def test_kv_produce_reports_rows_out_of_range():
    cfg, _ = gc.cfgs()
    hidden = torch.ones((2, om.HIDDEN), dtype=torch.bfloat16, device="cuda")
    W = torch.zeros((576, om.HIDDEN), dtype=torch.bfloat16, device="cuda")
    bt = torch.tensor([[0, 7]], dtype=torch.int32, device="cuda")  # block 7 outside a 1-block pool
    pool = torch.zeros((1, 64, 576), dtype=torch.bfloat16, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    xmla.xmla_kv_produce(hidden, W, None, 2, cfg, pool, 1, bt, 2, 1,
                         torch.zeros(2, dtype=torch.int32, device="cuda"),
                         torch.tensor([3, 70], dtype=torch.int64, device="cuda"), status)
    torch.cuda.synchronize()
    assert int(status.item()) == 5 and float(pool.float().abs().sum()) == 0.0


@pytest.mark.parametrize("batch,q_len,seqlens", [(1, 1, [300]), (2, 4, [1000, 257]),
                                                 (4, 1, [8, 16, 24, 40])])
def test_step_from_hidden_matches_the_oracle(batch, q_len, seqlens):
    """xmla_decode_step_from_hidden: the new tokens' cache rows come from their
    hidden states (projection, bf16, RoPE, append), then the layer attends.  The
    oracle builds the same rows from its own projection."""
    wl = workloads.custom(batch, q_len, seqlens, seed=90 + sum(seqlens))
    cfg, ocfg = gc.cfgs()
    inp = workloads.layer_inputs(wl, 0, "cpu")
    hidden, W_kva = workloads.producer_inputs(wl, 0, "cpu")
    rows = torch.tensor(workloads.new_token_rows(wl, inp.offsets))
    c, k = om.kv_a_projection(gc.f64(hidden), gc.f64(W_kva))
    inp.c_kv[rows] = torch.from_numpy(c).to(torch.bfloat16)
    inp.k_pe[rows] = torch.from_numpy(k).to(torch.bfloat16)
    ref = gc.oracle_out(wl, inp, ocfg)

    dev = torch.device("cuda")
    prefix, new = session.split_prefix(wl, inp)
    st = session.build_layer(cfg, wl, prefix, dev)
    dec = session.Decoder(wl.batch, wl.q_len, wl.max_seqlen, dev)
    out = dec.step_from_hidden(cfg, st, inp.q.to(dev), hidden.to(dev), W_kva.to(dev),
                               new.positions.to(dev), new.seq_ids.to(dev),
                               xmla.xmla_softmax_scale(cfg, 192)).clone()
    torch.cuda.synchronize()
    assert dec.check_status() == 0
    gc.assert_close(out, ref, f"from hidden {batch}x{q_len} {seqlens}")
