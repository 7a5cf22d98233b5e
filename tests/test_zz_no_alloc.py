"""xmla_decode_noalloc: the decode entry point for callers that cannot allocate
device memory (a backend inside a server that owns all allocations, a
latency-critical loop that must not hit cudaMalloc's implicit synchronisation,
a fixed memory arena).  It uses a fixed scratch array compiled into the
library instead of a caller workspace; its output must match xmla_decode's.

This file is collected last on purpose, so a run that stops at the first
failure has already run every other test."""
import pytest
import torch

from mla_latent_kv_yarn_b200 import workloads, xmla

import gpu_cases as gc

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from mla_latent_kv_yarn_b200 import build
    build.build()
    torch.cuda.init()


def test_noalloc_decode_matches_workspace_decode_on_two_calls():
    wl = workloads.custom(2, 2, [3000, 700], seed=41)
    cfg, ocfg = gc.cfgs()
    inp = workloads.layer_inputs(wl, 0, "cpu")
    # the cache with every token appended (one decode step through the workspace path)
    _, dec, st = gc.gpu_step(wl, inp, cfg)
    q = inp.q.cuda()
    scale = xmla.xmla_softmax_scale(cfg, 192)
    # reference: xmla_decode on the same cache with a caller-allocated workspace
    ref = dec.decode(cfg, st, q, scale).clone()
    torch.cuda.synchronize()
    assert dec.check_status() == 0
    gc.assert_close(ref, gc.oracle_out(wl, inp, ocfg), "workspace decode vs oracle",
                    plain_max_abs=True)
    for _ in range(2):  # the scratch keeps the previous call's contents
        out = torch.full_like(ref, float("nan"))
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        xmla.xmla_decode_noalloc(cfg, q, st.W_UK, st.W_UV, st.pool, st.num_blocks, st.block_table,
                                 st.max_blocks, st.seqlens, wl.batch, wl.q_len, wl.max_seqlen,
                                 scale, 0, status, out)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        # the same plan and kernels as xmla_decode: bit for bit the same output
        assert torch.equal(out, ref)


def test_noalloc_prompt_chunk_matches_workspace_decode():
    # a 128-token chunk runs the non-absorbed path (about 14 MB of workspace)
    wl = workloads.custom(1, 128, [700], seed=43)
    cfg, ocfg = gc.cfgs()
    inp = workloads.layer_inputs(wl, 0, "cpu")
    _, dec, st = gc.gpu_step(wl, inp, cfg)
    q = inp.q.cuda()
    scale = xmla.xmla_softmax_scale(cfg, 192)
    ref = dec.decode(cfg, st, q, scale).clone()
    torch.cuda.synchronize()
    assert dec.check_status() == 0
    assert xmla.xmla_decode_workspace_size(1, 128, 700, dec.sms, 0) <= (32 << 20)
    out = torch.full_like(ref, float("nan"))
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    xmla.xmla_decode_noalloc(cfg, q, st.W_UK, st.W_UV, st.pool, st.num_blocks, st.block_table,
                             st.max_blocks, st.seqlens, wl.batch, wl.q_len, wl.max_seqlen,
                             scale, 0, status, out)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert torch.equal(out, ref)


def test_noalloc_decode_rejects_sizes_beyond_its_scratch():
    cfg, _ = gc.cfgs()
    # 256 sequences x 8 queries at 1M context need far more than the fixed scratch
    need = xmla.xmla_decode_workspace_size(256, 8, 1 << 20, 148, 0)
    assert need > (32 << 20)  # XMLA_NOALLOC_SCRATCH_BYTES
    dummy = torch.zeros(16, dtype=torch.bfloat16, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    with pytest.raises(xmla.XmlaError) as e:
        xmla.xmla_decode_noalloc(cfg, dummy, dummy, dummy, dummy, 1 << 14, dummy, 1 << 14,
                                 dummy, 256, 8, 1 << 20, 0.1, 0, status, dummy)
    assert e.value.status == 3
