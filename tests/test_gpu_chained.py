"""Several layers captured back to back in one CUDA graph, sharing one decoder
workspace, as a multi-layer decode step runs.

The kernels of consecutive calls are chained with programmatic dependent launch:
layer k+1's first kernel may start while layer k's last kernels still run, and
it rewrites the same query buffer, split partials and work tables those
kernels read.  Each kernel waits (griddepcontrol.wait) for its predecessor
before it touches anything a predecessor writes or reads; this test pins that
ordering on the real chain.  The graph is replayed twice (the step appends the
same rows at the same positions, so a replay is idempotent) and every layer's
output is compared with the expanded fp64 oracle at the plain max-abs bound."""
import pytest
import torch

from mla_latent_kv_yarn_b200 import session, workloads, xmla

import gpu_cases as gc

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from mla_latent_kv_yarn_b200 import build
    build.build()
    torch.cuda.init()


CASES = [
    # batch, q_len, seqlens, layers
    (1, 1, [9000], 3),                              # one sequence: splits of equal size
    (6, 1, [5000, 300, 4200, 70, 6000, 2048], 4),   # device plan, per-sequence query precision
    (3, 4, [7000, 130, 5001], 3),                   # 64-row groups
    (2, 2, [3000, 900], 3),                         # hi/lo query for every sequence
    (1, 24, [600], 3),                              # a prompt chunk: tensor-core absorb and W_UV
]


@pytest.mark.parametrize("batch,q_len,seqlens,layers", CASES)
def test_layers_chained_in_one_graph(batch, q_len, seqlens, layers):
    wl = workloads.custom(batch, q_len, seqlens, seed=31 + sum(seqlens) + q_len, layers=layers)
    cfg, ocfg = gc.cfgs()
    dev = torch.device("cuda")
    scale = xmla.xmla_softmax_scale(cfg, 192)
    dec = session.Decoder(wl.batch, wl.q_len, wl.max_seqlen, dev)
    Ls = []
    for layer in range(layers):
        inp = workloads.layer_inputs(wl, layer, "cpu")
        prefix, new = session.split_prefix(wl, inp)
        st = session.build_layer(cfg, wl, prefix, dev)
        Ls.append({"ref": gc.oracle_out(wl, inp, ocfg), "st": st, "q": inp.q.to(dev),
                   "c": new.c_kv.to(dev), "k": new.k_pe.to(dev), "pos": new.positions.to(dev),
                   "sid": new.seq_ids.to(dev),
                   "out": torch.empty((batch, q_len, 32, 128), dtype=torch.bfloat16, device=dev)})
    torch.cuda.synchronize()

    def step():
        for L in Ls:
            dec.step(cfg, L["st"], L["q"], L["c"], L["k"], L["pos"], L["sid"], scale,
                     out=L["out"])

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    for rep in range(2):
        for L in Ls:
            L["out"].fill_(float("nan"))
        graph.replay()
        torch.cuda.synchronize()
        assert dec.check_status() == 0
        for k, L in enumerate(Ls):
            gc.assert_close(L["out"], L["ref"], f"replay {rep} layer {k}", plain_max_abs=True)
    del graph
