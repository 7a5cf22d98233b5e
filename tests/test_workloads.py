"""The seeded input recipe: the workloads' shapes, block tables, value
distributions and determinism, as the design states them.  CPU only (the large
workloads are checked by their shapes, not by drawing their tensors)."""
import math

import numpy as np
import pytest
import torch

from mla_latent_kv_yarn_b200 import workloads as W


def test_the_five_workloads_and_the_extra_one_have_the_stated_shapes():
    d4 = W.workload("decode_4k")
    assert (d4.batch, d4.q_len, d4.seqlens, d4.layers, d4.contiguous) == (1, 1, [4096], 1, True)
    d256 = W.workload("decode_256k")
    assert (d256.batch, d256.q_len, d256.seqlens, d256.contiguous) == (1, 1, [262144], False)
    s40 = W.workload("step_40l_b32")
    assert (s40.batch, s40.q_len, s40.layers) == (32, 1, 40)
    assert all(8192 <= n <= 65536 for n in s40.seqlens) and len(set(s40.seqlens)) > 16
    v4 = W.workload("verify_q4_b8")
    assert (v4.batch, v4.q_len, v4.seqlens) == (8, 4, [131072] * 8)
    d512 = W.workload("decode_512k_b4")
    assert (d512.batch, d512.q_len, d512.seqlens) == (4, 1, [524288] * 4)
    pf = W.workload("prefill_4k")
    assert (pf.batch, pf.q_len, pf.seqlens) == (1, 4096, [4096])
    # by index too, with distinct seeds
    assert [W.workload(i).name for i in range(5)] == W.WORKLOAD_NAMES
    assert len({W.workload(n).seed for n in W.WORKLOAD_NAMES + W.EXTRA_WORKLOADS}) == 6
    # one 64-token block per started page
    assert d256.max_blocks == 4096 and d256.num_blocks == 4096
    assert s40.num_blocks == sum(math.ceil(n / 64) for n in s40.seqlens)


def test_block_tables_are_a_permutation_of_the_pool_or_the_identity():
    paged = W.custom(3, 2, [130, 64, 700], seed=5)
    inp = W.layer_inputs(paged, 0, "cpu")
    bt = inp.block_table.numpy()
    used = np.concatenate([bt[s, :math.ceil(n / 64)] for s, n in enumerate(paged.seqlens)])
    assert sorted(used.tolist()) == list(range(inp.num_blocks))  # every block exactly once
    assert not np.array_equal(used, np.arange(inp.num_blocks))  # shuffled
    contig = W.custom(1, 1, [4096], contiguous=True, seed=5)
    bt = W.layer_inputs(contig, 0, "cpu").block_table.numpy()[0]
    assert np.array_equal(bt[:64], np.arange(64))


def test_value_distributions_dtypes_and_shapes():
    wl = W.workload("decode_4k")
    inp = W.layer_inputs(wl, 0, "cpu")
    assert inp.q.shape == (1, 1, 32, 192) and inp.c_kv.shape == (4096, 512)
    assert inp.k_pe.shape == (4096, 64) and inp.W_UK.shape == (32, 128, 512)
    assert inp.W_UV.shape == (32, 512, 128)
    for t in (inp.q, inp.c_kv, inp.k_pe, inp.W_UK, inp.W_UV):
        assert t.dtype == torch.bfloat16
    c = inp.c_kv.float()
    assert abs(c.mean().item()) < 0.01 and abs(c.std().item() - 1.0) < 0.01
    w = inp.W_UK.float()
    assert abs(w.std().item() - 1 / math.sqrt(512)) < 0.001
    assert int(inp.seqlens[0]) == 4096 and int(inp.positions[-1]) == 4095


def test_inputs_are_deterministic_per_workload_layer_and_tensor():
    wl = W.custom(2, 2, [300, 129], seed=11)
    a, b = W.layer_inputs(wl, 0, "cpu"), W.layer_inputs(wl, 0, "cpu")
    for x, y in ((a.q, b.q), (a.c_kv, b.c_kv), (a.W_UV, b.W_UV), (a.block_table, b.block_table)):
        assert torch.equal(x, y)
    other_layer = W.layer_inputs(wl, 1, "cpu")
    assert not torch.equal(a.c_kv, other_layer.c_kv)
    other_seed = W.layer_inputs(W.custom(2, 2, [300, 129], seed=12), 0, "cpu")
    assert not torch.equal(a.q, other_seed.q)


def test_unknown_workload_is_rejected():
    with pytest.raises(ValueError):
        W.workload("decode_1m")
