"""The kernels' bounded waits: with the wait limit set so that every pipeline
wait gives up at its first unsatisfied test, the bf16 heads and tree
attention calls return with MEDUSA_STATUS_TIMEOUT set (nothing hangs and
nothing faults: copies and MMAs already issued are still drained at the full
limit), and the next calls at the normal limit are correct again."""
import numpy as np
import pytest
import torch

import oracle
from helpers import assert_float_parity, float_tol
from medusa_tree_speculative_heads_b200 import api
from medusa_tree_speculative_heads_b200 import binding as B
from medusa_tree_speculative_heads_b200 import inputs as I
from medusa_tree_speculative_heads_b200.binding import Tree

pytestmark = pytest.mark.gpu


def _heads(w, parents, dev):
    return api.heads(dev["h"], dev["W_res"], dev["W_head"], Tree(parents), dev["root_token"], want_logits=True)


def _attention(w, parents, dev):
    return api.tree_attention(dev["q"], dev["k_tree"], dev["v_tree"], dev["k_cache"], dev["v_cache"],
                              dev["prefix_len"], Tree(parents), want_lse=True)


@pytest.mark.parametrize("B_", [1, 24])     # per-head merges; grid-barrier merges
def test_heads_wait_limit_times_out_then_recovers(B_):
    w = I.scaled(I.WORKLOADS["llama8b"], B=B_, d=1024, V=5000, K=2)
    parents = I.product_tree_parents((4, 2))
    inp = I.head_inputs(w)
    dev = {k: v.cuda() for k, v in inp.items()}
    B.set_wait_limit(1)
    try:
        bad = _heads(w, parents, dev)
        torch.cuda.synchronize()
    finally:
        B.set_wait_limit(0)
    assert int(bad["status"].item()) & B.STATUS_TIMEOUT
    good = _heads(w, parents, dev)
    torch.cuda.synchronize()
    assert int(good["status"].item()) == 0
    ref = oracle.heads(inp["h"], inp["W_res"], inp["W_head"], want_hk=False)
    assert_float_parity(good["logits"], ref["logits"], w.torch_dtype, "logits after a timed-out call")
    lg = good["logits"].double().cpu().numpy()
    ti = good["topk_idx"].cpu().numpy()
    for b in range(w.B):
        for k in range(w.K):
            assert np.array_equal(ti[b, k], oracle.topk(lg[b, k], 8))


@pytest.mark.parametrize("prefix", [300, 5000])   # several key splits (a cluster); one split per tile
def test_attention_wait_limit_times_out_then_recovers(prefix):
    w = I.scaled(I.WORKLOADS["llama8b"], B=2 if prefix > 1000 else 1, prefix=prefix)
    parents = I.product_tree_parents((4, 4, 2))
    inp = I.attention_inputs(w, len(parents))
    dev = {k: v.cuda() for k, v in inp.items()}
    B.set_wait_limit(1)
    try:
        bad = _attention(w, parents, dev)
        torch.cuda.synchronize()
    finally:
        B.set_wait_limit(0)
    assert int(bad["status"].item()) & B.STATUS_TIMEOUT
    good = _attention(w, parents, dev)
    torch.cuda.synchronize()
    assert int(good["status"].item()) == 0
    g = np.random.default_rng(3)
    T = len(parents)
    rows = np.array([[int(g.integers(w.B)), int(g.integers(T)), int(g.integers(w.Hq))] for _ in range(64)],
                    dtype=np.int32)
    ref_o, ref_l = oracle.tree_attention(inp["q"], inp["k_tree"], inp["v_tree"], inp["k_cache"], inp["v_cache"],
                                         inp["prefix_len"], parents, rows=rows)
    o = good["out"].float().cpu()[rows[:, 0], rows[:, 1], rows[:, 2]]
    assert_float_parity(o, ref_o, w.torch_dtype, "attention after a timed-out call")
    lse = good["lse"].cpu()[rows[:, 0], rows[:, 1], rows[:, 2]].numpy()
    assert np.abs(lse - ref_l).max() <= float_tol(w.torch_dtype)
