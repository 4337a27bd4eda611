"""Vocabulary-sharded heads on one GPU: every shard's partial computed in
turn from its slice of W_head, the partials stacked in shard order (what the
all-gather delivers on several GPUs) and merged.  One shard reproduces
medusa_heads bit for bit; several match the fp64 oracle over the full
vocabulary like medusa_heads does."""
import numpy as np
import pytest
import torch

import oracle
from helpers import check_topk, float_tol
from medusa_tree_speculative_heads_b200 import api
from medusa_tree_speculative_heads_b200 import inputs as I
from medusa_tree_speculative_heads_b200.binding import Tree
from medusa_tree_speculative_heads_b200.sharded import ShardedHeads, vocab_shard

pytestmark = pytest.mark.gpu


def run_sharded(w, dev, n_shards, tree):
    parts, sh = [], None
    for r in range(n_shards):
        v0, v1 = vocab_shard(w.V, n_shards, r)
        sh = ShardedHeads(B=w.B, d=w.d, V=w.V, K=w.K, v0=v0, v1=v1, dtype=w.torch_dtype, tree=tree, device="cuda")
        parts.append(sh.shard(dev["h"], dev["W_res"], dev["W_head"][:, v0:v1].contiguous()).clone())
        torch.cuda.synchronize()
        assert int(sh.status.item()) == 0
    out = sh.merge(torch.stack(parts), dev["root_token"])
    torch.cuda.synchronize()
    return {k: v.clone() for k, v in out.items()}


CASES = [
    ("llama8b", dict(B=3, d=512, V=3001, K=4)),     # bf16: tensor-core kernel per shard
    ("llama8b", dict(B=70, d=256, V=1000, K=3)),    # bf16, B > 64: the general kernels
    ("tiny", {}),                                   # fp32, B = 1: the fused kernel
    ("tiny", dict(B=3, V=1500)),                    # fp32 general kernels
]


@pytest.mark.parametrize("name,kw", CASES)
def test_one_shard_is_medusa_heads_bit_for_bit(name, kw):
    w = I.scaled(I.WORKLOADS[name], **kw)
    parents = I.product_tree_parents((4, 2, 2)[:w.K]) if w.K >= 3 else I.product_tree_parents((2, 2))
    tree = Tree(parents)
    dev = {k: v.cuda() for k, v in I.head_inputs(w).items()}
    ref = api.heads(dev["h"], dev["W_res"], dev["W_head"], tree, dev["root_token"])
    out = run_sharded(w, dev, 1, tree)
    for k in ("topk_idx", "topk_prob", "node_tokens", "node_q"):
        assert torch.equal(out[k], ref[k]), k


@pytest.mark.parametrize("name,kw,n_shards", [
    ("llama8b", dict(B=4, d=512, V=5003, K=4), 2),
    ("llama8b", dict(B=4, d=512, V=5003, K=4), 5),
    ("llama8b", dict(B=2, d=256, V=64, K=2), 7),       # shards of 9-10 rows
    ("tiny", dict(V=1024), 3),
])
def test_shards_match_the_oracle_over_the_full_vocabulary(name, kw, n_shards):
    w = I.scaled(I.WORKLOADS[name], **kw)
    parents = I.product_tree_parents((4, 2, 2, 2)[:w.K])
    tree = Tree(parents)
    inp = I.head_inputs(w)
    ref = oracle.heads(inp["h"], inp["W_res"], inp["W_head"])
    dev = {k: v.cuda() for k, v in inp.items()}
    out = run_sharded(w, dev, n_shards, tree)
    tol = float_tol(w.torch_dtype)
    ti = out["topk_idx"].cpu().numpy()
    tp = out["topk_prob"].cpu().numpy()
    nt = out["node_tokens"].cpu().numpy()
    depth, rank = oracle.tree_shape(parents)
    for b in range(w.B):
        assert nt[b, 0] == int(inp["root_token"][b])
        for k in range(w.K):
            check_topk(ti[b, k], ref["logits"][b, k], tol)
            np.testing.assert_allclose(tp[b, k], ref["probs"][b, k, ti[b, k]], rtol=0, atol=tol)
        for i in range(1, len(parents)):
            assert nt[b, i] == ti[b, depth[i] - 2, rank[i]]
    # and the unsharded call agrees wherever its top-8 agrees with the oracle
    full = api.heads(dev["h"], dev["W_res"], dev["W_head"], tree, dev["root_token"])
    torch.cuda.synchronize()
    same = (full["topk_idx"] == out["topk_idx"]).float().mean().item()
    assert same > 0.95
    np.testing.assert_allclose(tp, full["topk_prob"].cpu().numpy(), rtol=0, atol=tol)


def test_merge_with_one_tree_per_sequence():
    w = I.scaled(I.WORKLOADS["llama8b"], B=3, d=256, V=2000, K=4)
    g = torch.Generator().manual_seed(3)
    trees = [I.random_tree_parents(n, 5, 8, g) for n in (30, 117, 7)]
    tree = Tree(trees)
    dev = {k: v.cuda() for k, v in I.head_inputs(w).items()}
    out = run_sharded(w, dev, 3, tree)
    ti = out["topk_idx"].cpu().numpy()
    nt = out["node_tokens"].cpu().numpy()
    for b, par in enumerate(trees):
        depth, rank = oracle.tree_shape(par)
        assert nt[b, 0] == int(dev["root_token"][b])
        for i in range(1, len(par)):
            assert nt[b, i] == ti[b, depth[i] - 2, rank[i]]
        assert (nt[b, len(par):] == -1).all()
