"""The documented limits of the calls: trees of the maximum 128 nodes (a
128-deep chain and a wide random tree), 16 Medusa heads, d = 16384, against
the oracle."""
import numpy as np
import pytest
import torch

import oracle
from helpers import assert_float_parity, check_topk, float_tol
from medusa_tree_speculative_heads_b200 import api
from medusa_tree_speculative_heads_b200 import binding as B
from medusa_tree_speculative_heads_b200 import inputs as I
from medusa_tree_speculative_heads_b200.binding import Tree

pytestmark = pytest.mark.gpu

CHAIN = [-1] + list(range(127))                                     # 128 nodes, depth 128
WIDE = I.random_tree_parents(128, 8, 8, torch.Generator().manual_seed(17))   # 128 nodes, depth <= 8


@pytest.mark.parametrize("parents", [CHAIN, WIDE], ids=["chain128", "wide128"])
@pytest.mark.parametrize("name,kw", [
    ("llama8b", dict(B=2, prefix=300, cache_room=192)),                      # bf16 tcgen05 kernel
    ("tiny", dict(B=2, Hq=4, Hkv=2, D=64, prefix=64, cache_room=192)),       # fp32 kernel
])
def test_attention_on_128_node_trees(parents, name, kw):
    w = I.scaled(I.WORKLOADS[name], **kw)
    tree = Tree(parents)
    assert tree.T == 128
    pl = torch.tensor([300 if name == "llama8b" else 64, 0], dtype=torch.int32)
    inp = I.attention_inputs(w, 128, canary=float("nan"), prefix_len=pl)
    dev = {k: v.cuda() for k, v in inp.items()}
    out = api.tree_attention(dev["q"], dev["k_tree"], dev["v_tree"], dev["k_cache"], dev["v_cache"],
                             dev["prefix_len"], tree, max_prefix=int(pl.max()), want_lse=True)
    torch.cuda.synchronize()
    assert int(out["status"].item()) == 0
    ref_o, ref_l = oracle.tree_attention(inp["q"], inp["k_tree"], inp["v_tree"], inp["k_cache"], inp["v_cache"],
                                         inp["prefix_len"], parents)
    assert_float_parity(out["out"].float().cpu().reshape(-1, w.D), ref_o, w.torch_dtype, "out")
    assert np.abs(out["lse"].cpu().reshape(-1).numpy() - ref_l).max() <= float_tol(w.torch_dtype)


def test_greedy_verify_and_commit_along_a_128_deep_chain():
    # every node matches: the whole chain (128 nodes) is accepted and committed
    w = I.scaled(I.WORKLOADS["llama8b"], B=2, V=3000, prefix=100, cache_room=192)
    tree = Tree(CHAIN)
    g = torch.Generator().manual_seed(4)
    tok = torch.randint(0, w.V, (w.B, 128), generator=g, dtype=torch.int32)
    logits = torch.randn((w.B, 128, w.V), generator=g).bfloat16()
    for b in range(w.B):
        stop = 128 if b == 0 else 77           # sequence 1 stops matching after node 76
        for u in range(stop - 1):
            logits[b, u, int(tok[b, u + 1])] = 50.0
    out = api.tree_verify(B.GREEDY, logits.cuda(), tok.cuda(), tree, max_path=128)
    torch.cuda.synchronize()
    path, ln, bonus = oracle.verify_greedy(logits, tok, CHAIN, 128)
    assert out["accept_len"].tolist() == ln.tolist() == [128, 77]
    assert np.array_equal(out["accept_path"].cpu().numpy(), path)
    assert np.array_equal(out["bonus"].cpu().numpy(), bonus)
    pl = torch.tensor([100, 3], dtype=torch.int32)
    inp = I.attention_inputs(w, 128, prefix_len=pl)
    ref_k, ref_v, ref_npl, ref_st = oracle.kv_commit(inp["k_cache"], inp["v_cache"], inp["k_tree"], inp["v_tree"],
                                                     path, ln, pl)
    dev = {k: v.cuda() for k, v in inp.items()}
    res = api.kv_commit(dev["k_cache"], dev["v_cache"], dev["k_tree"], dev["v_tree"], out["accept_path"],
                        out["accept_len"], dev["prefix_len"])
    torch.cuda.synchronize()
    assert int(res["status"].item()) == 0 and ref_st == 0
    assert res["new_prefix_len"].cpu().tolist() == ref_npl.tolist() == [228, 80]
    assert torch.equal(dev["k_cache"].cpu(), ref_k) and torch.equal(dev["v_cache"].cpu(), ref_v)


def test_stochastic_verify_on_a_wide_128_node_tree():
    w = I.scaled(I.WORKLOADS["stoch_b64"], B=6, V=900)
    d = I.stochastic_inputs(w, WIDE)
    tree = Tree(WIDE)
    maxd = tree.max_depth
    for seed, step in ((1, 0), (2**40 + 3, 9)):
        out = api.tree_verify(B.STOCHASTIC, d["p"].cuda(), d["node_tokens"].cuda(), tree, q=d["q"].cuda(), seed=seed,
                              step=step)
        lg = api.tree_verify_logits(d["logits"].cuda(), I.STOCH_TEMPERATURE, d["q"].cuda(), d["node_tokens"].cuda(),
                                    tree, seed=seed, step=step)
        torch.cuda.synchronize()
        ref = oracle.verify_stochastic(d["p"], d["q"], d["node_tokens"], WIDE, seed, step, maxd)
        ref_l = oracle.verify_stochastic_logits(d["logits"], I.STOCH_TEMPERATURE, d["q"], d["node_tokens"], WIDE, seed,
                                                step, maxd)
        for o, r in ((out, ref), (lg, ref_l)):
            assert np.array_equal(o["accept_path"].cpu().numpy(), r[0])
            assert np.array_equal(o["accept_len"].cpu().numpy(), r[1])
            assert np.array_equal(o["bonus"].cpu().numpy(), r[2])


@pytest.mark.parametrize("name,kw", [
    ("llama8b", dict(B=2, d=256, V=900, K=16)),      # 16 heads, bf16 tensor-core kernel
    ("tiny", dict(d=128, V=700, K=16)),              # 16 heads, fp32
    ("llama8b", dict(B=1, d=16384, V=600, K=1)),     # the largest d
])
def test_heads_at_the_limits(name, kw):
    w = I.scaled(I.WORKLOADS[name], **kw)
    parents = [-1] + list(range(w.K))                # a chain through every head: depth K + 1
    tree = Tree(parents)
    inp = I.head_inputs(w)
    ref = oracle.heads(inp["h"], inp["W_res"], inp["W_head"])
    dev = {k: v.cuda() for k, v in inp.items()}
    out = api.heads(dev["h"], dev["W_res"], dev["W_head"], tree, dev["root_token"], want_logits=True)
    torch.cuda.synchronize()
    assert int(out["status"].item()) == 0
    tol = float_tol(w.torch_dtype)
    assert_float_parity(out["logits"], ref["logits"], w.torch_dtype, "logits")
    ti = out["topk_idx"].cpu().numpy()
    for b in range(w.B):
        for k in range(w.K):
            check_topk(ti[b, k], ref["logits"][b, k], tol)
        nt = out["node_tokens"][b].cpu().numpy()
        assert nt[0] == int(inp["root_token"][b])
        for k in range(w.K):
            assert nt[k + 1] == ti[b, k, 0]          # the chain takes every head's best entry
