"""Paged KV cache (a page pool read through a block table) for tree attention
and commit, against the fp64 oracle on the cache the oracle gathers through
the same table.  Slots no call may read hold NaN."""
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

NAN = float("nan")

CASES = [
    # workload, overrides, tree, page size, prefix lengths
    ("llama8b", dict(B=4, prefix=700), (4, 4, 2, 2), 16, [0, 1, 700, 333]),     # tcgen05, 16-row pages
    ("llama8b", dict(B=3, prefix=1000), (4, 2), 64, [64, 999, 130]),            # tcgen05, one box per page
    ("llama8b", dict(B=2, prefix=900), (3, 2, 1), 128, [900, 511]),             # tcgen05, pages of two chunks
    ("llama8b", dict(B=2, prefix=300), (3, 2), 8, [300, 47]),                   # tcgen05, 8-row pages
    ("llama8b", dict(B=3, D=64, prefix=260), (2, 2), 32, [260, 33, 0]),        # tcgen05, head_dim 64
    ("llama8b", dict(B=2, prefix=500), (4, 2), 24, [500, 73]),                  # fallback kernel: page size 24
    ("llama8b", dict(B=2, Hq=6, Hkv=2, prefix=400), (2, 2), 16, [400, 17]),    # fallback kernel: G = 3
    ("tiny", dict(B=2, Hq=4, Hkv=2, prefix=64), (2, 2), 5, [64, 9]),            # fp32 kernel
]


@pytest.mark.parametrize("name,kw,tree,ps,prefix", CASES)
def test_paged_attention_parity(name, kw, tree, ps, prefix):
    w = I.scaled(I.WORKLOADS[name], **kw)
    parents = I.product_tree_parents(tree)
    T = len(parents)
    pl = torch.tensor(prefix, dtype=torch.int32)
    inp = I.attention_inputs(w, T, prefix_len=pl)
    pc = I.paged_cache(w, ps, pl, room=T, canary=NAN)
    dev = {k: v.cuda() for k, v in list(inp.items()) + list(pc.items())}
    t = Tree(parents)
    out = api.tree_attention_paged(dev["q"], dev["k_tree"], dev["v_tree"], dev["k_pages"], dev["v_pages"],
                                   dev["block_table"], dev["prefix_len"], t, want_lse=True)
    torch.cuda.synchronize()
    assert int(out["status"].item()) == 0
    S_max = pc["block_table"].shape[1] * ps
    kc = oracle.gather_pages(pc["k_pages"], pc["block_table"], pl, S_max)
    vc = oracle.gather_pages(pc["v_pages"], pc["block_table"], pl, S_max)
    ref_o, ref_l = oracle.tree_attention(inp["q"], inp["k_tree"], inp["v_tree"], kc, vc, pl, parents)
    o = out["out"].float().cpu().reshape(-1, w.D)
    assert_float_parity(o, ref_o, w.torch_dtype, "out")
    assert np.abs(out["lse"].cpu().reshape(-1).numpy() - ref_l).max() <= float_tol(w.torch_dtype)


def test_paged_equals_contiguous_bitwise_when_pages_are_in_order():
    # pages taken in order (page p of sequence b = b * max_pages + p) hold
    # exactly the contiguous cache: both calls run the same chunks, so the
    # outputs agree to rounding, and with 64-row pages bit for bit
    w = I.scaled(I.WORKLOADS["llama8b"], B=2, prefix=1024)
    parents = I.product_tree_parents((4, 4, 2, 2))
    T = len(parents)
    pl = torch.tensor([1024, 640], dtype=torch.int32)
    inp = I.attention_inputs(w, T, prefix_len=pl)
    ps = 64
    mp = w.S_max // ps
    kp = inp["k_cache"].reshape(w.B, w.Hkv, mp, ps, w.D).permute(0, 2, 1, 3, 4).reshape(w.B * mp, w.Hkv, ps, w.D)
    vp = inp["v_cache"].reshape(w.B, w.Hkv, mp, ps, w.D).permute(0, 2, 1, 3, 4).reshape(w.B * mp, w.Hkv, ps, w.D)
    table = torch.arange(w.B * mp, dtype=torch.int32).reshape(w.B, mp)
    dev = {k: v.cuda() for k, v in inp.items()}
    t = Tree(parents)
    a = api.tree_attention(dev["q"], dev["k_tree"], dev["v_tree"], dev["k_cache"], dev["v_cache"], dev["prefix_len"],
                           t, max_prefix=w.S_max)
    b = api.tree_attention_paged(dev["q"], dev["k_tree"], dev["v_tree"], kp.contiguous().cuda(),
                                 vp.contiguous().cuda(), table.cuda(), dev["prefix_len"], t, max_prefix=w.S_max)
    torch.cuda.synchronize()
    assert int(a["status"].item()) == 0 and int(b["status"].item()) == 0
    assert torch.equal(a["out"], b["out"])


def test_paged_attention_reports_a_bad_page():
    w = I.scaled(I.WORKLOADS["llama8b"], B=2, prefix=300)
    parents = I.product_tree_parents((2, 2))
    T = len(parents)
    pl = torch.tensor([300, 200], dtype=torch.int32)
    inp = I.attention_inputs(w, T, prefix_len=pl)
    pc = I.paged_cache(w, 16, pl, room=T)
    table = pc["block_table"].clone()
    table[1, 3] = 10 ** 6  # a block sequence 1 needs
    dev = {k: v.cuda() for k, v in inp.items()}
    out = api.tree_attention_paged(dev["q"], dev["k_tree"], dev["v_tree"], pc["k_pages"].cuda(),
                                   pc["v_pages"].cuda(), table.cuda(), dev["prefix_len"], Tree(parents))
    torch.cuda.synchronize()
    assert int(out["status"].item()) & B.STATUS_BAD_PAGE
    # sequence 0 is unaffected
    S_max = table.shape[1] * 16
    kc = oracle.gather_pages(pc["k_pages"], pc["block_table"], pl, S_max)
    vc = oracle.gather_pages(pc["v_pages"], pc["block_table"], pl, S_max)
    ref_o, _ = oracle.tree_attention(inp["q"], inp["k_tree"], inp["v_tree"], kc, vc, pl, parents)
    n0 = T * w.Hq
    assert_float_parity(out["out"].float().cpu().reshape(-1, w.D)[:n0], ref_o[:n0], w.torch_dtype, "out[0]")


@pytest.mark.parametrize("dtype,ps", [("bf16", 16), ("bf16", 64), ("f32", 5)])
def test_paged_commit_parity(dtype, ps):
    w = I.scaled(I.WORKLOADS["llama8b" if dtype == "bf16" else "tiny"], B=4, prefix=200)
    parents = I.product_tree_parents((3, 2, 2))
    T = len(parents)
    pl = torch.tensor([0, 15, 200, 63], dtype=torch.int32)
    pc = I.paged_cache(w, ps, pl, room=T)
    g = torch.Generator().manual_seed(3)
    kt = torch.randn((w.B, T, w.Hkv, w.D), generator=g).to(w.torch_dtype)
    vt = torch.randn((w.B, T, w.Hkv, w.D), generator=g).to(w.torch_dtype)
    path = torch.tensor([[0, 1, 4, 10], [0, 3, -1, -1], [0, 2, 8, 21], [0, -1, -1, -1]], dtype=torch.int32)
    ln = torch.tensor([4, 2, 4, 1], dtype=torch.int32)
    kp, vp = pc["k_pages"].cuda(), pc["v_pages"].cuda()
    out = api.kv_commit_paged(kp, vp, kt.cuda(), vt.cuda(), pc["block_table"].cuda(), path.cuda(), ln.cuda(),
                              pl.cuda())
    torch.cuda.synchronize()
    rk, rv, npl, st = oracle.kv_commit_paged(pc["k_pages"], pc["v_pages"], kt, vt, pc["block_table"], path, ln, pl)
    assert st == 0 and int(out["status"].item()) == 0
    assert out["new_prefix_len"].cpu().tolist() == npl.tolist()
    assert torch.equal(kp.cpu(), rk) and torch.equal(vp.cpu(), rv)


def test_paged_commit_refuses_a_block_it_does_not_own():
    w = I.scaled(I.WORKLOADS["llama8b"], B=2, prefix=100)
    parents = I.product_tree_parents((2, 2))
    T = len(parents)
    pl = torch.tensor([100, 10], dtype=torch.int32)
    pc = I.paged_cache(w, 16, pl, room=0)  # no room past the prefix: sequence 0 owns blocks 0..6 (112 slots)
    kt = torch.zeros((w.B, T, w.Hkv, w.D), dtype=w.torch_dtype)
    path = torch.tensor([[0, 1, 3], [0, 2, 6]], dtype=torch.int32)
    ln = torch.tensor([3, 3], dtype=torch.int32)
    pl2 = torch.tensor([111, 10], dtype=torch.int32)  # positions 111..113 need block 7 of sequence 0
    kp, vp = pc["k_pages"].cuda(), pc["v_pages"].cuda()
    out = api.kv_commit_paged(kp, vp, kt.cuda(), kt.cuda(), pc["block_table"].cuda(), path.cuda(), ln.cuda(),
                              pl2.cuda())
    torch.cuda.synchronize()
    assert int(out["status"].item()) & B.STATUS_CACHE_OVERFLOW
    assert out["new_prefix_len"].cpu().tolist() == [111, 13]


def test_step_with_per_sequence_trees_and_paged_cache():
    # the whole step (heads -> paged attention -> greedy verify -> paged commit)
    # with a tree per sequence; verify and commit checked against the oracle
    w = I.scaled(I.WORKLOADS["ragged_paged_b8"], B=3, d=256, V=1000, prefix_range=(100, 700))
    trees = I.workload_tree(w)
    T = max(len(t) for t in trees)
    hin = {k: v.cuda() for k, v in I.head_inputs(w).items()}
    ain = I.attention_inputs(w, T)
    pc = I.paged_cache(w, w.page_size, ain["prefix_len"], room=T, capacity=w.max_prefix + T)
    step = api.MedusaStep(B=w.B, d=w.d, V=w.V, K=w.K, Hq=w.Hq, Hkv=w.Hkv, D=w.D, S_max=w.S_max, parents=trees,
                          dtype=w.torch_dtype, max_prefix=w.max_prefix, device="cuda", page_size=w.page_size,
                          max_pages=pc["block_table"].shape[1], num_pages=pc["k_pages"].shape[0])
    step.heads(hin["h"], hin["W_res"], hin["W_head"], hin["root_token"])
    torch.cuda.synchronize()
    node_tokens = step.node_tokens.cpu()
    logits = I.boosted_target_logits(w, trees, node_tokens)
    kp, vp, bt = pc["k_pages"].cuda(), pc["v_pages"].cuda(), pc["block_table"].cuda()
    dev = {k: v.cuda() for k, v in ain.items()}
    new_pl = torch.empty_like(dev["prefix_len"])
    step.run(h=hin["h"], W_res=hin["W_res"], W_head=hin["W_head"], root_token=hin["root_token"], q=dev["q"],
             k_tree=dev["k_tree"], v_tree=dev["v_tree"], k_cache=kp, v_cache=vp, prefix_len=dev["prefix_len"],
             new_prefix_len=new_pl, target=logits.cuda(), block_table=bt)
    torch.cuda.synchronize()
    assert int(step.status.item()) == 0
    maxd = step.tree.max_depth
    path = np.full((w.B, maxd), -1, np.int32)
    ln = np.zeros(w.B, np.int32)
    for b, par in enumerate(trees):
        Tb = len(par)
        pb, lb, _ = oracle.verify_greedy(logits[b:b + 1, :Tb], node_tokens[b:b + 1, :Tb], par, maxd)
        path[b], ln[b] = pb[0], lb[0]
    assert np.array_equal(step.accept_path.cpu().numpy(), path)
    rk, rv, npl, st = oracle.kv_commit_paged(pc["k_pages"], pc["v_pages"], ain["k_tree"], ain["v_tree"],
                                             pc["block_table"], path, ln, ain["prefix_len"])
    assert st == 0 and new_pl.cpu().tolist() == npl.tolist()
    assert torch.equal(kp.cpu(), rk) and torch.equal(vp.cpu(), rv)
    # the attention output against the oracle on the gathered cache, per sequence
    S_max = pc["block_table"].shape[1] * w.page_size
    kc = oracle.gather_pages(pc["k_pages"], pc["block_table"], ain["prefix_len"], S_max)
    vc = oracle.gather_pages(pc["v_pages"], pc["block_table"], ain["prefix_len"], S_max)
    o = step.attn_out.float().cpu()
    for b, par in enumerate(trees):
        Tb = len(par)
        ref_o, _ = oracle.tree_attention(ain["q"][b:b + 1, :Tb], ain["k_tree"][b:b + 1, :Tb],
                                         ain["v_tree"][b:b + 1, :Tb], kc[b:b + 1], vc[b:b + 1],
                                         ain["prefix_len"][b:b + 1], par)
        assert_float_parity(o[b, :Tb].reshape(-1, w.D), ref_o, w.torch_dtype, f"out[{b}]")
