"""medusa_heads on the GPU against the fp64 oracle (same seeded inputs)."""
import numpy as np
import pytest
import torch

import oracle
from helpers import assert_float_parity, assert_top_lists_exact, check_topk, float_tol
from medusa_tree_speculative_heads_b200 import api
from medusa_tree_speculative_heads_b200 import inputs as I
from medusa_tree_speculative_heads_b200.binding import Tree

pytestmark = pytest.mark.gpu


def run_case(w, parents):
    inp = I.head_inputs(w)
    ref = oracle.heads(inp["h"], inp["W_res"], inp["W_head"])
    dev = {k: v.cuda() for k, v in inp.items()}
    tree = Tree(parents) if parents is not None else None
    out = api.heads(dev["h"], dev["W_res"], dev["W_head"], tree, dev["root_token"], want_logits=True,
                    want_probs=True, want_hres=True)
    # the same call without the optional outputs must give the same discrete results
    out2 = api.heads(dev["h"], dev["W_res"], dev["W_head"], tree, dev["root_token"])
    torch.cuda.synchronize()
    return inp, ref, out, out2


def check(w, parents, inp, ref, out, out2):
    dt = w.torch_dtype
    tol = float_tol(dt)
    assert int(out["status"].item()) == 0
    assert_float_parity(out["logits"], ref["logits"], dt, "logits")
    assert_float_parity(out["probs"], ref["probs"], dt, "probs")
    # h^(k): fp32; or bf16 on both sides, equal up to one bf16 step where the
    # fp32 pre-activation sits on a rounding boundary (|step| <= 2^-7 |x|),
    # plus an absolute 1e-3 where SiLU(z) + h nearly cancels (there the fp32
    # accumulation order of z, ~d * 2^-24 relative, moves a tiny value)
    hres = out["h_res"].float().cpu().numpy()
    if dt == torch.float32:
        assert np.abs(hres - ref["hk"]).max() <= tol
    else:
        diff = np.abs(hres - ref["hk"])
        assert (diff <= 2.0 ** -7 * np.abs(ref["hk"]) + 1e-3).all()
        assert (diff == 0).mean() > 0.99
    ti = out["topk_idx"].cpu().numpy()
    tp = out["topk_prob"].cpu().numpy()
    B, K = ti.shape[:2]
    s = min(8, w.V)
    mismatches = 0
    for b in range(B):
        for k in range(K):
            mismatches += check_topk(ti[b, k, :s], ref["logits"][b, k], tol)
            assert (ti[b, k, s:] == -1).all()
            np.testing.assert_allclose(tp[b, k, :s], ref["probs"][b, k, ti[b, k, :s]], rtol=0, atol=tol)
    # decisions in the kernel's own precision: the list is exactly the
    # oracle's top-s of the kernel's own fp32 logits
    assert_top_lists_exact(out)
    assert torch.equal(out["topk_idx"], out2["topk_idx"])
    assert torch.equal(out["topk_prob"], out2["topk_prob"])
    if parents is not None:
        nt = out["node_tokens"].cpu().numpy()
        assert torch.equal(out["node_tokens"], out2["node_tokens"])
        depth, rank = oracle.tree_shape(parents)
        for b in range(B):
            assert nt[b, 0] == int(inp["root_token"][b])
            for i in range(1, len(parents)):
                assert nt[b, i] == ti[b, depth[i] - 2, rank[i]]
        if mismatches == 0:
            otop = np.stack([np.stack([oracle.topk(ref["logits"][b, k], 8) for k in range(K)]) for b in range(B)])
            otok, oq = oracle.tree_fill(parents, inp["root_token"], otop,
                                        np.take_along_axis(ref["probs"], np.maximum(otop, 0), axis=-1))
            assert np.array_equal(nt, otok)
            np.testing.assert_allclose(out["node_q"].cpu().numpy(), oq, rtol=0, atol=tol)
    return mismatches


@pytest.mark.parametrize("name,kw,tree", [
    ("tiny", {}, "workload"),                                           # fp32, d=256, V=1024, (2,2)
    ("tiny", dict(d=1024, V=5003, K=3), (3, 2, 1)),                     # fp32, ragged V
    ("llama8b", dict(d=512, V=3001, K=3), (3, 2, 1)),                   # bf16 register path, ragged V
    ("llama8b", dict(B=3, d=256, V=2000, K=2), (4, 2)),                 # bf16, several sequences
    ("llama8b", dict(B=10, d=128, V=700, K=2), (2, 2)),                 # tensor-core path, N = 16
    ("llama8b", dict(B=17, d=256, V=2003, K=2), (2, 2)),                # N = 32, 7 ragged row segments
    ("llama8b", dict(B=33, d=320, V=1000, K=2), (2,)),                  # N = 48
    ("llama8b", dict(B=64, d=512, V=3001, K=3), (3, 2, 1)),             # N = 64, the largest batch
    ("llama8b", dict(d=8192, V=1500, K=1), (4,)),                       # d too wide for registers
    ("llama8b", dict(d=64, V=5, K=2), (3, 2)),                          # V < 8: missing entries are -1
])
def test_heads_parity(name, kw, tree):
    w = I.scaled(I.WORKLOADS[name], **kw)
    parents = I.workload_tree(w) if tree == "workload" else I.product_tree_parents(tree)
    inp, ref, out, out2 = run_case(w, parents)
    check(w, parents, inp, ref, out, out2)


def test_heads_parity_llama8b_full_size():
    # the 8B-shaped workload at full size: d=4096, V=128256, K=4, 117 nodes
    w = I.WORKLOADS["llama8b"]
    parents = I.workload_tree(w)
    inp, ref, out, out2 = run_case(w, parents)
    check(w, parents, inp, ref, out, out2)
    # the other reading of the formula, h^(k) kept exact in fp64 (no bf16
    # activation): the kernel's logits and probabilities stay within the bf16
    # bounds of it too, so the reading changes no result beyond the tolerance
    exact = oracle.heads(inp["h"], inp["W_res"], inp["W_head"], want_hk=False, exact_hk=True)
    assert_float_parity(out["logits"], exact["logits"], w.torch_dtype, "logits vs exact h^(k)")
    assert_float_parity(out["probs"], exact["probs"], w.torch_dtype, "probs vs exact h^(k)")


def test_heads_parity_batch64_full_size_sampled():
    # B=64, d=4096, V=32000, K=3 at full size; the oracle recomputes three
    # sampled sequences (sequences are independent)
    w = I.WORKLOADS["stoch_b64"]
    inp = I.head_inputs(w)
    dev = {k: v.cuda() for k, v in inp.items()}
    out = api.heads(dev["h"], dev["W_res"], dev["W_head"], None, dev["root_token"], want_logits=True)
    torch.cuda.synchronize()
    assert int(out["status"].item()) == 0
    tol = float_tol(w.torch_dtype)
    ti = out["topk_idx"].cpu().numpy()
    tp = out["topk_prob"].cpu().numpy()
    for b in (0, 37, 63):
        ref = oracle.heads(inp["h"][b:b + 1], inp["W_res"], inp["W_head"])
        assert_float_parity(out["logits"][b:b + 1], ref["logits"], w.torch_dtype, f"logits[{b}]")
        for k in range(w.K):
            check_topk(ti[b, k], ref["logits"][0, k], tol)
            np.testing.assert_allclose(tp[b, k], ref["probs"][0, k, ti[b, k]], rtol=0, atol=tol)
    assert_top_lists_exact(out)


def test_heads_top_list_exact_when_separated():
    # planted vocabulary rows: for each head, eight rows are made parallel to
    # h (so their logits lead by a wide, known margin in a known order); the
    # discrete outputs must then equal the oracle's exactly
    w = I.scaled(I.WORKLOADS["llama8b"], B=1, d=1024, V=20000, K=2)
    parents = I.product_tree_parents((8, 4))
    inp = I.head_inputs(w)
    W_res = torch.zeros_like(inp["W_res"])            # h^(k) = h exactly
    W_head = inp["W_head"].clone()
    hn = inp["h"][0].float()
    g = torch.Generator().manual_seed(5)
    for k in range(w.K):
        rows = torch.randperm(w.V, generator=g)[:8]
        for j, r in enumerate(rows.tolist()):
            W_head[k, r] = (hn * (0.02 - 0.002 * j)).bfloat16()
    ref = oracle.heads(inp["h"], W_res, W_head)
    dev = {k: v.cuda() for k, v in dict(h=inp["h"], W_res=W_res, W_head=W_head, root=inp["root_token"]).items()}
    tree = Tree(parents)
    out = api.heads(dev["h"], dev["W_res"], dev["W_head"], tree, dev["root"], want_logits=True)
    torch.cuda.synchronize()
    otop = np.stack([np.stack([oracle.topk(ref["logits"][0, k], 8) for k in range(w.K)])])
    assert np.array_equal(out["topk_idx"].cpu().numpy(), otop)
    otok, _ = oracle.tree_fill(parents, inp["root_token"], otop, np.take_along_axis(ref["probs"], otop, axis=-1))
    assert np.array_equal(out["node_tokens"].cpu().numpy(), otok)


def test_heads_without_tree():
    w = I.scaled(I.WORKLOADS["llama8b"], d=256, V=999, K=2)
    inp, ref, out, out2 = run_case(w, None)
    check(w, None, inp, ref, out, out2)


def test_heads_rejects_deep_tree():
    w = I.scaled(I.WORKLOADS["tiny"], d=64, V=64, K=1)
    inp = {k: v.cuda() for k, v in I.head_inputs(w).items()}
    tree = Tree(I.product_tree_parents((2, 2)))
    from medusa_tree_speculative_heads_b200.binding import MedusaError
    with pytest.raises(MedusaError):
        api.heads(inp["h"], inp["W_res"], inp["W_head"], tree, inp["root_token"])
