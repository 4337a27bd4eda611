"""One candidate tree per sequence (ragged trees) through every call, against
the fp64 oracle run sequence by sequence on each sequence's own tree.

The [B, T, ...] arrays keep T = the largest tree's node count; rows past a
sequence's own tree are filled with NaN (or -1 for token ids) here, to show
that no call reads them."""
import numpy as np
import pytest
import torch

import oracle
from helpers import assert_float_parity, assert_top_lists_exact, float_tol
from medusa_tree_speculative_heads_b200 import api
from medusa_tree_speculative_heads_b200 import binding as B
from medusa_tree_speculative_heads_b200 import inputs as I
from medusa_tree_speculative_heads_b200.binding import Tree

pytestmark = pytest.mark.gpu


def ragged_trees(n, seed=0):
    """n parent arrays of mixed shapes and sizes (1 to 117 nodes), depth <= 5,
    sibling ranks < 8."""
    g = torch.Generator().manual_seed(seed)
    pool = [I.product_tree_parents((4, 4, 2, 2)), I.product_tree_parents((2,)), [-1],
            I.random_tree_parents(40, 5, 6, g), I.product_tree_parents((3, 2, 1)),
            I.random_tree_parents(64, 4, 8, g), I.product_tree_parents((1, 1, 1, 1))]
    return [pool[i % len(pool)] for i in range(n)]


def pad_rows(x, sizes, value):
    """x [B, T, ...]: rows t >= sizes[b] of sequence b set to value."""
    x = x.clone()
    for b, Tb in enumerate(sizes):
        x[b, Tb:] = value
    return x


@pytest.mark.parametrize("name,kw", [
    ("llama8b", dict(B=4, d=256, V=2000, K=4)),   # bf16: tensor-core heads kernel
    ("tiny", dict(B=3, d=256, V=1500, K=4)),      # fp32: general path
])
def test_heads_tree_fill_per_sequence(name, kw):
    w = I.scaled(I.WORKLOADS[name], **kw)
    trees = ragged_trees(w.B, seed=1)
    tree = Tree(trees)
    assert tree.ntrees == w.B and tree.T == max(len(t) for t in trees)
    inp = I.head_inputs(w)
    dev = {k: v.cuda() for k, v in inp.items()}
    out = api.heads(dev["h"], dev["W_res"], dev["W_head"], tree, dev["root_token"], want_logits=True)
    torch.cuda.synchronize()
    assert int(out["status"].item()) == 0
    ref = oracle.heads(inp["h"], inp["W_res"], inp["W_head"])
    assert_float_parity(out["logits"], ref["logits"], w.torch_dtype, "logits")
    assert_top_lists_exact(out)
    ti = out["topk_idx"].cpu().numpy()
    tp = out["topk_prob"].cpu().numpy()
    nt = out["node_tokens"].cpu().numpy()
    nq = out["node_q"].cpu().numpy()
    for b, par in enumerate(trees):
        Tb = len(par)
        depth, rank = oracle.tree_shape(par)
        want = np.full(tree.T, -1, np.int32)
        want_q = np.zeros(tree.T, np.float32)
        want[0], want_q[0] = int(inp["root_token"][b]), 1.0
        for i in range(1, Tb):
            want[i] = ti[b, depth[i] - 2, rank[i]]
            want_q[i] = tp[b, depth[i] - 2, rank[i]]
        assert np.array_equal(nt[b], want), b
        assert np.array_equal(nq[b], want_q), b


ATTN_CASES = [
    ("llama8b", dict(B=4, prefix=300), [0, 77, 300, 129]),                   # bf16, tcgen05 kernel
    ("llama8b", dict(B=3, Hq=6, Hkv=2, D=64, prefix=200), [5, 200, 64]),      # bf16, G=3: mma.sync kernel
    ("tiny", dict(B=3, Hq=4, Hkv=2, D=64, prefix=64), [10, 0, 64]),          # fp32 kernel
]


@pytest.mark.parametrize("name,kw,prefix", ATTN_CASES)
def test_attention_per_sequence_trees(name, kw, prefix):
    w = I.scaled(I.WORKLOADS[name], **kw)
    trees = ragged_trees(w.B, seed=2)
    sizes = [len(t) for t in trees]
    tree = Tree(trees)
    T = tree.T
    pl = torch.tensor(prefix, dtype=torch.int32)
    inp = I.attention_inputs(w, T, canary=float("nan"), prefix_len=pl)
    for key in ("q", "k_tree", "v_tree"):
        inp[key] = pad_rows(inp[key], sizes, float("nan"))
    dev = {k: v.cuda() for k, v in inp.items()}
    out = api.tree_attention(dev["q"], dev["k_tree"], dev["v_tree"], dev["k_cache"], dev["v_cache"],
                             dev["prefix_len"], tree, want_lse=True)
    torch.cuda.synchronize()
    assert int(out["status"].item()) == 0
    o = out["out"].float().cpu()
    lse = out["lse"].cpu()
    for b, par in enumerate(trees):
        Tb = sizes[b]
        ref_o, ref_l = oracle.tree_attention(inp["q"][b:b + 1, :Tb], inp["k_tree"][b:b + 1, :Tb],
                                             inp["v_tree"][b:b + 1, :Tb], inp["k_cache"][b:b + 1],
                                             inp["v_cache"][b:b + 1], inp["prefix_len"][b:b + 1], par)
        assert_float_parity(o[b, :Tb].reshape(-1, w.D), ref_o, w.torch_dtype, f"out[{b}]")
        assert np.abs(lse[b, :Tb].reshape(-1).numpy() - ref_l).max() <= float_tol(w.torch_dtype)
        assert (o[b, Tb:] == 0).all(), b
        assert torch.isinf(lse[b, Tb:]).all() and (lse[b, Tb:] < 0).all(), b


def greedy_inputs(w, trees, T):
    """Per-sequence node tokens and boosted target logits, padded to T rows
    (token -1, logits NaN)."""
    g = torch.Generator().manual_seed(5)
    tok = torch.full((w.B, T), -1, dtype=torch.int32)
    logits = torch.full((w.B, T, w.V), float("nan"), dtype=w.torch_dtype)
    for b, par in enumerate(trees):
        Tb = len(par)
        tok[b, :Tb] = torch.randint(0, w.V, (Tb,), generator=g, dtype=torch.int32)
        wb = I.scaled(w, B=1)
        logits[b, :Tb] = I.boosted_target_logits(wb, par, tok[b:b + 1, :Tb], seed_offset=b)[0]
    return tok, logits


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_greedy_verify_per_sequence_trees(dtype):
    base = I.WORKLOADS["llama8b" if dtype == "bf16" else "tiny"]
    w = I.scaled(base, B=6, V=3000)
    trees = ragged_trees(w.B, seed=3)
    tree = Tree(trees)
    tok, logits = greedy_inputs(w, trees, tree.T)
    out = api.tree_verify(B.GREEDY, logits.cuda(), tok.cuda(), tree)
    torch.cuda.synchronize()
    assert int(out["status"].item()) == 0
    for b, par in enumerate(trees):
        Tb = len(par)
        path, ln, bonus = oracle.verify_greedy(logits[b:b + 1, :Tb], tok[b:b + 1, :Tb], par, tree.max_depth)
        assert out["accept_path"][b].tolist() == path[0].tolist(), b
        assert int(out["accept_len"][b]) == int(ln[0]) and int(out["bonus"][b]) == int(bonus[0]), b


@pytest.mark.parametrize("with_q_row", [False, True])
def test_stochastic_verify_per_sequence_trees(with_q_row):
    w = I.scaled(I.WORKLOADS["stoch_b64"], B=5, V=700)
    trees = ragged_trees(w.B, seed=4)
    tree = Tree(trees)
    T = tree.T
    p = torch.full((w.B, T, w.V), float("nan"))
    q = torch.full((w.B, T, w.V), float("nan"))
    tok = torch.full((w.B, T), -1, dtype=torch.int32)
    for b, par in enumerate(trees):
        d = I.stochastic_inputs(I.scaled(w, B=1, seed=w.seed + b), par)
        Tb = len(par)
        p[b, :Tb], q[b, :Tb], tok[b, :Tb] = d["p"][0], d["q"][0], d["node_tokens"][0]
    q_rows, q_row = q, None
    if with_q_row:
        # Medusa-style shared draft rows: q [B, K, V], q_row [B, T] = depth - 1
        K = tree.max_depth
        q_rows = torch.stack([q[b, :K] for b in range(w.B)]).nan_to_num(0.5)
        q_row = np.zeros((w.B, T), np.int32)
        for b, par in enumerate(trees):
            depth, _ = oracle.tree_shape(par)
            q_row[b, :len(par)] = depth - 1
    for seed, step in ((7, 0), (2**64 - 3, 11)):
        out = api.tree_verify(B.STOCHASTIC, p.cuda(), tok.cuda(), tree, q=q_rows.cuda(),
                              q_row=None if q_row is None else torch.from_numpy(q_row).cuda(), seed=seed, step=step)
        torch.cuda.synchronize()
        assert int(out["status"].item()) == 0
        for b, par in enumerate(trees):
            Tb = len(par)
            qb = q_rows[b:b + 1] if with_q_row else q[b:b + 1, :Tb]
            path, ln, bonus, _ = oracle.verify_stochastic(p[b:b + 1, :Tb], qb, tok[b:b + 1, :Tb], par, seed, step,
                                                          tree.max_depth,
                                                          q_row=None if q_row is None else q_row[b, :Tb], b0=b)
            assert out["accept_path"][b].tolist() == path[0].tolist(), (b, seed)
            assert int(out["accept_len"][b]) == int(ln[0]) and int(out["bonus"][b]) == int(bonus[0]), (b, seed)


def test_step_with_per_sequence_trees():
    # heads -> attention -> greedy verify -> commit with one tree per sequence
    w = I.scaled(I.WORKLOADS["llama8b"], B=3, d=256, V=1000, K=4, prefix=200)
    trees = ragged_trees(w.B, seed=6)
    sizes = [len(t) for t in trees]
    step = api.MedusaStep(B=w.B, d=w.d, V=w.V, K=w.K, Hq=w.Hq, Hkv=w.Hkv, D=w.D, S_max=w.S_max, parents=trees,
                          dtype=w.torch_dtype, device="cuda")
    T = step.tree.T
    hin = {k: v.cuda() for k, v in I.head_inputs(w).items()}
    ain = {k: v.cuda() for k, v in I.attention_inputs(w, T).items()}
    step.heads(hin["h"], hin["W_res"], hin["W_head"], hin["root_token"])
    torch.cuda.synchronize()
    node_tokens = step.node_tokens.cpu()
    logits = torch.randn((w.B, T, w.V), generator=torch.Generator().manual_seed(8)).to(w.torch_dtype)
    new_pl = torch.empty_like(ain["prefix_len"])
    k0, v0 = ain["k_cache"].clone(), ain["v_cache"].clone()
    step.run(h=hin["h"], W_res=hin["W_res"], W_head=hin["W_head"], root_token=hin["root_token"], q=ain["q"],
             k_tree=ain["k_tree"], v_tree=ain["v_tree"], k_cache=ain["k_cache"], v_cache=ain["v_cache"],
             prefix_len=ain["prefix_len"], new_prefix_len=new_pl, target=logits.cuda())
    torch.cuda.synchronize()
    assert int(step.status.item()) == 0
    assert torch.equal(step.node_tokens.cpu(), node_tokens)
    for b, par in enumerate(trees):
        Tb = sizes[b]
        path, ln, bonus = oracle.verify_greedy(logits[b:b + 1, :Tb], node_tokens[b:b + 1, :Tb], par,
                                               step.tree.max_depth)
        assert step.accept_path[b].tolist() == path[0].tolist()
        L = int(ln[0])
        S = int(ain["prefix_len"][b])
        assert int(new_pl[b]) == S + L
        for t in range(L):
            assert torch.equal(ain["k_cache"][b, :, S + t], ain["k_tree"][b, int(path[0][t])])
        assert torch.equal(ain["k_cache"][b, :, :S], k0[b, :, :S])


def test_stochastic_logits_verify_per_sequence_trees():
    w = I.scaled(I.WORKLOADS["stoch_b64"], B=5, V=700)
    trees = ragged_trees(w.B, seed=9)
    tree = Tree(trees)
    T = tree.T
    z = torch.full((w.B, T, w.V), float("nan"))
    q = torch.full((w.B, T, w.V), float("nan"))
    tok = torch.full((w.B, T), -1, dtype=torch.int32)
    for b, par in enumerate(trees):
        d = I.stochastic_inputs(I.scaled(w, B=1, seed=w.seed + b), par)
        Tb = len(par)
        z[b, :Tb], q[b, :Tb], tok[b, :Tb] = d["logits"][0], d["q"][0], d["node_tokens"][0]
    zb = z.bfloat16()
    for seed, step in ((7, 0), (2**64 - 3, 11)):
        out = api.tree_verify_logits(zb.cuda(), 0.7, q.cuda(), tok.cuda(), tree, seed=seed, step=step)
        torch.cuda.synchronize()
        assert int(out["status"].item()) == 0
        for b, par in enumerate(trees):
            Tb = len(par)
            path, ln, bonus, _ = oracle.verify_stochastic_logits(zb[b:b + 1, :Tb], 0.7, q[b:b + 1, :Tb],
                                                                 tok[b:b + 1, :Tb], par, seed, step, tree.max_depth,
                                                                 b0=b)
            assert out["accept_path"][b].tolist() == path[0].tolist(), (b, seed)
            assert int(out["accept_len"][b]) == int(ln[0]) and int(out["bonus"][b]) == int(bonus[0]), (b, seed)
