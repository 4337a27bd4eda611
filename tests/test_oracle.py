"""Pins of the fp64 oracle against what the pages and the mathematics fix.

Each test checks the oracle against something other than itself: values the
pages print for their worked examples (tests/golden/), closed forms, brute
force over tiny inputs, library routines (numpy, torch SDPA, cuRAND's host
Philox generator) and statistical laws (chi-square, the expected acceptance
length).  None of these needs a GPU.
"""
import ctypes
import math

import numpy as np
import pytest
import torch

from conftest import read_golden
from medusa_tree_speculative_heads_b200 import inputs as I


# ----------------------------------------------------------------------------
# tree structure and mask
# ----------------------------------------------------------------------------

def _ints(s):
    return [int(x) for x in s.split()]


def test_mask_guide_5_candidates(orc):
    g = read_golden("guide_tree_mask_5.txt")
    par = _ints(g["parents"])
    expect = np.array([[0 if x == "0" else 1 for x in row.split()] for row in g["mask"]])
    allowed = orc.tree_mask(par)
    # the page prints the additive form: 0 = visible, -inf = blocked
    assert np.array_equal(allowed, (expect == 0).astype(np.uint8))


def test_mask_guide_paths_demo(orc):
    g = read_golden("guide_paths_demo.txt")
    paths = [[int(t) for t in p.split(",")] for p in g["paths"].split("|")]
    nodes = _ints(g["nodes"])
    par = _ints(g["parents"])
    expect = np.array([_ints(r) for r in g["mask"]], dtype=np.uint8)
    # the page's construction: unique nodes in first-appearance order; each
    # path position sees that path's prefix up to itself
    order = []
    for p in paths:
        for n in p:
            if n not in order:
                order.append(n)
    assert order == nodes
    via_paths = np.zeros((len(order), len(order)), np.uint8)
    for p in paths:
        for i, n in enumerate(p):
            for a in p[: i + 1]:
                via_paths[order.index(n), order.index(a)] = 1
    assert np.array_equal(via_paths, expect)
    assert np.array_equal(orc.tree_mask(par), expect)


def test_mask_mtp_parent_array_forest(orc):
    g = read_golden("mtp_parent_array.txt")
    par = _ints(g["parents"])
    m = orc.tree_mask(par)
    for row in g["attends"]:
        i, rest = row.split(":")
        assert sorted(np.nonzero(m[int(i)])[0].tolist()) == _ints(rest)
    # a forest is not a single-rooted tree: the step's functions reject it
    with pytest.raises(ValueError):
        orc.tree_shape(par)


def test_mask_rejects_bad_parents(orc):
    for bad in ([-1, 1], [-1, 0, 5], [-1, -2]):
        with pytest.raises(ValueError):
            orc.tree_mask(bad)
    for bad in ([0], [-1, 0, -1], [-1, 2, 0]):
        with pytest.raises(ValueError):
            orc.tree_shape(bad)


def test_tree_shape_hand_example(orc):
    # root 0; children 1,2,3; 4 under 2; 5, 6 under 1 (index order != BFS of
    # a product tree, still topologically ordered)
    par = [-1, 0, 0, 0, 2, 1, 1]
    depth, rank = orc.tree_shape(par)
    assert depth.tolist() == [1, 2, 2, 2, 3, 3, 3]
    assert rank.tolist() == [0, 0, 1, 2, 0, 0, 1]


@pytest.mark.parametrize("s,nodes,leaves", [((2, 2), 7, 4), ((4, 2, 2), 29, 16), ((4, 4, 2, 2), 117, 64)])
def test_product_tree_counts(orc, s, nodes, leaves):
    # [MTP] "Tree-Structured Attention Verification": depth 4 with branching
    # (4,2,2) gives 16 candidate trajectories; the 117-node tree of the
    # workloads is 1 + 4 + 16 + 32 + 64 with 64 leaf paths
    par = orc.product_tree(s)
    assert len(par) == nodes
    has_child = set(par[1:].tolist())
    assert sum(1 for i in range(nodes) if i not in has_child) == leaves
    assert par.tolist() == I.product_tree_parents(s)
    depth, rank = orc.tree_shape(par)
    assert depth.max() == len(s) + 1
    for k, sk in enumerate(s):
        assert rank[depth == k + 2].max() == sk - 1


def test_product_tree_matches_path_enumeration(orc):
    # brute force: enumerate the Cartesian product of rank tuples; every path
    # prefix is a node; compare parent relations as sets of prefixes
    s = (3, 2, 2)
    import itertools
    par = orc.product_tree(s)
    depth, rank = orc.tree_shape(par)

    def prefix_of(i):
        out = []
        while par[i] != -1:
            out.append(int(rank[i]))
            i = par[i]
        return tuple(reversed(out))

    got = sorted(prefix_of(i) for i in range(len(par)))
    want = sorted(set(p[:k] for p in itertools.product(*[range(x) for x in s]) for k in range(len(s) + 1)))
    assert got == want


def test_random_tree_generator_is_valid(orc):
    w = I.WORKLOADS["stoch_b64"]
    par = I.workload_tree(w)
    assert len(par) == 32
    depth, rank = orc.tree_shape(par)
    assert depth.max() <= 4
    assert max(np.bincount(np.array(par[1:]), minlength=32)) <= 6
    assert all(par[i] <= par[i + 1] for i in range(1, 31))   # breadth-first numbering


# ----------------------------------------------------------------------------
# Medusa heads
# ----------------------------------------------------------------------------

def _floats(s):
    return [float(x) for x in s.split()]


def _mat(s):
    return [[float(x) for x in row.split()] for row in s.split("|")]


def test_heads_hand_d4_case_a(orc):
    g = read_golden("guide_head_d4.txt")
    h = torch.tensor([_floats(g["h"])], dtype=torch.float32)
    W_res = torch.zeros((1, 4, 4), dtype=torch.float32)
    W_head = torch.tensor([_mat(g["W_head"])], dtype=torch.float32)
    r = orc.heads(h, W_res, W_head)
    np.testing.assert_array_equal(r["hk"][0, 0], _floats(g["A_hk"]))
    np.testing.assert_array_equal(r["logits"][0, 0], _floats(g["A_logits"]))
    np.testing.assert_allclose(r["probs"][0, 0], _floats(g["A_probs"]), rtol=0, atol=1e-15)
    assert orc.topk(r["logits"][0, 0], 2).tolist() == _ints(g["A_top2"])


def test_heads_hand_d4_case_b_silu_ln3(orc):
    g = read_golden("guide_head_d4.txt")
    h = torch.tensor([_floats(g["h"])], dtype=torch.float32)
    W_res = torch.zeros((1, 4, 4), dtype=torch.float32)
    W_res[0, 0, 0] = math.log(3.0)          # z = (ln 3, 0, 0, 0) up to fp32 rounding of ln 3
    W_head = torch.tensor([_mat(g["W_head"])], dtype=torch.float32)
    r = orc.heads(h, W_res, W_head)
    # fp32(ln 3) differs from ln 3 by < 6e-8; dSiLU/dz < 1 there
    np.testing.assert_allclose(r["hk"][0, 0], _floats(g["B_hk"]), rtol=0, atol=1e-7)
    np.testing.assert_allclose(r["logits"][0, 0], _floats(g["B_logits"]), rtol=0, atol=1e-7)


def test_heads_hand_d4_case_c_bf16_activation(orc):
    # bf16 inputs: h^(k) = SiLU(1) + 1 is stored as the nearest bf16 value
    # before the vocabulary projection; with exact_hk it stays exact
    g = read_golden("guide_head_d4.txt")
    h = torch.tensor([_floats(g["h"])], dtype=torch.float32).bfloat16()
    W_res = torch.zeros((1, 4, 4), dtype=torch.bfloat16)
    W_res[0, 0, 0] = 1.0
    W_head = torch.tensor([_mat(g["W_head"])], dtype=torch.float32).bfloat16()
    r = orc.heads(h, W_res, W_head)
    np.testing.assert_array_equal(r["hk"][0, 0], _floats(g["C_hk_bf16"]))
    np.testing.assert_array_equal(r["logits"][0, 0], _floats(g["C_logits_bf16"]))
    e = orc.heads(h, W_res, W_head, exact_hk=True)
    np.testing.assert_allclose(e["hk"][0, 0], _floats(g["C_hk_exact"]), rtol=0, atol=1e-15)
    np.testing.assert_allclose(e["logits"][0, 0], _floats(g["C_logits_exact"]), rtol=0, atol=1e-15)


def test_openmp_build_is_bit_identical_to_serial(orc):
    # the OpenMP build only spreads independent output elements over threads:
    # heads, attention and greedy verification give the serial build's bits
    g = torch.Generator().manual_seed(21)
    B, d, V, K = 2, 64, 300, 3
    h = torch.randn((B, d), generator=g).bfloat16()
    W_res = (torch.randn((K, d, d), generator=g) / 8).bfloat16()
    W_head = (torch.randn((K, V, d), generator=g) / 8).bfloat16()
    par = [-1, 0, 0, 1, 1, 2]
    T, Hq, Hkv, D, S_max = len(par), 4, 2, 64, 40
    q = torch.randn((B, T, Hq, D), generator=g).bfloat16()
    kt, vt = (torch.randn((B, T, Hkv, D), generator=g).bfloat16() for _ in range(2))
    kc, vc = (torch.randn((B, Hkv, S_max, D), generator=g).bfloat16() for _ in range(2))
    pl = torch.tensor([33, 7], dtype=torch.int32)
    logits = torch.randn((B, T, V), generator=g)
    tok = torch.randint(0, V, (B, T), generator=g, dtype=torch.int32)
    res = []
    for on in (False, True):
        orc.use_openmp(on)
        try:
            hr = orc.heads(h, W_res, W_head)
            o, l = orc.tree_attention(q, kt, vt, kc, vc, pl, par)
            path, ln, bonus = orc.verify_greedy(logits, tok, par, 4)
            res.append((hr["hk"], hr["logits"], hr["probs"], o, l, path, ln, bonus, orc.threads()))
        finally:
            orc.use_openmp(False)
    for a, b in zip(res[0][:-1], res[1][:-1]):
        np.testing.assert_array_equal(a, b)
    assert res[0][-1] == 1 and res[1][-1] >= 1


def test_heads_silu_limits(orc):
    # SiLU(z) -> z for z >> 0 and -> 0 for z << 0
    h = torch.tensor([[1.0, 0.0]], dtype=torch.float32)
    W_res = torch.tensor([[[1000.0, 0.0], [-1000.0, 0.0]]], dtype=torch.float32)
    W_head = torch.eye(2, dtype=torch.float32)[None]
    r = orc.heads(h, W_res, W_head)
    assert r["hk"][0, 0].tolist() == [1001.0, 0.0]


def test_heads_vs_numpy_matmul_and_softmax_sum(orc):
    # random small case against numpy's fp64 matmul (a library routine) with
    # the head formula; softmax rows sum to 1
    g = torch.Generator().manual_seed(11)
    B, d, V, K = 3, 16, 50, 2
    h = torch.randn((B, d), generator=g)
    W_res = torch.randn((K, d, d), generator=g) / 4
    W_head = torch.randn((K, V, d), generator=g) / 4
    r = orc.heads(h, W_res, W_head)
    hn, Wr, Wh = h.double().numpy(), W_res.double().numpy(), W_head.double().numpy()
    for k in range(K):
        z = hn @ Wr[k].T
        hk = z / (1 + np.exp(-z)) + hn
        lg = hk @ Wh[k].T
        np.testing.assert_allclose(r["hk"][:, k], hk, rtol=1e-13, atol=1e-13)
        np.testing.assert_allclose(r["logits"][:, k], lg, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(r["probs"].sum(-1), 1.0, rtol=0, atol=1e-12)
    # bf16 inputs are widened exactly: with W_res = 0, h^(k) = h is already a
    # bf16 value, so the bf16 and fp32 copies give identical results
    Z = torch.zeros_like(W_res)
    rb = orc.heads(h.bfloat16(), Z.bfloat16(), W_head.bfloat16())
    rf = orc.heads(h.bfloat16().float(), Z, W_head.bfloat16().float())
    np.testing.assert_array_equal(rb["logits"], rf["logits"])


def test_round_bf16_ties_and_library(orc):
    # 8 significant bits, ties to even: 1 + 2^-8 lies halfway between 1 and
    # 1 + 2^-7 (odd mantissa) -> 1; 1 + 3 * 2^-8 lies between 1 + 2^-7 (odd)
    # and 1 + 2^-6 (even) -> 1 + 2^-6
    assert orc.round_bf16(1 + 2 ** -8) == 1.0
    assert orc.round_bf16(1 + 3 * 2 ** -8) == 1 + 2 ** -6
    assert orc.round_bf16(-(1 + 3 * 2 ** -8)) == -(1 + 2 ** -6)
    assert orc.round_bf16(1 + 2 ** -8 + 2 ** -30) == 1 + 2 ** -7   # just above halfway
    assert orc.round_bf16(0.0) == 0.0
    # against torch's fp32 -> bf16 conversion (round to nearest even) on
    # values exactly representable in fp32
    x = torch.randn(20000, generator=torch.Generator().manual_seed(4)) * torch.logspace(-30, 30, 20000)
    want = x.bfloat16().double().numpy()
    got = np.array([orc.round_bf16(float(v)) for v in x.double().numpy()])
    assert np.array_equal(got, want)


def test_heads_bf16_stores_hk_as_bf16(orc):
    # for bf16 inputs h^(k) is the bf16 rounding of the exact value, and the
    # logits are the exact products with that rounded activation
    g = torch.Generator().manual_seed(13)
    B, d, V, K = 2, 32, 40, 2
    h = torch.randn((B, d), generator=g).bfloat16()
    W_res = (torch.randn((K, d, d), generator=g) / 4).bfloat16()
    W_head = (torch.randn((K, V, d), generator=g) / 4).bfloat16()
    r = orc.heads(h, W_res, W_head)
    hn, Wr, Wh = h.double().numpy(), W_res.double().numpy(), W_head.double().numpy()
    for k in range(K):
        z = hn @ Wr[k].T
        exact = z / (1 + np.exp(-z)) + hn
        rounded = torch.from_numpy(exact).float().bfloat16().double().numpy()   # fp32 first: tiny double-rounding risk
        assert (r["hk"][:, k] == rounded).mean() > 0.999
        assert (np.abs(r["hk"][:, k] - exact) <= 2.0 ** -8 * np.abs(exact)).all()   # half an ulp of 8 bits
        np.testing.assert_allclose(r["logits"][:, k], r["hk"][:, k] @ Wh[k].T, rtol=1e-12, atol=1e-12)


def test_heads_subset_selection(orc):
    g = torch.Generator().manual_seed(12)
    B, d, V, K = 2, 8, 20, 3
    h = torch.randn((B, d), generator=g)
    W_res = torch.randn((K, d, d), generator=g)
    W_head = torch.randn((K, V, d), generator=g)
    full = orc.heads(h, W_res, W_head)
    one = orc.heads(h, W_res, W_head, b_only=1, k_only=2)
    np.testing.assert_array_equal(one["logits"][1, 2], full["logits"][1, 2])
    assert np.isnan(one["logits"][0]).all() and np.isnan(one["logits"][1, :2]).all()


def test_topk_equals_stable_sort(orc):
    rng = np.random.default_rng(5)
    for trial in range(200):
        n = int(rng.integers(1, 40))
        x = rng.integers(-3, 4, size=n).astype(np.float64)   # many ties
        if trial % 5 == 0:
            x[rng.integers(0, n)] = np.nan
        s = int(rng.integers(1, 9))
        got = orc.topk(x, s)
        keys = np.where(np.isnan(x), np.inf, -x)
        want = np.argsort(keys, kind="stable")
        want = [int(i) for i in want if not np.isnan(x[i])][:s]
        want += [-1] * (s - len(want))
        assert got.tolist() == want


def test_tree_fill_product_tree(orc):
    par = orc.product_tree((2, 3))
    B, K, S = 2, 2, 8
    ti = np.arange(B * K * S, dtype=np.int32).reshape(B, K, S) + 1000
    tp = np.random.default_rng(0).random((B, K, S))
    tok, nq = orc.tree_fill(par, [7, 9], ti, tp)
    # root, then head-1 entries 0..1, then for each depth-2 node head-2 entries 0..2
    assert tok[0].tolist() == [7, 1000, 1001] + [1008, 1009, 1010] * 2
    assert tok[1].tolist() == [9, 1016, 1017] + [1024, 1025, 1026] * 2
    assert nq[0, 0] == 1.0 and nq[1, 4] == tp[1, 1, 1]
    with pytest.raises(ValueError):
        orc.tree_fill(orc.product_tree((2, 2, 2)), [1, 1], ti, tp)   # deeper than K+1


# ----------------------------------------------------------------------------
# tree attention
# ----------------------------------------------------------------------------

def _sdpa_reference(q, kt, vt, kc, vc, pl, allowed_tree, scale=None):
    """torch SDPA in fp64 (a library routine) with an explicit dense boolean
    mask over [prefix ; tree] keys; kv heads repeated for GQA."""
    B, T, Hq, D = q.shape
    Hkv = kt.shape[2]
    G = Hq // Hkv
    outs = []
    for b in range(B):
        S = int(pl[b])
        K_ = torch.cat([kc[b, :, :S].double(), kt[b].double().permute(1, 0, 2)], dim=1)  # [Hkv, S+T, D]
        V_ = torch.cat([vc[b, :, :S].double(), vt[b].double().permute(1, 0, 2)], dim=1)
        K_ = K_.repeat_interleave(G, dim=0)
        V_ = V_.repeat_interleave(G, dim=0)
        Q_ = q[b].double().permute(1, 0, 2)                                              # [Hq, T, D]
        mask = torch.cat([torch.ones((T, S), dtype=torch.bool), torch.as_tensor(allowed_tree, dtype=torch.bool)],
                         dim=1)
        o = torch.nn.functional.scaled_dot_product_attention(Q_, K_, V_, attn_mask=mask, scale=scale)
        outs.append(o.permute(1, 0, 2))                                                  # [T, Hq, D]
    return torch.stack(outs).numpy()


def _attn_case(B, T, Hq, Hkv, D, S_max, pl, seed):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn((B, T, Hq, D), generator=g)
    kt = torch.randn((B, T, Hkv, D), generator=g)
    vt = torch.randn((B, T, Hkv, D), generator=g)
    kc = torch.randn((B, Hkv, S_max, D), generator=g)
    vc = torch.randn((B, Hkv, S_max, D), generator=g)
    return q, kt, vt, kc, vc, torch.tensor(pl, dtype=torch.int32)


def test_attention_chain_tree_is_causal_attention(orc):
    # a chain tree (parent i-1) must equal plain causal attention over
    # prefix + chain, written here with numpy from the softmax definition
    B, T, Hq, Hkv, D, S_max = 2, 5, 4, 2, 8, 12
    q, kt, vt, kc, vc, pl = _attn_case(B, T, Hq, Hkv, D, S_max, [7, 0], 1)
    par = [-1] + list(range(T - 1))
    out, lse = orc.tree_attention(q, kt, vt, kc, vc, pl, par)
    out = out.reshape(B, T, Hq, D)
    for b in range(B):
        S = int(pl[b])
        for h in range(Hq):
            g_ = h // (Hq // Hkv)
            keys = np.concatenate([kc[b, g_, :S].double().numpy(), kt[b, :, g_].double().numpy()])
            vals = np.concatenate([vc[b, g_, :S].double().numpy(), vt[b, :, g_].double().numpy()])
            for i in range(T):
                n = S + i + 1                                   # causal: prefix and chain up to i
                sc = keys[:n] @ q[b, i, h].double().numpy() / math.sqrt(D)
                w = np.exp(sc - sc.max())
                np.testing.assert_allclose(out[b, i, h], (w / w.sum()) @ vals[:n], rtol=1e-12, atol=1e-12)
                np.testing.assert_allclose(lse.reshape(B, T, Hq)[b, i, h], sc.max() + np.log(w.sum()),
                                           rtol=1e-12, atol=1e-12)


def test_attention_single_node_is_decode_attention(orc):
    B, T, Hq, Hkv, D, S_max = 1, 1, 2, 1, 16, 40
    q, kt, vt, kc, vc, pl = _attn_case(B, T, Hq, Hkv, D, S_max, [33], 2)
    out, _ = orc.tree_attention(q, kt, vt, kc, vc, pl, [-1])
    ref = _sdpa_reference(q, kt, vt, kc, vc, pl, np.ones((1, 1)))
    np.testing.assert_allclose(out.reshape(ref.shape), ref, rtol=1e-12, atol=1e-12)


def test_attention_product_tree_vs_sdpa_with_path_mask(orc):
    # mask built from the candidate paths (prefixes of rank tuples), not from
    # parent pointers; GQA with 3 q-heads per kv-head; custom scale
    s = (3, 2)
    par = orc.product_tree(s)
    T = len(par)
    depth, rank = orc.tree_shape(par)
    B, Hq, Hkv, D, S_max = 2, 6, 2, 8, 20
    q, kt, vt, kc, vc, pl = _attn_case(B, T, Hq, Hkv, D, S_max, [20, 3], 3)

    def tuple_of(i):
        t = []
        while par[i] != -1:
            t.append(int(rank[i]))
            i = par[i]
        return tuple(reversed(t))

    tuples = [tuple_of(i) for i in range(T)]
    allowed = np.array([[1 if tuples[i][: len(tuples[j])] == tuples[j] else 0 for j in range(T)] for i in range(T)])
    out, _ = orc.tree_attention(q, kt, vt, kc, vc, pl, par, scale=0.3)
    ref = _sdpa_reference(q, kt, vt, kc, vc, pl, allowed, scale=0.3)
    np.testing.assert_allclose(out.reshape(ref.shape), ref, rtol=1e-12, atol=1e-12)


def test_attention_row_subset_matches_full(orc):
    par = orc.product_tree((2, 2))
    B, T, Hq, Hkv, D, S_max = 2, 7, 4, 4, 8, 10
    q, kt, vt, kc, vc, pl = _attn_case(B, T, Hq, Hkv, D, S_max, [10, 5], 4)
    full, lse = orc.tree_attention(q, kt, vt, kc, vc, pl, par)
    rows = np.array([[1, 6, 3], [0, 0, 0], [1, 2, 1]])
    sub, lsub = orc.tree_attention(q, kt, vt, kc, vc, pl, par, rows=rows)
    for r, (b, i, h) in enumerate(rows):
        n = (b * T + i) * Hq + h
        np.testing.assert_array_equal(sub[r], full[n])
        assert lsub[r] == lse[n]


# ----------------------------------------------------------------------------
# greedy verification
# ----------------------------------------------------------------------------

def _brute_force_greedy(logits, tok, par):
    """Every root-to-leaf path in leaf order; the longest matched prefix wins,
    a strictly longer one replacing it (first found wins ties)."""
    T = len(par)
    pred = [int(np.argmax(logits[u])) for u in range(T)]   # numpy: first maximum
    children = I.tree_children(par)
    leaves = [i for i in range(T) if not children[i]]
    best = [0]
    for leaf in leaves:
        path = []
        cur = leaf
        while cur != -1:
            path.append(cur)
            cur = par[cur]
        path.reverse()
        ok = [0]
        for a, c in zip(path[:-1], path[1:]):
            if tok[c] != pred[a]:
                break
            ok.append(c)
        if len(ok) > len(best):
            best = ok
    return best, pred[best[-1]]


def test_greedy_vs_brute_force(orc):
    rng = np.random.default_rng(7)
    par = orc.product_tree((3, 2, 2))
    T, V = len(par), 12
    children = I.tree_children(par.tolist())
    for trial in range(300):
        logits = rng.standard_normal((1, T, V)).astype(np.float32)
        tok = np.zeros((1, T), np.int32)
        for u in range(T):
            if children[u]:
                picks = rng.choice(V, size=len(children[u]), replace=False)
                tok[0, children[u]] = picks
        # force many matches
        for u in range(T):
            if children[u] and rng.random() < 0.7:
                c = children[u][rng.integers(len(children[u]))]
                logits[0, u, tok[0, c]] = 10.0
        path, ln, bonus = orc.verify_greedy(torch.from_numpy(logits), tok, par, max_path=4)
        want, wb = _brute_force_greedy(logits[0], tok[0], par.tolist())
        assert path[0, : ln[0]].tolist() == want
        assert bonus[0] == wb
        assert (path[0, ln[0]:] == -1).all()


def test_greedy_equally_deep_nodes_take_the_lowest_index(orc):
    # two siblings carry the same (matching) token, and so do their children:
    # nodes 3 and 4 are both accepted at depth 3; the path ends at node 3
    par = [-1, 0, 0, 1, 2]
    V = 10
    logits = torch.zeros((1, 5, V))
    logits[0, 0, 7] = 5.0          # prediction after the root: 7
    logits[0, 1, 4] = 5.0          # after node 1: 4
    logits[0, 2, 4] = 5.0          # after node 2: 4
    logits[0, 3, 1] = 5.0          # after node 3: 1 (the bonus)
    logits[0, 4, 2] = 5.0          # after node 4: 2
    tok = [[0, 7, 7, 4, 4]]
    path, ln, bonus = orc.verify_greedy(logits, tok, par, max_path=3)
    assert ln[0] == 3 and path[0].tolist() == [0, 1, 3] and bonus[0] == 1
    # with duplicated sibling tokens drawn at random, the brute force over
    # paths (first longest in leaf order = lowest index in breadth-first
    # order) still agrees
    rng = np.random.default_rng(17)
    par = orc.product_tree((3, 2, 2))
    T, V = len(par), 4
    children = I.tree_children(par.tolist())
    ties = 0
    for trial in range(300):
        logits = rng.standard_normal((1, T, V)).astype(np.float32)
        tok = rng.integers(0, V, (1, T)).astype(np.int32)     # few tokens: siblings often repeat
        for u in range(T):
            if children[u] and rng.random() < 0.8:
                logits[0, u, tok[0, children[u][rng.integers(len(children[u]))]]] = 10.0
        path, ln, bonus = orc.verify_greedy(torch.from_numpy(logits), tok, par, max_path=4)
        want, wb = _brute_force_greedy(logits[0], tok[0], par.tolist())
        assert path[0, : ln[0]].tolist() == want and bonus[0] == wb
        pred = logits[0].argmax(-1)
        deep = [c for c in range(T) if len(_ancestors(par.tolist(), c)) == ln[0] and
                all(tok[0, a] == pred[par[a]] for a in _ancestors(par.tolist(), c)[1:])]
        ties += len(deep) > 1
    assert ties > 20                  # the tie rule was exercised


def _ancestors(par, c):
    out = []
    while c != -1:
        out.append(c)
        c = par[c]
    return out[::-1]


def test_greedy_draft_equals_target(orc):
    # every node's first child carries the target's prediction at its parent:
    # the whole first-child chain is accepted, bonus = prediction at its end
    par = orc.product_tree((4, 4, 2, 2))
    T, V = len(par), 64
    children = I.tree_children(par.tolist())
    rng = np.random.default_rng(8)
    logits = rng.standard_normal((2, T, V)).astype(np.float32)
    tok = np.zeros((2, T), np.int32)
    for b in range(2):
        for u in range(T):
            if children[u]:
                am = int(np.argmax(logits[b, u]))
                others = [x for x in range(V) if x != am]
                tok[b, children[u]] = [am] + list(rng.choice(others, len(children[u]) - 1, replace=False))
    path, ln, bonus = orc.verify_greedy(torch.from_numpy(logits), tok, par, max_path=5)
    chain = [0]
    while children[chain[-1]]:
        chain.append(children[chain[-1]][0])
    for b in range(2):
        assert ln[b] == 5 and path[b].tolist() == chain
        assert bonus[b] == int(np.argmax(logits[b, chain[-1]]))


def test_greedy_argmax_ties_lowest_index(orc):
    logits = torch.zeros((1, 3, 8), dtype=torch.bfloat16)
    logits[0, 0, 5] = 2.0
    logits[0, 0, 3] = 2.0       # tie: index 3 wins
    logits[0, 1, :] = float("nan")
    logits[0, 1, 6] = 1.0       # NaN never wins
    par = [-1, 0, 1]
    path, ln, bonus = orc.verify_greedy(logits, [[0, 3, 6]], par, max_path=3)
    assert ln[0] == 3 and path[0].tolist() == [0, 1, 2] and bonus[0] == 0   # row 2 all zero -> index 0
    path, ln, bonus = orc.verify_greedy(logits, [[0, 5, 6]], par, max_path=3)
    assert ln[0] == 1 and bonus[0] == 3


def test_greedy_mtp_engine_demo_longest_path(orc):
    # The page's engine uses a fixed score threshold as its acceptance test;
    # reproduce the same accepted set with the greedy rule (a matching child
    # token for every passing node, under a virtual root joining the two
    # roots) and check the committed path and count the page prints.
    g = read_golden("mtp_engine_demo.txt")
    par0 = _ints(g["parents"])
    scores = _floats(g["scores"])
    thr = float(g["threshold"])
    n = len(par0)
    par = [-1] + [p + 1 for p in par0]          # node i -> i+1; roots hang under 0
    T, V = n + 1, 32
    tok = np.zeros((1, T), np.int32)
    logits = torch.zeros((1, T, V))
    children = I.tree_children(par)
    for u in range(T):
        kids = children[u]
        passing = [c for c in kids if scores[c - 1] >= thr]
        # passing siblings share the parent's predicted token; failing ones differ
        pred = 1 + u
        logits[0, u, pred] = 5.0
        for j, c in enumerate(kids):
            tok[0, c] = pred if c in passing else 20 + j
    path, ln, bonus = orc.verify_greedy(logits, tok, par, max_path=T)
    committed = [int(x) - 1 for x in path[0, 1: ln[0]]]
    assert committed == _ints(g["committed_nodes"])
    words = g["tokens"].split()
    assert " ".join(words[i] for i in committed) == g["committed_tokens"]
    assert len(committed) == int(g["count"])
    assert round((len(committed) + 1) / (1 + float(g["overhead"])), 2) == float(g["speedup"])


@pytest.mark.parametrize("branching,pi,V,n_steps", [((2, 2), 0.6, 1024, 20000), ((4, 4, 2, 2), 0.6, 256, 6000),
                                                    ((4, 4, 2, 2), 0.7, 256, 6000)])
def test_greedy_expected_acceptance_length(orc, branching, pi, V, n_steps):
    # [MTP] "Expected Acceptance Length": tau = 1 + sum_k prod_{j<=k} alpha_j.
    # Boost model: at an accepted node with s children, with probability pi
    # one child's token gets +10 on the node's row (so it is the argmax);
    # otherwise the argmax of i.i.d. N(0,1) logits is uniform over V and hits
    # one of the s distinct child tokens with probability s/V.  So depth j is
    # accepted with alpha_j = pi + (1 - pi) s_j / V.
    par = orc.product_tree(branching)
    T, K = len(par), len(branching)
    children = I.tree_children(par.tolist())
    rng = np.random.default_rng(99)
    lens = []
    chunk = 1000
    for c0 in range(0, n_steps, chunk):
        B = min(chunk, n_steps - c0)
        logits = rng.standard_normal((B, T, V)).astype(np.float32)
        tok = np.zeros((B, T), np.int32)
        for u in range(T):
            if children[u]:
                m = len(children[u])
                start = rng.integers(0, V - m + 1, size=B)
                tok[:, children[u]] = start[:, None] + np.arange(m)[None, :]
                hit = rng.random(B) < pi
                which = rng.integers(0, m, size=B)
                bb = np.nonzero(hit)[0]
                logits[bb, u, tok[bb, np.array(children[u])[which[bb]]]] += 10.0
        _, ln, _ = orc.verify_greedy(torch.from_numpy(logits), tok, par, max_path=K + 1)
        lens.append(ln)
    lens = np.concatenate(lens).astype(np.float64)
    alpha = [pi + (1 - pi) * s / V for s in branching]
    tau = 1 + sum(float(np.prod(alpha[:k])) for k in range(1, K + 1))
    se = lens.std() / math.sqrt(len(lens))
    assert abs(lens.mean() - tau) < 4 * se, (lens.mean(), tau, se)


# ----------------------------------------------------------------------------
# Philox and stochastic verification
# ----------------------------------------------------------------------------

def test_philox_known_answers(orc):
    g = read_golden("philox4x32_10_kat.txt")
    for row in g["_rows"]:
        lhs, rhs = row.split("->")
        w = [int(x, 16) for x in lhs.split()]
        want = [int(x, 16) for x in rhs.split()]
        assert orc.philox4x32_10(w[:4], w[4:6]).tolist() == want


def test_philox_vs_curand_host_generator(orc):
    # cuRAND's host Philox4x32-10 generator with seed s emits, as its n-th
    # 4-word block, the block of counter (0, 0, n, 0) under key
    # (s low word, s high word)
    import os
    path = "/usr/local/cuda/lib64/libcurand.so"
    if not os.path.exists(path):
        pytest.skip("libcurand not installed")
    lib = ctypes.CDLL(path)
    for seed in (0, 0x0123456789ABCDEF, 2**64 - 1):
        gen = ctypes.c_void_p()
        assert lib.curandCreateGeneratorHost(ctypes.byref(gen), 161) == 0
        assert lib.curandSetPseudoRandomGeneratorSeed(gen, ctypes.c_ulonglong(seed)) == 0
        n = 4 * 40
        buf = (ctypes.c_uint32 * n)()
        assert lib.curandGenerate(gen, buf, ctypes.c_size_t(n)) == 0
        lib.curandDestroyGenerator(gen)
        got = np.array(buf[:], dtype=np.uint32).reshape(-1, 4)
        key = [seed & 0xFFFFFFFF, seed >> 32]
        for c in range(got.shape[0]):
            assert orc.philox4x32_10([0, 0, c, 0], key).tolist() == got[c].tolist()


def test_residual_normalises_and_closed_form(orc):
    rng = np.random.default_rng(3)
    for _ in range(50):
        V = int(rng.integers(2, 300))
        P = rng.dirichlet(np.ones(V))
        Q = rng.dirichlet(np.ones(V)).astype(np.float32)
        out, W, S = orc.residual(P, Q)
        assert S == int(W.sum()) and S > 0
        assert abs(out.sum() - 1.0) < 1e-12
        r = np.maximum(0.0, P - Q.astype(np.float64))
        np.testing.assert_allclose(out, r / r.sum(), rtol=0, atol=V * 2.0 ** -31)
    # P <= Q everywhere: the residual is empty and P is kept
    P = np.array([0.25, 0.25, 0.5])
    out, W, S = orc.residual(P, np.array([0.25, 0.25, 0.5], np.float32))
    assert S == 0 and out.tolist() == P.tolist()


def _chi2_pvalue(counts, probs):
    from scipy.stats import chisquare
    n = counts.sum()
    probs = np.asarray(probs, np.float64)
    assert (counts[probs == 0] == 0).all()          # impossible outcomes never occur
    keep = probs > 0
    return chisquare(counts[keep], probs[keep] / probs[keep].sum() * n).pvalue


P8 = np.array([0.30, 0.05, 0.15, 0.02, 0.18, 0.10, 0.12, 0.08], np.float32)
Q8 = np.array([0.10, 0.25, 0.05, 0.20, 0.10, 0.05, 0.15, 0.10], np.float32)


@pytest.mark.parametrize("n_children", [1, 3])
def test_stochastic_first_token_follows_target(orc, n_children):
    # [SPEC] "The Acceptance Sampling Rule (Zero Distributional Drift)": the
    # emitted token follows P_target.  Children are drawn i.i.d. from the
    # draft; over 10^6 trials the first emitted token must match p (root row)
    # and, when the first child was accepted, the second must match that
    # child's row.
    N = 1_000_000
    T, V = 1 + n_children, 8
    par = [-1] + [0] * n_children
    rng = np.random.default_rng(100 + n_children)
    p_child = np.array([0.05, 0.4, 0.05, 0.1, 0.1, 0.1, 0.1, 0.1], np.float32)
    p = np.empty((N, T, V), np.float32)
    p[:, 0] = P8
    p[:, 1:] = p_child
    q = np.empty((N, T, V), np.float32)
    q[:, :] = Q8
    tok = np.zeros((N, T), np.int32)
    tok[:, 1:] = rng.choice(V, size=(N, n_children), p=Q8.astype(np.float64) / Q8.sum())
    path, ln, bonus, st = orc.verify_stochastic(p, q, tok, par, seed=1234, step=7, max_path=2)
    assert st == 0
    first = np.where(ln >= 2, tok[np.arange(N), np.maximum(path[:, 1], 0)], bonus)
    assert _chi2_pvalue(np.bincount(first, minlength=V), P8.astype(np.float64)) > 1e-3
    acc = ln >= 2
    second = bonus[acc]                     # the child is a leaf: bonus from its row
    assert _chi2_pvalue(np.bincount(second, minlength=V), p_child.astype(np.float64)) > 1e-3


def test_stochastic_one_hot_draft_closed_form(orc):
    # draft q = one-hot at x: P(accept) = p(x); on rejection the bonus follows
    # p with x removed and renormalised
    N, V, x = 400_000, 8, 2
    par = [-1, 0]
    p = np.broadcast_to(P8, (N, 2, V)).copy()
    q = np.zeros((N, 2, V), np.float32)
    q[:, :, x] = 1.0
    tok = np.full((N, 2), x, np.int32)
    path, ln, bonus, _ = orc.verify_stochastic(p, q, tok, par, seed=77, step=0, max_path=2)
    acc = (ln == 2).mean()
    assert abs(acc - P8[x]) < 4 * math.sqrt(P8[x] * (1 - P8[x]) / N)
    rej = bonus[ln == 1]
    assert (rej != x).all()
    want = P8.astype(np.float64).copy()
    want[x] = 0
    want /= want.sum()
    assert _chi2_pvalue(np.bincount(rej, minlength=V), want) > 1e-3


def test_stochastic_draft_equals_target_accepts_all(orc):
    # q = p: u * q(x) < p(x) whenever p(x) > 0, so every first child is taken
    w = I.scaled(I.WORKLOADS["stoch_b64"], B=3, V=500)
    par = I.workload_tree(w)
    d = I.stochastic_inputs(w, par)
    children = I.tree_children(par)
    path, ln, bonus, _ = orc.verify_stochastic(d["p"], d["p"], d["node_tokens"], par, seed=5, step=1,
                                               max_path=4)
    chain = [0]
    while children[chain[-1]]:
        chain.append(children[chain[-1]][0])
    for b in range(3):
        ok = all(float(d["p"][b, a, int(d["node_tokens"][b, c])]) > 0 for a, c in zip(chain, chain[1:]))
        assert ok
        assert path[b, : ln[b]].tolist() == chain


def test_stochastic_q_row_mapping(orc):
    # q_row maps each node to a shared draft row (Medusa: one row per head)
    w = I.scaled(I.WORKLOADS["stoch_b64"], B=2, V=300)
    par = I.workload_tree(w)
    d = I.stochastic_inputs(w, par)
    depth, _ = orc.tree_shape(par)
    K = int(depth.max())
    q_rows = d["q"][:, :K].clone()
    q_row = (depth - 1).astype(np.int32)
    q_full = torch.stack([q_rows[:, int(r)] for r in q_row], dim=1)
    a = orc.verify_stochastic(d["p"], q_rows, d["node_tokens"], par, 9, 3, 4, q_row=q_row)
    b = orc.verify_stochastic(d["p"], q_full, d["node_tokens"], par, 9, 3, 4)
    for x, y in zip(a[:3], b[:3]):
        assert np.array_equal(x, y)


# ----------------------------------------------------------------------------
# commit
# ----------------------------------------------------------------------------

def test_kv_commit_exact_and_canaries(orc):
    g = torch.Generator().manual_seed(21)
    B, Hkv, S_max, D, T = 3, 2, 16, 4, 7
    kc = torch.full((B, Hkv, S_max, D), -777.0).bfloat16()
    vc = torch.full((B, Hkv, S_max, D), 555.0).bfloat16()
    kt = torch.randn((B, T, Hkv, D), generator=g).bfloat16()
    vt = torch.randn((B, T, Hkv, D), generator=g).bfloat16()
    path = np.array([[0, 2, 5], [0, -1, -1], [0, 1, 4]], np.int32)
    ln = np.array([3, 1, 3], np.int32)
    pl = np.array([4, 0, 14], np.int32)          # sequence 2 would overflow
    k2, v2, npl, st = orc.kv_commit(kc, vc, kt, vt, path, ln, pl)
    assert npl.tolist() == [7, 1, 14] and st == 1
    ek, ev = kc.clone(), vc.clone()
    for b in range(2):
        for t in range(ln[b]):
            ek[b, :, pl[b] + t] = kt[b, path[b, t]]
            ev[b, :, pl[b] + t] = vt[b, path[b, t]]
    assert torch.equal(k2, ek) and torch.equal(v2, ev)


def test_stochastic_rows_checked_one_by_one_match_the_batch(orc):
    # the sequence index only selects the Philox counter: row b on its own
    # (b0 = b) gives what it gives inside the whole batch
    w = I.scaled(I.WORKLOADS["stoch_b64"], B=5, V=300)
    parents = I.workload_tree(w)
    d = I.stochastic_inputs(w, parents)
    maxd = int(max(orc.tree_shape(parents)[0]))
    path, ln, bonus, _ = orc.verify_stochastic(d["p"], d["q"], d["node_tokens"], parents, 11, 3, maxd)
    for b in range(w.B):
        pb, lb, bb, _ = orc.verify_stochastic(d["p"][b:b + 1], d["q"][b:b + 1], d["node_tokens"][b:b + 1],
                                                 parents, 11, 3, maxd, b0=b)
        assert np.array_equal(pb[0], path[b]) and lb[0] == ln[b] and bb[0] == bonus[b]
    # and the counter does matter: row 1 checked as if it were row 0 differs somewhere over a few steps
    diff = False
    for step in range(6):
        p1 = orc.verify_stochastic(d["p"][1:2], d["q"][1:2], d["node_tokens"][1:2], parents, 11, step, maxd, b0=1)
        p0 = orc.verify_stochastic(d["p"][1:2], d["q"][1:2], d["node_tokens"][1:2], parents, 11, step, maxd, b0=0)
        diff |= not (np.array_equal(p1[0], p0[0]) and p1[2][0] == p0[2][0])
    assert diff


def test_gather_pages_identity_table_is_a_reshape(orc):
    # pages laid out in order, one sequence after another: the gather is a reshape
    B, Hkv, D, ps, npg = 2, 3, 8, 4, 5
    pages = torch.randn((B * npg, Hkv, ps, D), dtype=torch.float64)
    table = torch.arange(B * npg, dtype=torch.int32).reshape(B, npg)
    n_pos = torch.tensor([npg * ps, 7], dtype=torch.int32)
    cache = orc.gather_pages(pages, table, n_pos, npg * ps)
    want = pages.reshape(B, npg, Hkv, ps, D).permute(0, 2, 1, 3, 4).reshape(B, Hkv, npg * ps, D)
    assert torch.equal(cache[0], want[0])
    assert torch.equal(cache[1, :, :7], want[1, :, :7]) and (cache[1, :, 7:] == 0).all()


def test_gather_pages_follows_the_table_and_rejects_holes(orc):
    g = torch.Generator().manual_seed(0)
    Hkv, D, ps = 2, 4, 3
    pages = torch.randn((6, Hkv, ps, D), generator=g)
    table = torch.tensor([[4, 1, -1], [0, 5, 2]], dtype=torch.int32)
    cache = orc.gather_pages(pages, table, torch.tensor([5, 9], dtype=torch.int32), 9)
    for b, n in ((0, 5), (1, 9)):
        for s in range(n):
            assert torch.equal(cache[b, :, s], pages[int(table[b, s // ps]), :, s % ps])
    with pytest.raises(ValueError):  # position 6 needs block 2 of sequence 0, which is -1
        orc.gather_pages(pages, table, torch.tensor([7, 0], dtype=torch.int32), 9)


def test_paged_commit_equals_contiguous_commit_through_the_table(orc):
    # committing into pages, then gathering, equals committing into the
    # gathered contiguous cache
    w = I.scaled(I.WORKLOADS["tiny"], B=3, Hkv=2, D=8, prefix=20)
    parents = I.product_tree_parents((2, 2))
    T = len(parents)
    pl = torch.tensor([3, 20, 9], dtype=torch.int32)
    pc = I.paged_cache(w, 4, pl, room=T)
    g = torch.Generator().manual_seed(1)
    kt = torch.randn((w.B, T, w.Hkv, w.D), generator=g)
    vt = torch.randn((w.B, T, w.Hkv, w.D), generator=g)
    path = torch.tensor([[0, 1, 3], [0, 2, -1], [0, -1, -1]], dtype=torch.int32)
    ln = torch.tensor([3, 2, 1], dtype=torch.int32)
    S_max = int((pc["block_table"] >= 0).sum(1).max()) * 4
    kp2, vp2, npl, st = orc.kv_commit_paged(pc["k_pages"], pc["v_pages"], kt, vt, pc["block_table"], path, ln, pl)
    assert st == 0 and npl.tolist() == [6, 22, 10]
    kc, vc, npl_c, st_c = orc.kv_commit(orc.gather_pages(pc["k_pages"], pc["block_table"], pl, S_max),
                                        orc.gather_pages(pc["v_pages"], pc["block_table"], pl, S_max),
                                        kt, vt, path, ln, pl)
    assert st_c == 0 and npl_c.tolist() == npl.tolist()
    assert torch.equal(orc.gather_pages(kp2, pc["block_table"], torch.from_numpy(npl), S_max), kc)
    assert torch.equal(orc.gather_pages(vp2, pc["block_table"], torch.from_numpy(npl), S_max), vc)
    # a commit past the owned pages is refused; the other sequences still commit
    pl4 = torch.tensor([3, 27, 9], dtype=torch.int32)  # sequence 1 owns 7 pages: positions 27, 28 need block 7
    kp4, _, npl4, st4 = orc.kv_commit_paged(pc["k_pages"], pc["v_pages"], kt, vt, pc["block_table"], path, ln, pl4)
    assert st4 == 1 and npl4.tolist() == [6, 27, 10]
    before = orc.gather_pages(pc["k_pages"], pc["block_table"], torch.tensor([0, 28, 0], dtype=torch.int32), 28)
    after = orc.gather_pages(kp4, pc["block_table"], torch.tensor([0, 28, 0], dtype=torch.int32), 28)
    assert torch.equal(before[1], after[1])


# ----------------------------------------------------------------------------
# stochastic verification from logits at a temperature
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("tau", [1.0, 0.7, 2.5])
def test_softmax_temperature_vs_scipy(orc, tau):
    # P = softmax(z / tau): the library routine on the same fp64 values
    from scipy.special import softmax
    rng = np.random.default_rng(31)
    z = rng.normal(0.0, 3.0, 5000)
    z[::97] = -np.inf                                   # masked entries get exactly zero mass
    P = orc.softmax_temperature(z, tau)
    want = softmax(z / tau)
    assert np.abs(P - want).max() <= 1e-15 + 1e-13 * want.max()
    assert (P[::97] == 0).all()
    assert abs(P.sum() - 1.0) < 1e-12
    # one finite entry: a point mass
    z1 = np.full(9, -np.inf)
    z1[4] = -12.5
    assert orc.softmax_temperature(z1, tau).tolist() == [0, 0, 0, 0, 1.0, 0, 0, 0, 0]


def _distinct_sibling_tokens(parents, B, V, rng, favour=None, p_favour=0.0):
    """node tokens [B,T]: siblings distinct; with probability p_favour a
    child gets favour[b, parent] (when no sibling holds it yet)."""
    T = len(parents)
    ch = I.tree_children(parents)
    tok = np.zeros((B, T), np.int32)
    for b in range(B):
        tok[b, 0] = rng.integers(V)
        for u in range(T):
            used = set()
            for c in ch[u]:
                if favour is not None and favour[b, u] not in used and rng.random() < p_favour:
                    t = int(favour[b, u])
                else:
                    t = int(rng.integers(V))
                    while t in used:
                        t = int(rng.integers(V))
                used.add(t)
                tok[b, c] = t
    return tok


def test_stochastic_logits_cold_limit_is_greedy(orc):
    # tau -> 0: gaps of at least 1 between the largest logit and the rest make
    # exp((z - m) / tau) underflow to 0, so P is the argmax point mass; a child
    # is then accepted iff its token is the parent's argmax (u * Q(x) < 1),
    # the residual keeps that point mass, and the bonus is the argmax: the
    # walk is greedy verification (siblings carry distinct tokens)
    B, V = 24, 64
    par = I.product_tree_parents((3, 2, 2))
    T = len(par)
    rng = np.random.default_rng(41)
    z = rng.normal(0.0, 1.0, (B, T, V)).astype(np.float32)
    top = rng.integers(V, size=(B, T))
    z[np.arange(B)[:, None], np.arange(T)[None, :], top] = z.max(axis=-1) + 1.5
    tok = _distinct_sibling_tokens(par, B, V, rng, favour=top, p_favour=0.6)
    q = rng.random((B, T, V)).astype(np.float32)
    q /= q.sum(-1, keepdims=True)
    maxd = int(max(orc.tree_shape(par)[0]))
    gpath, glen, gbonus = orc.verify_greedy(torch.from_numpy(z), torch.from_numpy(tok), par, maxd)
    for seed in (3, 2**63 + 11):
        path, ln, bonus, st = orc.verify_stochastic_logits(torch.from_numpy(z), 1e-3, q, tok, par, seed, 5, maxd)
        assert st == 0
        assert np.array_equal(path, gpath) and np.array_equal(ln, glen) and np.array_equal(bonus, gbonus)
    assert len(set(glen.tolist())) > 2   # the cases reach several depths


def test_stochastic_logits_temperature_scaling_and_shift(orc):
    # P depends on z only through (z - max z) / tau: (2z, 2 tau) and (z + 8, tau)
    # give the same walk bit for bit (z on a 2^-12 grid, so every shift and
    # doubling is exact), bf16 logits give what their fp32 widening gives, and
    # another temperature changes the walk
    w = I.scaled(I.WORKLOADS["stoch_b64"], B=6, V=400)
    par = I.workload_tree(w)
    d = I.stochastic_inputs(w, par)
    z = torch.round(d["logits"] * 4096) / 4096
    maxd = int(max(orc.tree_shape(par)[0]))

    def walk(zz, tau):
        return orc.verify_stochastic_logits(zz, tau, d["q"], d["node_tokens"], par, 17, 2, maxd)[:3]

    base = walk(z, 0.7)
    for other in (walk(z * 2, 1.4), walk(z + 8.0, 0.7)):
        assert all(np.array_equal(x, y) for x, y in zip(base, other))
    zb = z.bfloat16()
    assert all(np.array_equal(x, y) for x, y in zip(walk(zb, 0.7), walk(zb.float(), 0.7)))
    assert not all(np.array_equal(x, y) for x, y in zip(base, walk(z, 3.0)))


def test_stochastic_logits_first_token_follows_target(orc):
    # [SPEC] "The Acceptance Sampling Rule (Zero Distributional Drift)" with P
    # from logits: z = tau * log(P8) makes softmax(z / tau) = P8, so the first
    # emitted token must follow P8 (3 drafted children from Q8)
    N, V, tau = 300_000, 8, 0.6
    par = [-1, 0, 0, 0]
    rng = np.random.default_rng(7)
    z = np.broadcast_to((tau * np.log(P8.astype(np.float64))).astype(np.float32), (N, 4, V)).copy()
    q = np.broadcast_to(Q8, (N, 4, V)).copy()
    tok = np.zeros((N, 4), np.int32)
    tok[:, 1:] = rng.choice(V, size=(N, 3), p=Q8.astype(np.float64) / Q8.sum())
    path, ln, bonus, st = orc.verify_stochastic_logits(torch.from_numpy(z), tau, q, tok, par, 99, 1, 2)
    assert st == 0
    first = np.where(ln >= 2, tok[np.arange(N), np.maximum(path[:, 1], 0)], bonus)
    assert _chi2_pvalue(np.bincount(first, minlength=V), P8.astype(np.float64)) > 1e-3


def test_stochastic_logits_rows_without_mass(orc):
    # a row of -inf logits has no finite maximum: no child is accepted there
    # and the bonus reports no mass
    V = 16
    par = [-1, 0]
    z = torch.zeros((2, 2, V))
    z[0, 0] = -float("inf")
    q = np.full((2, 2, V), 1.0 / V, np.float32)
    tok = np.array([[0, 3], [0, 3]], np.int32)
    path, ln, bonus, st = orc.verify_stochastic_logits(z, 1.0, q, tok, par, 1, 0, 2)
    assert ln[0] == 1 and bonus[0] == 0 and st == 1
    path, ln, bonus, st = orc.verify_stochastic_logits(z[1:], 1.0, q[1:], tok[1:], par, 1, 0, 2, b0=1)
    assert st == 0


# ----------------------------------------------------------------------------
# tree K/V in the cache after the prefix; compaction of every layer
# ----------------------------------------------------------------------------

def test_attention_incache_chain_is_causal_attention_over_the_cache(orc):
    # with the tree's rows in the cache right after the prefix, a chain tree is
    # plain causal attention over cache rows [0, S + i] (torch SDPA, a library
    # routine, with a causal mask offset by S); rows past S + T hold NaN
    B, T, Hq, Hkv, D, S_max = 2, 5, 4, 2, 8, 16
    g = torch.Generator().manual_seed(12)
    q = torch.randn((B, T, Hq, D), generator=g)
    kc = torch.randn((B, Hkv, S_max, D), generator=g)
    vc = torch.randn((B, Hkv, S_max, D), generator=g)
    pl = torch.tensor([9, 0], dtype=torch.int32)
    for b in range(B):
        kc[b, :, int(pl[b]) + T:] = float("nan")
        vc[b, :, int(pl[b]) + T:] = float("nan")
    par = [-1] + list(range(T - 1))
    out, _ = orc.tree_attention_incache(q, kc, vc, pl, par)
    out = out.reshape(B, T, Hq, D)
    for b in range(B):
        S = int(pl[b])
        K_ = kc[b, :, :S + T].double().repeat_interleave(Hq // Hkv, dim=0)
        V_ = vc[b, :, :S + T].double().repeat_interleave(Hq // Hkv, dim=0)
        mask = torch.arange(S + T)[None, :] <= (S + torch.arange(T))[:, None]
        ref = torch.nn.functional.scaled_dot_product_attention(q[b].double().permute(1, 0, 2), K_, V_,
                                                               attn_mask=mask)
        np.testing.assert_allclose(out[b], ref.permute(1, 0, 2).numpy(), rtol=1e-12, atol=1e-12)


def _row_id_cache(n_layers, B, Hkv, S_max, D, dtype=torch.float32):
    # every row's values name it: layer * 1e6 + b * 1e4 + g * 1e3 + row + (lane / D)
    c = torch.empty((n_layers, B, Hkv, S_max, D), dtype=torch.float64)
    for l in range(n_layers):
        for b in range(B):
            for g in range(Hkv):
                c[l, b, g] = (l * 1e6 + b * 1e4 + g * 1e3 + torch.arange(S_max, dtype=torch.float64)[:, None]
                              + torch.arange(D, dtype=torch.float64)[None, :] / D)
    return c.to(dtype)


def test_kv_compact_hand_example(orc):
    # S = 3, path (0, 2, 5): rows 3, 4, 5 <- old rows 3, 5, 8; everything else kept
    kc = _row_id_cache(1, 1, 2, 12, 4)
    vc = -kc
    path = np.array([[0, 2, 5, -1]], np.int32)
    k2, v2, npl, st = orc.kv_compact([kc[0]], [vc[0]], path, np.array([3], np.int32), np.array([3], np.int32), T=7)
    assert st == 0 and npl.tolist() == [6]
    rows = k2[0, 0, 0, :, 0].tolist()
    assert rows == [0, 1, 2, 3, 5, 8, 6, 7, 8, 9, 10, 11]
    assert torch.equal(v2, -k2)


def test_kv_compact_equals_append_then_commit(orc):
    # the tree's rows appended after each prefix and compacted = the commit of
    # the same rows taken as k_tree/v_tree (ragged lengths, every layer alike)
    B, Hkv, S_max, D, T, n_layers = 3, 2, 24, 8, 7, 3
    g = torch.Generator().manual_seed(3)
    kc = torch.randn((n_layers, B, Hkv, S_max, D), generator=g).bfloat16()
    vc = torch.randn((n_layers, B, Hkv, S_max, D), generator=g).bfloat16()
    pl = np.array([5, 0, 17], np.int32)
    path = np.array([[0, 1, 4, 6], [0, 3, -1, -1], [0, 2, 5, -1]], np.int32)
    ln = np.array([4, 2, 3], np.int32)
    k2, v2, npl, st = orc.kv_compact(list(kc), list(vc), path, ln, pl, T)
    assert st == 0 and npl.tolist() == (pl + ln).tolist()
    for l in range(n_layers):
        kt = orc.tree_rows_from_cache(kc[l], pl, T)
        vt = orc.tree_rows_from_cache(vc[l], pl, T)
        kr, vr, npl_r, st_r = orc.kv_commit(kc[l], vc[l], kt, vt, path, ln, pl)
        assert st_r == 0 and npl_r.tolist() == npl.tolist()
        assert torch.equal(k2[l], kr) and torch.equal(v2[l], vr)
    # and each layer compacted on its own gives the same
    k1, v1, _, _ = orc.kv_compact([kc[1]], [vc[1]], path, ln, pl, T)
    assert torch.equal(k1[0], k2[1]) and torch.equal(v1[0], v2[1])


def test_kv_compact_refusals(orc):
    B, Hkv, S_max, D, T = 4, 1, 10, 4, 6
    kc = _row_id_cache(2, B, Hkv, S_max, D)
    vc = kc + 0.5
    pl = np.array([2, 2, 2, 7], np.int32)
    path = np.array([[0, 3, 3], [0, 6, -1], [0, 1, 2], [0, 1, 3]], np.int32)
    ln = np.array([3, 2, 4, 3], np.int32)   # repeated node; node >= T; len > max_path; 7 + 3 >= S_max
    k2, v2, npl, st = orc.kv_compact(list(kc), list(vc), path, ln, pl, T)
    assert st == 3 and npl.tolist() == pl.tolist()
    assert torch.equal(k2, kc) and torch.equal(v2, vc)
