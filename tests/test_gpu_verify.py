"""tree_verify on the GPU against the oracle: bit-exact paths, lengths and
bonus tokens on identical logits / probabilities and Philox counters."""
import numpy as np
import pytest
import torch

import oracle
from medusa_tree_speculative_heads_b200 import api
from medusa_tree_speculative_heads_b200 import binding as B
from medusa_tree_speculative_heads_b200 import inputs as I
from medusa_tree_speculative_heads_b200.binding import Tree

pytestmark = pytest.mark.gpu


def greedy_case(w, parents, seed_offset=0):
    tok = I.random_node_tokens(w, parents, seed_offset)
    logits = I.boosted_target_logits(w, parents, tok, seed_offset=seed_offset)
    return tok, logits


def run_greedy(parents, tok, logits):
    tree = Tree(parents)
    out = api.tree_verify(B.GREEDY, logits.cuda(), tok.cuda(), tree)
    torch.cuda.synchronize()
    return out


def assert_same(out, ref):
    path, ln, bonus = ref[:3]
    assert np.array_equal(out["accept_len"].cpu().numpy(), ln)
    assert np.array_equal(out["accept_path"].cpu().numpy(), path)
    assert np.array_equal(out["bonus"].cpu().numpy(), bonus)


@pytest.mark.parametrize("name,kw,tree", [
    ("tiny", {}, "workload"),
    ("llama8b", dict(B=4, V=1001), (4, 4, 2, 2)),      # rows not 16-byte aligned: scalar path
    ("llama8b", dict(B=2), (4, 4, 2, 2)),              # full vocabulary, 117 nodes
    ("llama70b_b8", dict(V=20000), (4, 4, 2, 2)),       # 8 sequences, match prob 0.7
    ("stoch_b64", dict(B=6, V=5000), "workload"),       # random sparse tree
])
def test_greedy_parity(name, kw, tree):
    w = I.scaled(I.WORKLOADS[name], **kw)
    parents = I.workload_tree(w) if tree == "workload" else I.product_tree_parents(tree)
    for off in range(3):
        tok, logits = greedy_case(w, parents, off)
        out = run_greedy(parents, tok, logits)
        ref = oracle.verify_greedy(logits, tok, parents, max_path=max(oracle.tree_shape(parents)[0]))
        assert_same(out, ref)


def test_greedy_ties_nan_and_float32():
    parents = [-1, 0, 0, 1]
    V = 40
    logits = torch.zeros((2, 4, V))
    logits[0, 0, 7] = 3.0
    logits[0, 0, 5] = 3.0                # tie: 5 wins
    logits[0, 1, :] = float("nan")
    logits[0, 1, 9] = 1.0                # NaN never wins
    logits[1, :, :] = float("nan")       # all NaN: index 0
    tok = torch.tensor([[1, 5, 7, 9], [1, 0, 0, 0]], dtype=torch.int32)
    for dt in (torch.float32, torch.bfloat16):
        out = run_greedy(parents, tok, logits.to(dt))
        ref = oracle.verify_greedy(logits.to(dt), tok, parents, max_path=3)
        assert_same(out, ref)
        assert out["accept_len"].tolist() == [3, 3]


@pytest.mark.parametrize("dt", [torch.bfloat16, torch.float32])
def test_greedy_argmax_edges_full_vocab(dt):
    # the row maxima sit next to NaN in the same 16-byte vector, tie across
    # vocabulary splits and between -0.0 and +0.0, or are -inf; the kernel's
    # per-vector maximum must pick what a plain scan picks.  The tree is a
    # chain whose every token is its parent's prediction, so each row's
    # argmax decides the accepted length (or the bonus token).
    T, V = 7, 32000
    parents = [-1] + list(range(T - 1))
    g = np.random.default_rng(11)
    z = torch.from_numpy(g.standard_normal((2, T, V)).astype(np.float32))
    z[0, 0, 100:108] = float("nan")
    z[0, 0, 103] = 9.0                  # the maximum among NaNs of its vector
    z[0, 1, 30001] = 8.0                # equal maxima in different splits: the lower index
    z[0, 1, 5] = 8.0
    z[0, 2, :] = -float("inf")          # nothing beats -inf: index 0
    z[0, 3, :] = -1.0
    z[0, 3, 17] = -0.0                  # -0.0 and +0.0 are equal: the lower index
    z[0, 3, 21] = 0.0
    z[0, 4, :] = float("nan")
    z[0, 4, V - 1] = -5.0               # the last logit of the row, the rest NaN
    z[0, 5, 8:16] = 7.0                 # a whole vector of equal maxima: its first
    z[0, 6, 24] = 50.0
    z[1, 0, 7] = float("inf")
    z[1, 0, 6] = float("inf")           # two +inf: the lower index
    z[1, 1, :] = float("nan")           # all NaN: index 0
    z = z.to(dt)
    zf = z.float()
    pred = np.zeros((2, T), np.int64)
    for b in range(2):
        for r in range(T):
            row = zf[b, r]
            ok = ~torch.isnan(row)
            pred[b, r] = int(torch.nonzero(row == row[ok].max())[0]) if ok.any() else 0
    assert pred[0].tolist() == [103, 5, 0, 17, V - 1, 8, 24] and pred[1, :2].tolist() == [6, 0]
    tok = torch.zeros((2, T), dtype=torch.int32)
    tok[:, 1:] = torch.from_numpy(pred[:, :-1].astype(np.int32))
    out = run_greedy(parents, tok, z)
    ref = oracle.verify_greedy(z, tok, parents, max_path=T)
    assert_same(out, ref)
    assert out["accept_len"].tolist() == [T, T] and out["bonus"].tolist() == pred[:, -1].tolist()


def test_greedy_draft_equals_target_full_vocab():
    w = I.scaled(I.WORKLOADS["llama8b"], B=2)
    parents = I.workload_tree(w)
    tok, logits = greedy_case(w, parents)
    ch = I.tree_children(parents)
    am = logits.float().argmax(-1)
    for b in range(w.B):
        for u in range(len(parents)):
            if ch[u]:
                tok[b, ch[u][0]] = am[b, u]
    out = run_greedy(parents, tok, logits)
    assert out["accept_len"].tolist() == [5, 5]
    assert_same(out, oracle.verify_greedy(logits, tok, parents, max_path=5))


@pytest.mark.parametrize("dt", [torch.float32, torch.bfloat16])
def test_greedy_full_vocab_row_scan_paths(dt):
    # 117 rows of V=128256: bf16 chunks are staged in shared memory by bulk
    # copies, fp32 chunks (100 KB) are too large for the stage and take the
    # register-load scan; both must pick exactly the oracle's argmax
    w = I.scaled(I.WORKLOADS["llama8b"], B=1)
    parents = I.workload_tree(w)
    tok, logits = greedy_case(w, parents, 5)
    logits = logits.to(dt)
    ch = I.tree_children(parents)
    am = logits.float().argmax(-1)
    for u in range(len(parents)):     # the first child of every node is its parent's prediction
        if ch[u]:
            tok[0, ch[u][0]] = am[0, u]
    out = run_greedy(parents, tok, logits)
    assert_same(out, oracle.verify_greedy(logits, tok, parents, max_path=5))
    assert out["accept_len"].tolist() == [5]


def stoch_case(w, parents):
    d = I.stochastic_inputs(w, parents)
    return d["p"], d["q"], d["node_tokens"]


def run_stoch(parents, p, q, tok, seed, step, q_row=None):
    tree = Tree(parents)
    out = api.tree_verify(B.STOCHASTIC, p.cuda(), tok.cuda(), tree, q=q.cuda(),
                          q_row=None if q_row is None else torch.as_tensor(q_row, dtype=torch.int32).cuda(),
                          seed=seed, step=step)
    torch.cuda.synchronize()
    return out


@pytest.mark.parametrize("kw", [dict(B=8), dict(B=3, V=777), dict(), dict(B=1), dict(B=12, V=3001)])
def test_stochastic_parity(kw):
    w = I.scaled(I.WORKLOADS["stoch_b64"], **kw)
    parents = I.workload_tree(w)
    p, q, tok = stoch_case(w, parents)
    maxd = int(max(oracle.tree_shape(parents)[0]))
    for seed, step in ((0, 0), (0x123456789ABCDEF0, 17), (2**64 - 1, 2**32 - 1)):
        out = run_stoch(parents, p, q, tok, seed, step)
        ref = oracle.verify_stochastic(p, q, tok, parents, seed, step, maxd)
        assert_same(out, ref)
        assert int(out["status"].item()) == 0


def test_stochastic_many_siblings_and_q_row():
    # a wide product tree (many rejections per node), Medusa-style shared
    # draft rows: q [B, K, V] with q_row[u] = depth(u) - 1
    w = I.scaled(I.WORKLOADS["stoch_b64"], B=5, V=600)
    parents = I.product_tree_parents((6, 3, 2))
    p, q, tok = stoch_case(w, parents)
    depth, _ = oracle.tree_shape(parents)
    K = int(depth.max())
    q_rows = q[:, :K].contiguous()
    q_row = (depth - 1).astype(np.int32)
    for step in range(4):
        out = run_stoch(parents, p, q_rows, tok, 99, step, q_row=q_row)
        ref = oracle.verify_stochastic(p, q_rows, tok, parents, 99, step, K, q_row=q_row)
        assert_same(out, ref)


def test_stochastic_draft_equals_target_accepts_first_children():
    w = I.scaled(I.WORKLOADS["stoch_b64"], B=4)
    parents = I.workload_tree(w)
    p, q, tok = stoch_case(w, parents)
    out = run_stoch(parents, p, p, tok, 3, 1)
    ch = I.tree_children(parents)
    chain = [0]
    while ch[chain[-1]]:
        chain.append(ch[chain[-1]][0])
    for b in range(w.B):
        assert out["accept_path"][b, : len(chain)].tolist() == chain


# ---------------------------------------------------------------------------
# stochastic verification reading logits at a temperature
# ---------------------------------------------------------------------------

def run_stoch_logits(parents, z, tau, q, tok, seed, step, q_row=None):
    tree = Tree(parents)
    out = api.tree_verify_logits(z.cuda(), tau, q.cuda(), tok.cuda(), tree,
                                 q_row=None if q_row is None else torch.as_tensor(q_row, dtype=torch.int32).cuda(),
                                 seed=seed, step=step)
    torch.cuda.synchronize()
    return out


@pytest.mark.parametrize("kw,dtype,tau", [
    (dict(B=8), torch.float32, I.STOCH_TEMPERATURE),
    (dict(B=3, V=777), torch.bfloat16, 1.0),
    (dict(B=12, V=3001), torch.float32, 2.5),
    (dict(B=1), torch.bfloat16, I.STOCH_TEMPERATURE),
    (dict(), torch.bfloat16, I.STOCH_TEMPERATURE),            # the full B=64, V=32000 batch
])
def test_stochastic_logits_parity(kw, dtype, tau):
    # the walk's decisions are integer or fp64; the kernel's exponentials and
    # its cluster-ordered sum of Z differ from the oracle's only in the last
    # bits of P, which no decision of these cases falls within
    w = I.scaled(I.WORKLOADS["stoch_b64"], **kw)
    parents = I.workload_tree(w)
    d = I.stochastic_inputs(w, parents)
    z = d["logits"].to(dtype)
    maxd = int(max(oracle.tree_shape(parents)[0]))
    for seed, step in ((0, 0), (0x123456789ABCDEF0, 17), (2**64 - 1, 2**32 - 1)):
        out = run_stoch_logits(parents, z, tau, d["q"], d["node_tokens"], seed, step)
        ref = oracle.verify_stochastic_logits(z, tau, d["q"], d["node_tokens"], parents, seed, step, maxd)
        assert_same(out, ref)
        assert int(out["status"].item()) == 0


def test_stochastic_logits_wide_tree_and_q_row():
    # many rejections per node (the residual passes re-read P from logits once
    # per node), Medusa-style shared draft rows
    w = I.scaled(I.WORKLOADS["stoch_b64"], B=5, V=600)
    parents = I.product_tree_parents((6, 3, 2))
    d = I.stochastic_inputs(w, parents)
    depth, _ = oracle.tree_shape(parents)
    K = int(depth.max())
    q_rows = d["q"][:, :K].contiguous()
    q_row = (depth - 1).astype(np.int32)
    z = d["logits"].bfloat16()
    for step in range(4):
        out = run_stoch_logits(parents, z, 0.7, q_rows, d["node_tokens"], 99, step, q_row=q_row)
        ref = oracle.verify_stochastic_logits(z, 0.7, q_rows, d["node_tokens"], parents, 99, step, K, q_row=q_row)
        assert_same(out, ref)


def test_stochastic_logits_cold_limit_equals_greedy_kernel():
    # tau -> 0 with a gap of 1.5 above the rest: P is the argmax point mass and
    # the stochastic walk reproduces the greedy kernel's result
    g = np.random.default_rng(5)
    nb, V = 16, 5000
    parents = I.product_tree_parents((4, 2, 2))
    T = len(parents)
    z = g.normal(0, 1, (nb, T, V)).astype(np.float32)
    top = g.integers(V, size=(nb, T))
    z[np.arange(nb)[:, None], np.arange(T)[None, :], top] = z.max(-1) + 1.5
    ch = I.tree_children(parents)
    tok = np.zeros((nb, T), np.int32)
    for b in range(nb):
        for u in range(T):
            for i, c in enumerate(ch[u]):   # the first child takes the parent's argmax half the time
                tok[b, c] = top[b, u] if (i == 0 and g.random() < 0.7) else (top[b, u] + 1 + i) % V
    q = torch.full((nb, T, V), 1.0 / V)
    zt, tt = torch.from_numpy(z), torch.from_numpy(tok)
    out = run_stoch_logits(parents, zt, 1e-3, q, tt, 7, 3)
    gre = api.tree_verify(B.GREEDY, zt.cuda(), tt.cuda(), Tree(parents))
    torch.cuda.synchronize()
    for k in ("accept_path", "accept_len", "bonus"):
        assert torch.equal(out[k], gre[k]), k
    assert len(set(out["accept_len"].tolist())) > 1


def test_stochastic_logits_no_mass_and_bad_temperature():
    V = 256
    parents = [-1, 0]
    z = torch.zeros((2, 2, V))
    z[0, 0] = -float("inf")                                     # no finite maximum
    z[1, 0, 7] = float("nan")                                   # NaN is skipped by the maximum
    q = torch.full((2, 2, V), 1.0 / V)
    tok = torch.tensor([[0, 3], [0, 3]], dtype=torch.int32)
    out = run_stoch_logits(parents, z, 1.0, q, tok, 1, 0)
    ref = oracle.verify_stochastic_logits(z, 1.0, q, tok, parents, 1, 0, 2)
    assert_same(out, ref)
    assert int(out["status"].item()) & B.STATUS_NO_MASS
    for tau in (0.0, -1.0, float("inf"), float("nan"), 1e-320):
        with pytest.raises(B.MedusaError) as e:
            api.tree_verify_logits(z.cuda(), tau, q.cuda(), tok.cuda(), Tree(parents))
        assert e.value.code == B.MEDUSA_ERR_INVALID_ARG


def test_greedy_rows_then_walk_on_two_streams_is_tree_verify():
    # the row scan on one stream, the walk on another after an event: the same
    # result as the one-call greedy verification
    w = I.scaled(I.WORKLOADS["llama8b"], B=3, V=5000)
    parents = I.workload_tree(w)
    tok, logits = greedy_case(w, parents)
    tree = Tree(parents)
    lg, tk = logits.cuda(), tok.cuda()
    ref = api.tree_verify(B.GREEDY, lg, tk, tree)
    nb = B.tree_verify_workspace_size(B.GREEDY, w.B, w.V, tree)
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
    path = torch.full_like(ref["accept_path"], -7)
    ln = torch.full_like(ref["accept_len"], -7)
    bonus = torch.full_like(ref["bonus"], -7)
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    done = torch.cuda.Event()
    with torch.cuda.stream(s1):
        B.tree_verify_greedy_rows(lg, B.dtype_code(lg.dtype), w.B, w.V, tree, ws, nb)
        done.record(s1)
    s2.wait_event(done)
    with torch.cuda.stream(s2):
        B.tree_verify_greedy_walk(tk, w.B, w.V, tree, path, tree.max_depth, ln, bonus, ws, nb)
    torch.cuda.synchronize()
    assert torch.equal(path, ref["accept_path"]) and torch.equal(ln, ref["accept_len"])
    assert torch.equal(bonus, ref["bonus"])
    assert_same({"accept_path": path, "accept_len": ln, "bonus": bonus},
                oracle.verify_greedy(logits, tok, parents, tree.max_depth))


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_greedy_equally_deep_accepted_nodes(dtype):
    # sibling tokens drawn from a 4-token vocabulary repeat often, so several
    # equally deep nodes are accepted: the path must end at the lowest index
    rng = np.random.default_rng(23)
    parents = I.product_tree_parents((3, 2, 2))
    T, V, nb = len(parents), 4, 64
    ch = I.tree_children(parents)
    tok = rng.integers(0, V, (nb, T)).astype(np.int32)
    logits = rng.standard_normal((nb, T, V)).astype(np.float32)
    for b in range(nb):
        for u in range(T):
            if ch[u] and rng.random() < 0.8:
                logits[b, u, tok[b, ch[u][rng.integers(len(ch[u]))]]] = 10.0
    lg = torch.from_numpy(logits).to(dtype)
    out = run_greedy(parents, torch.from_numpy(tok), lg)
    assert_same(out, oracle.verify_greedy(lg, tok, parents, max_path=4))


@pytest.mark.parametrize("paged", [False, True])
def test_greedy_walk_with_commit_equals_walk_then_commit(paged):
    # the fused walk + commit launch gives exactly the walk followed by
    # kv_commit (kv_commit_paged), including a sequence whose cache is full
    from medusa_tree_speculative_heads_b200.api import kv_commit, kv_commit_paged
    w = I.scaled(I.WORKLOADS["llama8b"], B=4, V=3000, Hkv=2, prefix=40)
    parents = I.workload_tree(w)
    tok, logits = greedy_case(w, parents)
    tree = Tree(parents)
    T = len(parents)
    lg, tk = logits.cuda(), tok.cuda()
    nb = B.tree_verify_workspace_size(B.GREEDY, w.B, w.V, tree)
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
    B.tree_verify_greedy_rows(lg, B.dtype_code(lg.dtype), w.B, w.V, tree, ws, nb)
    ain = I.attention_inputs(w, T)
    pl = torch.tensor([0, 17, 40, w.S_max], dtype=torch.int32)          # the last cache is full
    pc = I.paged_cache(w, 16, pl, room=4) if paged else None
    if paged:
        pc["block_table"][3, int(pl[3]) // 16:] = -1                        # and owns no page past its prefix

    def caches():
        if paged:
            return pc["k_pages"].clone().cuda(), pc["v_pages"].clone().cuda()
        return ain["k_cache"].clone().cuda(), ain["v_cache"].clone().cuda()

    kt, vt, table = ain["k_tree"].cuda(), ain["v_tree"].cuda(), pc["block_table"].cuda() if paged else None
    # reference: the walk, then the separate commit
    path = torch.empty((w.B, tree.max_depth), dtype=torch.int32, device="cuda")
    ln = torch.empty(w.B, dtype=torch.int32, device="cuda")
    bonus = torch.empty(w.B, dtype=torch.int32, device="cuda")
    B.tree_verify_greedy_walk(tk, w.B, w.V, tree, path, tree.max_depth, ln, bonus, ws, nb)
    kc1, vc1 = caches()
    if paged:
        r1 = kv_commit_paged(kc1, vc1, kt, vt, table, path, ln, pl.cuda())
    else:
        r1 = kv_commit(kc1, vc1, kt, vt, path, ln, pl.cuda())
    # fused
    kc2, vc2 = caches()
    path2, ln2, bonus2 = torch.full_like(path, -7), torch.full_like(ln, -7), torch.full_like(bonus, -7)
    npl2 = torch.full_like(ln, -7)
    st2 = torch.zeros(1, dtype=torch.int32, device="cuda")
    S_max = kc2.shape[2] if not paged else 0
    B.tree_verify_greedy_walk_commit(tk, w.B, w.V, tree, path2, tree.max_depth, ln2, bonus2, ws, nb, kc2, vc2, kt,
                                     vt, pl.cuda(), npl2, w.Hkv, w.D, S_max, table,
                                     table.shape[1] if paged else 0, 16 if paged else 0,
                                     kc2.shape[0] if paged else 0, B.dtype_code(kc2.dtype), st2)
    torch.cuda.synchronize()
    assert torch.equal(path2, path) and torch.equal(ln2, ln) and torch.equal(bonus2, bonus)
    assert torch.equal(npl2, r1["new_prefix_len"]) and torch.equal(st2, r1["status"])
    assert int(st2.item()) == B.STATUS_CACHE_OVERFLOW
    assert torch.equal(kc2, kc1) and torch.equal(vc2, vc1)
    assert int(npl2[3]) == int(pl[3])          # the overflowing sequence was not committed
