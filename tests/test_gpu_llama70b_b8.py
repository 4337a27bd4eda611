"""The 70B-shaped batched workload at its own full sizes, every call against
the fp64 oracle: B=8, d=8192, V=128256, K=4 Medusa heads, top-s (4,4,2,2) =
117 nodes, 64 q-heads / 8 kv-heads, head_dim 128, each sequence's prefix
drawn from U[4096, 8192], greedy verification with match probability 0.7.

The kernels run exactly as the benchmark launches them (the heads' N=16
tensor-core tile with its stream-K split over 8.9 GB of weights; attention
planned for max_prefix 8192).  The oracle recomputes what it can in seconds:
two whole sequences of the heads (every logit and probability), a seeded
sample of attention rows from every sequence, and verification and the
commit whole.  The OpenMP build of the oracle is used for speed; it gives
the serial build's bits (pinned on the CPU).
"""
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

W = I.WORKLOADS["llama70b_b8"]
SAMPLED = (0, 5)          # sequences the oracle recomputes whole


@pytest.fixture
def omp_oracle():
    oracle.use_openmp(True)
    yield oracle
    oracle.use_openmp(False)


@pytest.fixture(scope="module")
def heads_run():
    hin = I.head_inputs(W)
    parents = I.workload_tree(W)
    tree = Tree(parents)
    dev = {k: v.cuda() for k, v in hin.items()}
    out = api.heads(dev["h"], dev["W_res"], dev["W_head"], tree, dev["root_token"], want_logits=True,
                    want_probs=True)
    torch.cuda.synchronize()
    out = {k: v.cpu() for k, v in out.items()}
    del dev
    torch.cuda.empty_cache()
    return hin, parents, out


def test_heads_full_size_sampled_sequences(heads_run, omp_oracle):
    hin, parents, out = heads_run
    assert int(out["status"].item()) == 0
    tol = float_tol(W.torch_dtype)
    ti = out["topk_idx"].numpy()
    tp = out["topk_prob"].numpy()
    for b in SAMPLED:
        ref = omp_oracle.heads(hin["h"], hin["W_res"], hin["W_head"], b_only=b, want_hk=False)
        assert_float_parity(out["logits"][b], ref["logits"][b], W.torch_dtype, f"logits[{b}]")
        assert_float_parity(out["probs"][b], ref["probs"][b], W.torch_dtype, f"probs[{b}]")
        for k in range(W.K):
            check_topk(ti[b, k], ref["logits"][b, k], tol)
            np.testing.assert_allclose(tp[b, k], ref["probs"][b, k, ti[b, k]], rtol=0, atol=tol)


def test_heads_full_size_top_lists_and_tree_exact(heads_run):
    # every sequence: the top-8 list is exactly the oracle's top-s of the
    # kernel's own fp32 logits (the decision taken in the kernel's precision),
    # and the node tokens are exactly the oracle's tree fill of those lists
    hin, parents, out = heads_run
    ti = out["topk_idx"].numpy()
    lg = out["logits"].double().numpy()
    for b in range(W.B):
        for k in range(W.K):
            assert np.array_equal(ti[b, k], oracle.topk(lg[b, k], 8)), (b, k)
    otok, oq = oracle.tree_fill(parents, hin["root_token"], ti, out["topk_prob"].double().numpy())
    assert np.array_equal(out["node_tokens"].numpy(), otok)
    np.testing.assert_array_equal(out["node_q"].double().numpy(), oq)


def test_heads_full_size_against_unrounded_activation(heads_run, omp_oracle):
    # the other reading of the head formula: h^(k) kept exact in fp64 (no
    # bf16 activation); the kernel's logits stay within the bf16 bounds of it
    hin, parents, out = heads_run
    b = 3
    ref = omp_oracle.heads(hin["h"], hin["W_res"], hin["W_head"], b_only=b, want_hk=False, want_probs=False,
                           exact_hk=True)
    assert_float_parity(out["logits"][b], ref["logits"][b], W.torch_dtype, "logits vs exact h^(k)")


def test_attention_full_size_sampled_rows(omp_oracle):
    parents = I.workload_tree(W)
    T = len(parents)
    ain = I.attention_inputs(W, T, canary=float("nan"))   # slots past each prefix hold NaN
    pl = ain["prefix_len"]
    assert int(pl.min()) >= 4096 and int(pl.max()) <= 8192 and len(set(pl.tolist())) > 1
    dev = {k: v.cuda() for k, v in ain.items()}
    out = api.tree_attention(dev["q"], dev["k_tree"], dev["v_tree"], dev["k_cache"], dev["v_cache"],
                             dev["prefix_len"], Tree(parents), max_prefix=W.max_prefix, want_lse=True)
    torch.cuda.synchronize()
    assert int(out["status"].item()) == 0
    o = out["out"].float().cpu()
    lse = out["lse"].cpu()
    assert torch.isfinite(o).all() and torch.isfinite(lse).all()
    g = np.random.default_rng(70)
    rows = np.array([[b, int(g.integers(T)), int(g.integers(W.Hq))] for b in range(W.B) for _ in range(40)] +
                    [[b, T - 1, W.Hq - 1] for b in range(W.B)] + [[b, 0, 0] for b in range(W.B)], dtype=np.int32)
    ref_o, ref_l = omp_oracle.tree_attention(ain["q"], ain["k_tree"], ain["v_tree"], ain["k_cache"],
                                             ain["v_cache"], pl, parents, rows=rows)
    assert_float_parity(o[rows[:, 0], rows[:, 1], rows[:, 2]], ref_o, W.torch_dtype, "attention rows")
    assert np.abs(lse[rows[:, 0], rows[:, 1], rows[:, 2]].numpy() - ref_l).max() <= float_tol(W.torch_dtype)


def test_verify_and_commit_full_size():
    parents = I.workload_tree(W)
    T = len(parents)
    tree = Tree(parents)
    maxd = int(max(oracle.tree_shape(parents)[0]))
    ain = I.attention_inputs(W, T)
    for off in range(2):
        tok = I.random_node_tokens(W, parents, off)
        logits = I.boosted_target_logits(W, parents, tok, seed_offset=off)   # bf16 [8, 117, 128256]
        out = api.tree_verify(B.GREEDY, logits.cuda(), tok.cuda(), tree)
        torch.cuda.synchronize()
        path, ln, bonus = oracle.verify_greedy(logits, tok, parents, maxd)
        assert np.array_equal(out["accept_path"].cpu().numpy(), path)
        assert np.array_equal(out["accept_len"].cpu().numpy(), ln)
        assert np.array_equal(out["bonus"].cpu().numpy(), bonus)
        assert ln.max() > 1
        kc, vc = ain["k_cache"].cuda(), ain["v_cache"].cuda()
        res = api.kv_commit(kc, vc, ain["k_tree"].cuda(), ain["v_tree"].cuda(), out["accept_path"],
                            out["accept_len"], ain["prefix_len"].cuda())
        torch.cuda.synchronize()
        okc, ovc, onpl, _ = oracle.kv_commit(ain["k_cache"], ain["v_cache"], ain["k_tree"], ain["v_tree"], path, ln,
                                             ain["prefix_len"])
        assert int(res["status"].item()) == 0
        assert np.array_equal(res["new_prefix_len"].cpu().numpy(), onpl)
        assert torch.equal(kc.cpu(), okc) and torch.equal(vc.cpu(), ovc)
