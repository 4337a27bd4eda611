"""tree_attention on the GPU against the fp64 oracle (same seeded inputs)."""
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


def run(w, parents, prefix=None, canary=None, rows=None, max_prefix=0, scale=0.0):
    T = len(parents)
    pl = None if prefix is None else torch.tensor(prefix, dtype=torch.int32)
    inp = I.attention_inputs(w, T, canary=canary, prefix_len=pl)
    dev = {k: v.cuda() for k, v in inp.items()}
    tree = Tree(parents)
    out = api.tree_attention(dev["q"], dev["k_tree"], dev["v_tree"], dev["k_cache"], dev["v_cache"],
                             dev["prefix_len"], tree, scale=scale, max_prefix=max_prefix, want_lse=True)
    torch.cuda.synchronize()
    ref_o, ref_l = oracle.tree_attention(inp["q"], inp["k_tree"], inp["v_tree"], inp["k_cache"], inp["v_cache"],
                                         inp["prefix_len"], parents, scale=scale, rows=rows)
    return inp, out, ref_o, ref_l


def compare(w, parents, out, ref_o, ref_l, rows=None):
    dt = w.torch_dtype
    o = out["out"].float().cpu()
    l = out["lse"].cpu()
    if rows is not None:
        rows = np.asarray(rows)
        o = o[rows[:, 0], rows[:, 1], rows[:, 2]]
        l = l[rows[:, 0], rows[:, 1], rows[:, 2]]
    else:
        o = o.reshape(-1, o.shape[-1])
        l = l.reshape(-1)
    assert_float_parity(o, ref_o, dt, "out")
    assert np.abs(l.numpy() - ref_l).max() <= float_tol(dt)
    assert int(out["status"].item()) == 0


CASES = [
    # name, overrides, tree, prefix per sequence
    ("tiny", {}, "workload", None),                                        # fp32, T=7, D=64, S=64
    ("tiny", dict(B=2, Hq=8, Hkv=2, D=128, prefix=100), (3, 2), [100, 0]),  # fp32, GQA, empty prefix
    ("llama8b", dict(Hq=4, Hkv=4, D=64, prefix=100), (2, 2), None),         # bf16, G=1, D=64
    ("llama8b", dict(B=3, prefix=300), (4, 4, 2, 2), [0, 1, 300]),          # 117 nodes, ragged prefixes
    ("llama8b", dict(B=2, Hq=64, Hkv=8, prefix=5000), (4, 4, 2, 2), [4097, 5000]),  # G=8, several splits
    ("stoch_b64", dict(B=4), "workload", None),                             # 32-node random tree, S=1024
    ("llama8b", dict(prefix=200), (1, 1, 1, 1, 1, 1, 1), None),             # chain tree (causal)
    ("llama8b", dict(prefix=77), (), None),                                 # T=1: plain decode
    ("llama8b", dict(B=2, Hq=16, Hkv=4, D=64, prefix=700), (4, 4, 2, 2), [700, 65]),  # D=64, two tiles per CTA
]


@pytest.mark.parametrize("name,kw,tree,prefix", CASES)
def test_attention_parity(name, kw, tree, prefix):
    w = I.scaled(I.WORKLOADS[name], **kw)
    parents = I.workload_tree(w) if tree == "workload" else I.product_tree_parents(tree)
    inp, out, ref_o, ref_l = run(w, parents, prefix=prefix, canary=float("nan"))
    compare(w, parents, out, ref_o, ref_l)


def test_attention_parity_llama8b_full_size():
    w = I.WORKLOADS["llama8b"]
    parents = I.workload_tree(w)
    inp, out, ref_o, ref_l = run(w, parents, max_prefix=w.prefix)
    compare(w, parents, out, ref_o, ref_l)


@pytest.mark.parametrize("name", ["long32k", "long128k"])
def test_attention_long_context_sampled_rows(name):
    w = I.WORKLOADS[name]
    parents = I.workload_tree(w)
    g = np.random.default_rng(3)
    rows = np.stack([np.zeros(48, int), g.integers(0, len(parents), 48), g.integers(0, w.Hq, 48)], axis=1)
    rows[0] = [0, 0, 0]
    rows[1] = [0, len(parents) - 1, w.Hq - 1]
    inp, out, ref_o, ref_l = run(w, parents, rows=rows, max_prefix=w.prefix)
    compare(w, parents, out, ref_o, ref_l, rows=rows)


def test_attention_custom_scale_and_max_prefix():
    w = I.scaled(I.WORKLOADS["llama8b"], B=2, prefix=640)
    parents = I.product_tree_parents((3, 2))
    inp, out, ref_o, ref_l = run(w, parents, prefix=[640, 320], max_prefix=640, scale=0.05)
    compare(w, parents, out, ref_o, ref_l)


def test_attention_bad_prefix_sets_status():
    w = I.scaled(I.WORKLOADS["llama8b"], prefix=256)
    parents = I.product_tree_parents((2,))
    T = len(parents)
    inp = {k: v.cuda() for k, v in I.attention_inputs(w, T).items()}
    tree = Tree(parents)
    inp["prefix_len"][0] = 300     # above max_prefix = 256
    out = api.tree_attention(inp["q"], inp["k_tree"], inp["v_tree"], inp["k_cache"], inp["v_cache"],
                             inp["prefix_len"], tree, max_prefix=256)
    torch.cuda.synchronize()
    assert int(out["status"].item()) & B.STATUS_BAD_PREFIX
    assert torch.isfinite(out["out"].float()).all()


def test_attention_back_to_back_calls_identical():
    # many launches in a row (the timing loop's pattern): every call must end
    # with status 0 and give bit-identical output; catches pipeline waits that
    # pass early or late depending on how far the tensor cores have run ahead
    w = I.scaled(I.WORKLOADS["llama8b"], prefix=8192)
    parents = I.workload_tree(w)
    T = len(parents)
    inp = I.attention_inputs(w, T)
    dev = {k: v.cuda() for k, v in inp.items()}
    tree = Tree(parents)
    outs = []
    for _ in range(12):
        out = api.tree_attention(dev["q"], dev["k_tree"], dev["v_tree"], dev["k_cache"], dev["v_cache"],
                                 dev["prefix_len"], tree, max_prefix=w.prefix)
        outs.append(out)
    torch.cuda.synchronize()
    for out in outs:
        assert int(out["status"].item()) == 0
        assert torch.equal(out["out"], outs[0]["out"])
    rows = np.array([[0, 0, 0], [0, T - 1, w.Hq - 1], [0, 5, 3], [0, 60, 17]])
    ref_o, ref_l = oracle.tree_attention(inp["q"], inp["k_tree"], inp["v_tree"], inp["k_cache"], inp["v_cache"],
                                         inp["prefix_len"], parents, rows=rows)
    o = outs[-1]["out"].float().cpu()[rows[:, 0], rows[:, 1], rows[:, 2]]
    assert_float_parity(o, ref_o, w.torch_dtype, "out")
