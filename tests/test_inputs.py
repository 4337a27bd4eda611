"""The seeded input generators: the same workload gives the same tensors on
every call (the CUDA path and the oracle are fed from separate calls), and
every workload's shapes are consistent with its description."""
import torch

from medusa_tree_speculative_heads_b200 import inputs as I


def _small(name):
    w = I.WORKLOADS[name]
    return I.scaled(w, B=min(w.B, 2), d=64, V=300, prefix=min(w.max_prefix, 96),
                    prefix_range=None if w.prefix_range is None else (8, 96))


def test_generators_are_deterministic():
    for name in ("tiny", "llama8b", "stoch_b64", "ragged_paged_b8", "llama8b_incache"):
        w = _small(name)
        trees = I.sequence_trees(w)
        T = max(len(t) for t in trees)
        for gen in (lambda: I.head_inputs(w), lambda: I.attention_inputs(w, T)):
            a, b = gen(), gen()
            assert a.keys() == b.keys()
            for k in a:
                assert torch.equal(a[k], b[k]), (name, k)
        if w.stochastic:
            a, b = I.stochastic_inputs(w, trees[0]), I.stochastic_inputs(w, trees[0])
            for k in a:
                assert torch.equal(a[k], b[k]), (name, k)
            # p is the softmax of the logits at the stated temperature
            p = torch.softmax(a["logits"] / I.STOCH_TEMPERATURE, dim=-1)
            assert torch.allclose(p, a["p"], atol=1e-6)


def test_workload_shapes():
    for name, w in I.WORKLOADS.items():
        trees = I.sequence_trees(w)
        assert len(trees) == w.B
        for par in trees:
            assert par[0] == -1 and all(0 <= par[i] < i for i in range(1, len(par)))
            assert len(par) <= 128
        assert w.Hq % w.Hkv == 0 and w.D in (64, 128)
        assert w.S_max >= w.max_prefix + (max(len(t) for t in trees) if w.tree_in_cache else 5)
        if w.topk:
            T = 1
            n = 1
            for s in w.topk:
                n *= s
                T += n
            assert len(trees[0]) == T
