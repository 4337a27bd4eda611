"""The tree's K/V appended to the cache right after each prefix before
attention: tree_attention_incache reads them there, and kv_compact commits
the accepted path of every layer in one in-place launch.  Checked against the
oracle (attention within the dtype's tolerance, compaction bit for bit) and
against the separate-buffer calls on the same values."""
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


def bits_equal(a, b) -> bool:
    """Bit-for-bit equality (NaN payloads included)."""
    it = {2: torch.int16, 4: torch.int32}[a.element_size()]
    return torch.equal(a.cpu().contiguous().view(it), b.cpu().contiguous().view(it))


def append_tree(w, trees, T, prefix, seed=0):
    """Attention inputs with the tree's K/V written into the cache after each
    prefix; cache rows past prefix + T_b hold NaN."""
    pl = torch.tensor(prefix, dtype=torch.int32)
    inp = I.attention_inputs(w, T, canary=float("nan"), prefix_len=pl)
    for b, par in enumerate(trees):
        S, Tb = int(pl[b]), len(par)
        inp["k_cache"][b, :, S:S + Tb] = inp["k_tree"][b, :Tb].transpose(0, 1)
        inp["v_cache"][b, :, S:S + Tb] = inp["v_tree"][b, :Tb].transpose(0, 1)
        inp["k_cache"][b, :, S + Tb:] = float("nan")
        inp["v_cache"][b, :, S + Tb:] = float("nan")
    return inp


ROOM = dict(cache_room=160)   # S_max = max prefix + 160 >= max prefix + T
ATTN_CASES = [
    ("llama8b", dict(B=3, prefix=300, **ROOM), [0, 77, 300], "shared"),             # bf16 tcgen05 kernel
    ("llama8b", dict(B=4, prefix=400, **ROOM), [13, 400, 129, 64], "ragged"),       # tcgen05, a tree per sequence
    ("llama8b", dict(B=2, Hq=6, Hkv=2, D=64, prefix=200, **ROOM), [5, 200], "shared"),   # mma.sync kernel (G = 3)
    ("tiny", dict(B=3, Hq=4, Hkv=2, D=64, prefix=64, **ROOM), [10, 0, 64], "ragged"),    # fp32 kernel
]


@pytest.mark.parametrize("name,kw,prefix,shape", ATTN_CASES)
def test_attention_incache_parity(name, kw, prefix, shape):
    w = I.scaled(I.WORKLOADS[name], **kw)
    if shape == "shared":
        trees = [I.workload_tree(w)] * w.B
        tree = Tree(trees[0])
    else:
        g = torch.Generator().manual_seed(4)
        trees = [I.random_tree_parents(n, 5, 6, g) for n in (40, 117, 9, 64)[:w.B]]
        tree = Tree(trees)
    T = tree.T
    inp = append_tree(w, trees, T, prefix)
    dev = {k: v.cuda() for k, v in inp.items()}
    max_prefix = max(prefix)
    out = api.tree_attention_incache(dev["q"], dev["k_cache"], dev["v_cache"], dev["prefix_len"], tree,
                                     max_prefix=max_prefix, want_lse=True)
    sep = api.tree_attention(dev["q"], dev["k_tree"], dev["v_tree"], dev["k_cache"], dev["v_cache"],
                             dev["prefix_len"], tree, max_prefix=max_prefix, want_lse=True)
    torch.cuda.synchronize()
    assert int(out["status"].item()) == 0
    # the same values read from another place: the same bits
    for b, par in enumerate(trees):
        Tb = len(par)
        assert torch.equal(out["out"][b, :Tb], sep["out"][b, :Tb]), b
        assert torch.equal(out["lse"][b, :Tb], sep["lse"][b, :Tb]), b
    o = out["out"].float().cpu()
    for b, par in enumerate(trees):
        Tb = len(par)
        ref_o, ref_l = oracle.tree_attention_incache(inp["q"][b:b + 1, :Tb], inp["k_cache"][b:b + 1],
                                                     inp["v_cache"][b:b + 1], inp["prefix_len"][b:b + 1], par)
        assert_float_parity(o[b, :Tb].reshape(-1, w.D), ref_o, w.torch_dtype, f"out[{b}]")
        assert np.abs(out["lse"][b, :Tb].cpu().reshape(-1).numpy() - ref_l).max() <= float_tol(w.torch_dtype)


def test_attention_incache_refuses_a_cache_without_room():
    w = I.scaled(I.WORKLOADS["llama8b"], B=1, prefix=100)
    tree = Tree(I.workload_tree(w))
    S_max = 128
    q = torch.zeros((1, tree.T, w.Hq, w.D), dtype=torch.bfloat16, device="cuda")
    kc = torch.zeros((1, w.Hkv, S_max, w.D), dtype=torch.bfloat16, device="cuda")
    pl = torch.zeros(1, dtype=torch.int32, device="cuda")
    with pytest.raises(B.MedusaError) as e:   # 100 + 117 > 128
        api.tree_attention_incache(q, kc, kc, pl, tree, max_prefix=100)
    assert e.value.code == B.MEDUSA_ERR_INVALID_ARG


@pytest.mark.parametrize("dtype,n_layers", [(torch.bfloat16, 32), (torch.float32, 3)])
def test_kv_compact_parity(dtype, n_layers):
    # every layer compacted in one launch, bit for bit; rows past each new
    # prefix keep what they held (NaN canaries included)
    B_, Hkv, S_max, D, T = 5, 4, 96, 64, 33
    g = torch.Generator().manual_seed(8)
    ks = [torch.randn((B_, Hkv, S_max, D), generator=g).to(dtype) for _ in range(n_layers)]
    vs = [torch.randn((B_, Hkv, S_max, D), generator=g).to(dtype) for _ in range(n_layers)]
    for x in ks + vs:
        x[:, :, 90:] = float("nan")
    pl = np.array([0, 17, 40, 63, 5], np.int32)
    max_path = 6
    path = np.full((B_, max_path), -1, np.int32)
    ln = np.array([1, 6, 3, 4, 2], np.int32)
    rng = np.random.default_rng(2)
    for b in range(B_):
        path[b, :ln[b]] = np.sort(np.concatenate([[0], rng.choice(np.arange(1, T), ln[b] - 1, replace=False)]))
    ref_k, ref_v, ref_npl, ref_st = oracle.kv_compact(ks, vs, path, ln, pl, T)
    kd = [x.cuda() for x in ks]
    vd = [x.cuda() for x in vs]
    res = api.kv_compact(kd, vd, torch.from_numpy(path).cuda(), torch.from_numpy(ln).cuda(),
                         torch.from_numpy(pl).cuda(), T)
    torch.cuda.synchronize()
    assert int(res["status"].item()) == 0 and ref_st == 0
    assert res["new_prefix_len"].cpu().numpy().tolist() == ref_npl.tolist()
    for l in range(n_layers):
        # bitwise, NaN payloads included
        assert bits_equal(kd[l], ref_k[l]), l
        assert bits_equal(vd[l], ref_v[l]), l


def test_kv_compact_refusals():
    B_, Hkv, S_max, D, T = 4, 2, 12, 64, 6
    g = torch.Generator().manual_seed(1)
    ks = [torch.randn((B_, Hkv, S_max, D), generator=g).bfloat16() for _ in range(2)]
    vs = [torch.randn((B_, Hkv, S_max, D), generator=g).bfloat16() for _ in range(2)]
    pl = np.array([2, 2, 2, 9], np.int32)
    path = np.array([[0, 3, 3], [0, 6, -1], [0, 1, 2], [0, 1, 3]], np.int32)
    ln = np.array([3, 2, 4, 3], np.int32)
    ref_k, ref_v, ref_npl, ref_st = oracle.kv_compact(ks, vs, path, ln, pl, T)
    kd = [x.cuda() for x in ks]
    vd = [x.cuda() for x in vs]
    res = api.kv_compact(kd, vd, torch.from_numpy(path).cuda(), torch.from_numpy(ln).cuda(),
                         torch.from_numpy(pl).cuda(), T)
    torch.cuda.synchronize()
    st = int(res["status"].item())
    assert st & B.STATUS_BAD_TOKEN and st & B.STATUS_CACHE_OVERFLOW
    assert res["new_prefix_len"].cpu().numpy().tolist() == ref_npl.tolist() == pl.tolist()
    for l in range(2):
        assert bits_equal(kd[l], ks[l]) and bits_equal(vd[l], vs[l])
    # new_prefix_len may not alias prefix_len (the layers' CTAs all read it)
    p_dev = torch.from_numpy(pl).cuda()
    with pytest.raises(B.MedusaError):
        api.kv_compact(kd, vd, torch.from_numpy(path).cuda(), torch.from_numpy(ln).cuda(), p_dev, T,
                       new_prefix_len=p_dev)


def test_step_with_the_tree_in_the_cache_matches_the_separate_layout():
    # heads -> attention (tree in the cache) -> greedy verify -> compaction of
    # 4 layers, against the same step with separate tree buffers and kv_commit
    w = I.scaled(I.WORKLOADS["llama8b"], B=2, d=256, V=1000, K=4, prefix=200, **ROOM)
    parents = I.workload_tree(w)
    T = len(parents)
    n_layers = 4
    hin = {k: v.cuda() for k, v in I.head_inputs(w).items()}
    inp = append_tree(w, [parents] * w.B, T, [150, 200])
    ain = {k: v.cuda() for k, v in inp.items()}
    logits = torch.randn((w.B, T, w.V), generator=torch.Generator().manual_seed(3)).to(w.torch_dtype).cuda()
    g = torch.Generator().manual_seed(5)
    shape = inp["k_cache"].shape
    kl = [ain["k_cache"]] + [torch.randn(shape, generator=g).to(w.torch_dtype).cuda() for _ in range(n_layers - 1)]
    vl = [ain["v_cache"]] + [torch.randn(shape, generator=g).to(w.torch_dtype).cuda() for _ in range(n_layers - 1)]
    k_before = [x.clone() for x in kl]
    v_before = [x.clone() for x in vl]
    mk = dict(B=w.B, d=w.d, V=w.V, K=w.K, Hq=w.Hq, Hkv=w.Hkv, D=w.D, S_max=w.S_max, parents=parents,
              dtype=w.torch_dtype, max_prefix=200, device="cuda")
    inc = api.MedusaStep(tree_in_cache=True, **mk)
    sep = api.MedusaStep(**mk)
    npl_i = torch.empty_like(ain["prefix_len"])
    npl_s = torch.empty_like(ain["prefix_len"])
    common = dict(h=hin["h"], W_res=hin["W_res"], W_head=hin["W_head"], root_token=hin["root_token"], q=ain["q"],
                  prefix_len=ain["prefix_len"], target=logits)
    kc_s, vc_s = ain["k_cache"].clone(), ain["v_cache"].clone()
    sep.run(k_tree=ain["k_tree"], v_tree=ain["v_tree"], k_cache=kc_s, v_cache=vc_s, new_prefix_len=npl_s, **common)
    inc.run(k_tree=None, v_tree=None, k_cache=ain["k_cache"], v_cache=ain["v_cache"], new_prefix_len=npl_i,
            k_layers=kl, v_layers=vl, **common)
    torch.cuda.synchronize()
    assert int(inc.status.item()) == 0 and int(sep.status.item()) == 0
    assert torch.equal(inc.attn_out, sep.attn_out)
    for a, b in ((inc.accept_path, sep.accept_path), (inc.accept_len, sep.accept_len), (inc.bonus, sep.bonus),
                 (npl_i, npl_s)):
        assert torch.equal(a, b)
    # layer 0: rows below the new prefix equal the separate layout's commit
    for b in range(w.B):
        n = int(npl_i[b])
        assert bits_equal(kl[0][b, :, :n], kc_s[b, :, :n]) and bits_equal(vl[0][b, :, :n], vc_s[b, :, :n])
    # every layer: the oracle's compaction of that layer
    ref_k, ref_v, ref_npl, _ = oracle.kv_compact(k_before, v_before, inc.accept_path.cpu(), inc.accept_len.cpu(),
                                                 ain["prefix_len"].cpu(), T)
    assert ref_npl.tolist() == npl_i.cpu().tolist()
    for l in range(n_layers):
        assert bits_equal(kl[l], ref_k[l]) and bits_equal(vl[l], ref_v[l])
