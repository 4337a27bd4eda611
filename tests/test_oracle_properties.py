"""Property checks of the oracle's tree and cache functions over random
inputs (hypothesis): every tree's ancestor mask, depths and sibling ranks
follow from the parent array alone, and the in-place compaction of a cache
equals the commit of the rows it reads, for any strictly increasing path."""
import numpy as np
import torch
from hypothesis import given, settings
from hypothesis import strategies as st

import oracle


@st.composite
def parent_arrays(draw):
    T = draw(st.integers(1, 40))
    return [-1] + [draw(st.integers(0, i - 1)) for i in range(1, T)]


@settings(max_examples=200, deadline=None)
@given(parent_arrays())
def test_mask_depth_and_rank_follow_from_the_parents(par):
    oracle.build()
    T = len(par)
    mask = oracle.tree_mask(par)
    depth, rank = oracle.tree_shape(par)
    for i in range(T):
        want = np.zeros(T, np.uint8)
        want[i] = 1
        if par[i] >= 0:
            want |= mask[par[i]]
        assert np.array_equal(mask[i], want)
        assert depth[i] == mask[i].sum()
        siblings = [c for c in range(T) if par[c] == par[i] and c < i] if i > 0 else []
        assert rank[i] == len(siblings)


@st.composite
def compaction_cases(draw):
    T = draw(st.integers(1, 12))
    B = draw(st.integers(1, 3))
    S_max = draw(st.integers(T + 1, T + 20))
    cases = []
    for _ in range(B):
        S = draw(st.integers(0, S_max - T))
        L = draw(st.integers(1, T))
        rest = sorted(draw(st.lists(st.integers(1, T - 1), min_size=L - 1, max_size=L - 1, unique=True))) if T > 1 \
            else []
        cases.append((S, [0] + rest[:L - 1]))
    return T, S_max, cases


@settings(max_examples=100, deadline=None)
@given(compaction_cases(), st.integers(0, 2**31 - 1))
def test_compaction_is_the_commit_of_the_rows_it_reads(case, seed):
    oracle.build()
    T, S_max, cases = case
    B, Hkv, D = len(cases), 2, 4
    g = torch.Generator().manual_seed(seed)
    kc = torch.randn((B, Hkv, S_max, D), generator=g)
    vc = torch.randn((B, Hkv, S_max, D), generator=g)
    pl = np.array([c[0] for c in cases], np.int32)
    max_path = T
    path = np.full((B, max_path), -1, np.int32)
    ln = np.zeros(B, np.int32)
    for b, (_, p) in enumerate(cases):
        path[b, :len(p)] = p
        ln[b] = len(p)
    k2, v2, npl, st_ = oracle.kv_compact([kc], [vc], path, ln, pl, T)
    kt = oracle.tree_rows_from_cache(kc, pl, T)
    vt = oracle.tree_rows_from_cache(vc, pl, T)
    kr, vr, npl_r, st_r = oracle.kv_commit(kc, vc, kt, vt, path, ln, pl)
    assert st_ == st_r == 0 and npl.tolist() == npl_r.tolist() == (pl + ln).tolist()
    assert torch.equal(k2[0], kr) and torch.equal(v2[0], vr)
