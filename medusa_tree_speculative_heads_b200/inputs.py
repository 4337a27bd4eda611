"""Seeded synthetic inputs for one Medusa decode step.

This module only *draws* inputs: shapes, value distributions and tree
topologies of the five workloads.  It holds none of the step's arithmetic
(no head, no attention, no verification, no commit), so the CUDA path and the
fp64 oracle can both be fed from it without sharing any of the method.

Workloads (all synthetic, no dataset or trained weights exist for them):

* ``tiny``   fp32, B=1, d=256, V=1024, K=2 heads, top-s (2,2) -> 7 nodes,
  4 q-heads = 4 kv-heads, head_dim 64, prefix 64, greedy, match prob 0.6.
* ``llama8b`` bf16, B=1, d=4096, V=128256, K=4, top-s (4,4,2,2) -> 117 nodes
  (64 leaf paths), 32/8 heads GQA, head_dim 128, prefix 2048, match prob 0.6.
* ``llama70b_b8`` bf16, B=8, d=8192, V=128256, K=4, 117 nodes, 64/8 heads,
  head_dim 128, per-sequence prefix uniform in [4096, 8192], match prob 0.7.
* ``long32k`` / ``long128k`` llama8b shapes at prefix 32768 / 131072.
* ``stoch_b64`` bf16, B=64, d=4096, V=32000, K=3, a seeded random 32-node tree
  (depth <= 4 counting the root as 1, <= 6 children), 32/8 heads, head_dim
  128, prefix 1024, stochastic verification.
* ``llama8b_incache`` llama8b with the tree's K/V appended to the cache after
  the prefix before attention (S_max = prefix + 128) and the commit as one
  in-place compaction of 32 layers' caches.
* ``stoch_logits_b64`` stoch_b64 with verification reading the target's bf16
  logits at temperature 0.7 instead of fp32 probabilities.
* ``ragged_paged_b8`` bf16, B=8, the llama8b shapes, a random tree per
  sequence (32 to 117 nodes, depth <= 5, <= 8 children), prefix uniform in
  [1024, 8192], the KV cache in 16-row pages read through a block table.

Value distributions: hidden state and all attention tensors N(0,1); head
weights N(0, 1/d).  Greedy target logits are N(0,1) and, for every node that
has children, with the workload's match probability one uniformly chosen
child's token gets +10 on the parent's row.  Stochastic targets: logit of a
token = -1.1 ln(rank) + N(0, variance 0.5) over a per-row random ranking,
p = softmax(logit / 0.7) in fp32 (the logits themselves for the logits form);
the draft is q = 0.7 p + 0.3 Zipf(1.1) on an
independent ranking; every child token is drawn from q at its parent.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, List, Optional, Sequence

import torch

F32 = "f32"
BF16 = "bf16"


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    seed: int
    dtype: str
    B: int
    d: int
    V: int
    K: int
    Hq: int
    Hkv: int
    D: int
    prefix: int                      # nominal prefix length
    prefix_range: Optional[tuple] = None   # (lo, hi) inclusive, per sequence
    topk: Optional[tuple] = None     # branching factors of a full product tree
    random_tree: Optional[tuple] = None    # (T, max_depth, max_children)
    match_prob: float = 0.6          # greedy boost probability
    stochastic: bool = False
    ragged_trees: Optional[tuple] = None   # (T_min, T_max, max_depth, max_children): a random tree per sequence
    page_size: int = 0               # > 0: the KV cache is a page pool read through a block table
    temperature: float = 0.0         # > 0: stochastic verification reads bf16 target logits at this temperature
    cache_room: int = 64             # cache slots past the longest prefix (S_max = max_prefix + cache_room)
    tree_in_cache: bool = False      # the tree's K/V are appended to the cache after each prefix before attention
    layers: int = 1                  # caches compacted per step when the tree is in the cache

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == F32 else torch.bfloat16

    @property
    def max_prefix(self) -> int:
        return self.prefix_range[1] if self.prefix_range else self.prefix

    @property
    def S_max(self) -> int:
        # room past the longest prefix: one commit of up to K+1 tokens, or the
        # whole tree when its K/V are appended to the cache
        return self.max_prefix + self.cache_room


WORKLOADS: Dict[str, Workload] = {
    "tiny": Workload("tiny", 0, F32, 1, 256, 1024, 2, 4, 4, 64, 64, topk=(2, 2), match_prob=0.6),
    "llama8b": Workload("llama8b", 1, BF16, 1, 4096, 128256, 4, 32, 8, 128, 2048,
                        topk=(4, 4, 2, 2), match_prob=0.6),
    "llama70b_b8": Workload("llama70b_b8", 2, BF16, 8, 8192, 128256, 4, 64, 8, 128, 8192,
                            prefix_range=(4096, 8192), topk=(4, 4, 2, 2), match_prob=0.7),
    "long32k": Workload("long32k", 3, BF16, 1, 4096, 128256, 4, 32, 8, 128, 32768,
                        topk=(4, 4, 2, 2), match_prob=0.6),
    "long128k": Workload("long128k", 3, BF16, 1, 4096, 128256, 4, 32, 8, 128, 131072,
                         topk=(4, 4, 2, 2), match_prob=0.6),
    "stoch_b64": Workload("stoch_b64", 4, BF16, 64, 4096, 32000, 3, 32, 8, 128, 1024,
                          random_tree=(32, 4, 6), stochastic=True),
    "llama8b_incache": Workload("llama8b_incache", 1, BF16, 1, 4096, 128256, 4, 32, 8, 128, 2048,
                                topk=(4, 4, 2, 2), match_prob=0.6, cache_room=128, tree_in_cache=True, layers=32),
    "stoch_logits_b64": Workload("stoch_logits_b64", 4, BF16, 64, 4096, 32000, 3, 32, 8, 128, 1024,
                                 random_tree=(32, 4, 6), stochastic=True, temperature=0.7),
    "ragged_paged_b8": Workload("ragged_paged_b8", 5, BF16, 8, 4096, 128256, 4, 32, 8, 128, 8192,
                                prefix_range=(1024, 8192), ragged_trees=(32, 117, 5, 8), page_size=16),
}


def scaled(w: Workload, **kw) -> Workload:
    """The same workload with some sizes replaced (for small parity cases)."""
    return dataclasses.replace(w, **kw)


# ----------------------------------------------------------------------------
# tree topologies (parent arrays, root = node 0 with parent -1)
# ----------------------------------------------------------------------------

def product_tree_parents(branching: Sequence[int]) -> List[int]:
    """Parent array, in breadth-first order, of the full tree whose nodes at
    depth k (root depth 1) each have ``branching[k-1]`` children."""
    parents = [-1]
    level = [0]
    for s in branching:
        nxt = []
        for u in level:
            for _ in range(s):
                parents.append(u)
                nxt.append(len(parents) - 1)
        level = nxt
    return parents


def random_tree_parents(T: int, max_depth: int, max_children: int, gen: torch.Generator) -> List[int]:
    """Seeded random tree of T nodes: grow by attaching each new node to a
    uniformly chosen eligible node (depth < max_depth, fewer than
    max_children children), then renumber breadth-first (siblings keep their
    insertion order)."""
    parent = [-1]
    depth = [1]
    nchild = [0]
    for _ in range(1, T):
        elig = [u for u in range(len(parent)) if depth[u] < max_depth and nchild[u] < max_children]
        u = elig[int(torch.randint(len(elig), (1,), generator=gen))]
        parent.append(u)
        depth.append(depth[u] + 1)
        nchild.append(0)
        nchild[u] += 1
    children = [[] for _ in range(T)]
    for i in range(1, T):
        children[parent[i]].append(i)
    order = [0]
    for u in order:
        order.extend(children[u])
    new_id = {old: new for new, old in enumerate(order)}
    return [-1] + [new_id[parent[old]] for old in order[1:]]


def tree_children(parents: Sequence[int]) -> List[List[int]]:
    ch = [[] for _ in parents]
    for i, p in enumerate(parents):
        if p >= 0:
            ch[p].append(i)
    return ch


def workload_tree(w: Workload):
    """The workload's tree (a parent list), or with ``ragged_trees`` one
    parent list per sequence (sizes uniform in [T_min, T_max])."""
    if w.ragged_trees is not None:
        g = torch.Generator().manual_seed(1000 + w.seed)
        lo, hi, md, mc = w.ragged_trees
        return [random_tree_parents(int(torch.randint(lo, hi + 1, (1,), generator=g)), md, mc, gen=g)
                for _ in range(w.B)]
    if w.topk is not None:
        return product_tree_parents(w.topk)
    g = torch.Generator().manual_seed(1000 + w.seed)
    return random_tree_parents(*w.random_tree, gen=g)


def sequence_trees(w: Workload) -> List[List[int]]:
    """Parent list of every sequence's tree (the shared tree repeated)."""
    t = workload_tree(w)
    return t if w.ragged_trees is not None else [t] * w.B


# ----------------------------------------------------------------------------
# tensors
# ----------------------------------------------------------------------------

def _randn(shape, gen, std=1.0, dtype=torch.float32, device="cpu", chunk_rows=8192):
    """N(0, std^2) drawn in fixed-size row chunks (bounded fp32 temporaries)."""
    shape = tuple(shape)
    out = torch.empty(shape, dtype=dtype, device=device)
    flat = out.view(-1, shape[-1])
    for r0 in range(0, flat.shape[0], chunk_rows):
        r1 = min(r0 + chunk_rows, flat.shape[0])
        t = torch.randn((r1 - r0, shape[-1]), generator=gen, device=device)
        if std != 1.0:
            t.mul_(std)
        flat[r0:r1].copy_(t)
    return out


def _gen(seed: int, device: str) -> torch.Generator:
    return torch.Generator(device=device).manual_seed(seed)


def head_inputs(w: Workload, device: str = "cpu") -> Dict[str, torch.Tensor]:
    """h [B,d], W_res [K,d,d] (out x in), W_head [K,V,d], root_token [B]."""
    dt = w.torch_dtype
    g = _gen(w.seed * 7919 + 1, device)
    h = _randn((w.B, w.d), g, dtype=dt, device=device)
    W_res = _randn((w.K, w.d, w.d), g, std=1.0 / math.sqrt(w.d), dtype=dt, device=device)
    W_head = _randn((w.K, w.V, w.d), g, std=1.0 / math.sqrt(w.d), dtype=dt, device=device)
    root = torch.randint(0, w.V, (w.B,), generator=g, device=device, dtype=torch.int32)
    return {"h": h, "W_res": W_res, "W_head": W_head, "root_token": root}


def prefix_lengths(w: Workload) -> torch.Tensor:
    if w.prefix_range is None:
        return torch.full((w.B,), w.prefix, dtype=torch.int32)
    g = _gen(w.seed * 7919 + 2, "cpu")
    lo, hi = w.prefix_range
    return torch.randint(lo, hi + 1, (w.B,), generator=g, dtype=torch.int32)


def attention_inputs(w: Workload, T: int, device: str = "cpu", canary: Optional[float] = None,
                     prefix_len: Optional[torch.Tensor] = None) -> Dict[str, torch.Tensor]:
    """q [B,T,Hq,D]; k_tree, v_tree [B,T,Hkv,D]; k_cache, v_cache
    [B,Hkv,S_max,D]; prefix_len [B].  With ``canary`` the cache slots at and
    beyond each sequence's prefix are filled with that value instead."""
    dt = w.torch_dtype
    g = _gen(w.seed * 7919 + 3, device)
    pl = prefix_lengths(w) if prefix_len is None else prefix_len
    k_cache = _randn((w.B, w.Hkv, w.S_max, w.D), g, dtype=dt, device=device)
    v_cache = _randn((w.B, w.Hkv, w.S_max, w.D), g, dtype=dt, device=device)
    q = _randn((w.B, T, w.Hq, w.D), g, dtype=dt, device=device)
    k_tree = _randn((w.B, T, w.Hkv, w.D), g, dtype=dt, device=device)
    v_tree = _randn((w.B, T, w.Hkv, w.D), g, dtype=dt, device=device)
    if canary is not None:
        for b in range(w.B):
            k_cache[b, :, int(pl[b]):, :] = canary
            v_cache[b, :, int(pl[b]):, :] = canary
    return {"q": q, "k_tree": k_tree, "v_tree": v_tree, "k_cache": k_cache, "v_cache": v_cache,
            "prefix_len": pl.to(device)}


def paged_cache(w: Workload, page_size: int, prefix_len: torch.Tensor, room: int = 64, extra_pages: int = 3,
                device: str = "cpu", canary: Optional[float] = None, capacity: int = 0) -> Dict[str, torch.Tensor]:
    """A page pool k_pages, v_pages [num_pages, Hkv, page_size, D] and a block
    table [B, max_pages] int32: sequence b owns ceil((prefix_len[b] + room) /
    page_size) pages taken from a seeded random permutation of the pool (its
    other table entries are -1), and `extra_pages` pages belong to nobody.
    With ``canary`` every slot no call may read (positions at or past each
    sequence's prefix, unowned pages) holds that value.  The table has room
    for at least ``capacity`` positions per sequence (entries past the owned
    pages are -1)."""
    dt = w.torch_dtype
    g = _gen(w.seed * 7919 + 9, "cpu")
    pl = [int(x) for x in prefix_len]
    need = [(n + room + page_size - 1) // page_size for n in pl]
    max_pages = max(max(need), (capacity + page_size - 1) // page_size)
    num_pages = sum(need) + extra_pages
    perm = torch.randperm(num_pages, generator=g)
    table = torch.full((w.B, max_pages), -1, dtype=torch.int32)
    k = 0
    for b in range(w.B):
        table[b, :need[b]] = perm[k:k + need[b]].to(torch.int32)
        k += need[b]
    k_pages = _randn((num_pages, w.Hkv, page_size, w.D), g, dtype=dt)
    v_pages = _randn((num_pages, w.Hkv, page_size, w.D), g, dtype=dt)
    if canary is not None:
        owned = torch.zeros(num_pages, dtype=torch.bool)
        for b in range(w.B):
            for blk in range(need[b]):
                page = int(table[b, blk])
                owned[page] = True
                lo = max(0, pl[b] - blk * page_size)
                if lo < page_size:
                    k_pages[page, :, lo:] = canary
                    v_pages[page, :, lo:] = canary
        k_pages[~owned] = canary
        v_pages[~owned] = canary
    return {"k_pages": k_pages.to(device), "v_pages": v_pages.to(device), "block_table": table.to(device)}


def random_node_tokens(w: Workload, parents: Sequence[int], seed_offset: int = 0) -> torch.Tensor:
    """[B,T] int32 tokens: a random root token and, under every node, distinct
    random tokens for its children (as a top-s list would give)."""
    g = _gen(w.seed * 7919 + 4 + seed_offset, "cpu")
    T = len(parents)
    ch = tree_children(parents)
    tok = torch.empty((w.B, T), dtype=torch.int32)
    for b in range(w.B):
        tok[b, 0] = int(torch.randint(0, w.V, (1,), generator=g))
        for u in range(T):
            if ch[u]:
                pick = torch.randperm(w.V, generator=g)[: len(ch[u])]
                for c, t in zip(ch[u], pick.tolist()):
                    tok[b, c] = t
    return tok


def boosted_target_logits(w: Workload, parents: Sequence[int], node_tokens: torch.Tensor,
                          device: str = "cpu", boost: float = 10.0, seed_offset: int = 0) -> torch.Tensor:
    """[B,T,V] target logits ~ N(0,1) in the workload dtype; for each node
    with children, with probability ``match_prob`` one uniformly chosen
    child's token gets ``boost`` added on the parent's row.  ``parents`` may
    be one parent list per sequence (T = the largest tree)."""
    g = _gen(w.seed * 7919 + 5 + seed_offset, device)
    per_seq = len(parents) > 0 and hasattr(parents[0], "__len__")
    trees = list(parents) if per_seq else [parents] * w.B
    T = max(len(t) for t in trees)
    logits = _randn((w.B, T, w.V), g, dtype=torch.float32, device=device)
    gc = _gen(w.seed * 7919 + 6 + seed_offset, "cpu")
    nt = node_tokens.cpu()
    for b in range(w.B):
        ch = tree_children(trees[b])
        for u in range(len(trees[b])):
            if not ch[u]:
                continue
            if float(torch.rand((1,), generator=gc)) < w.match_prob:
                c = ch[u][int(torch.randint(len(ch[u]), (1,), generator=gc))]
                logits[b, u, int(nt[b, c])] += boost
    return logits.to(w.torch_dtype)


STOCH_TEMPERATURE = 0.7   # the target's sampling temperature in stochastic_inputs


def stochastic_inputs(w: Workload, parents: Sequence[int], device: str = "cpu") -> Dict[str, torch.Tensor]:
    """p, q [B,T,V] fp32 and node_tokens [B,T] (children drawn from q at
    their parent; the root token uniform); also the target's logits [B,T,V]
    fp32 with p = softmax(logits / STOCH_TEMPERATURE)."""
    g = _gen(w.seed * 7919 + 7, "cpu")
    T = len(parents)
    V = w.V
    ranks = torch.arange(1, V + 1, dtype=torch.float64)
    p = torch.empty((w.B, T, V), dtype=torch.float32)
    q = torch.empty((w.B, T, V), dtype=torch.float32)
    logits = torch.empty((w.B, T, V), dtype=torch.float32)
    zipf = ranks.pow(-1.1)
    zipf = (zipf / zipf.sum()).to(torch.float32)
    for b in range(w.B):
        for u in range(T):
            perm = torch.randperm(V, generator=g)
            logit = torch.empty(V, dtype=torch.float32)
            logit[perm] = (-1.1 * torch.log(ranks)).to(torch.float32)
            logit += torch.randn(V, generator=g) * math.sqrt(0.5)
            logits[b, u] = logit
            p[b, u] = torch.softmax(logit / STOCH_TEMPERATURE, dim=0)
            perm2 = torch.randperm(V, generator=g)
            z = torch.empty(V, dtype=torch.float32)
            z[perm2] = zipf
            q[b, u] = 0.7 * p[b, u] + 0.3 * z
    ch = tree_children(parents)
    tok = torch.empty((w.B, T), dtype=torch.int32)
    for b in range(w.B):
        tok[b, 0] = int(torch.randint(0, V, (1,), generator=g))
        for u in range(T):
            if ch[u]:
                draws = torch.multinomial(q[b, u].double(), len(ch[u]), replacement=True, generator=g)
                for c, t in zip(ch[u], draws.tolist()):
                    tok[b, c] = t
    return {"p": p.to(device), "q": q.to(device), "node_tokens": tok.to(device), "logits": logits.to(device)}
