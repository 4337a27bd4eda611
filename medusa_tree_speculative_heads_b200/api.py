"""Tensor-level API over the C ABI.

The functions here allocate outputs and workspaces with torch and call the
binding; every step of the computation runs in libmedusa's CUDA kernels.
``MedusaStep`` preallocates everything for a fixed shape, so a decode step
is four library calls with no allocation (and can be captured in a CUDA
graph).
"""
from __future__ import annotations

from typing import Dict, Optional, Sequence

import torch

from . import binding as _b
from .binding import Tree


def _ws(nbytes: int, device) -> torch.Tensor:
    return torch.empty(max(int(nbytes), 16), dtype=torch.uint8, device=device)


def _status(device) -> torch.Tensor:
    return torch.zeros(1, dtype=torch.int32, device=device)


def heads(h: torch.Tensor, W_res: torch.Tensor, W_head: torch.Tensor, tree: Optional[Tree] = None,
          root_token: Optional[torch.Tensor] = None, want_logits: bool = False, want_probs: bool = False,
          want_hres: bool = False) -> Dict[str, torch.Tensor]:
    """Medusa heads: top-8 ids/probabilities per head and, with a tree, the
    tree's node tokens.  h [B,d], W_res [K,d,d], W_head [K,V,d]."""
    B, d = h.shape
    K, V, _ = W_head.shape
    dev = h.device
    dt = _b.dtype_code(h.dtype)
    out = {
        "topk_idx": torch.empty((B, K, _b.TOPK), dtype=torch.int32, device=dev),
        "topk_prob": torch.empty((B, K, _b.TOPK), dtype=torch.float32, device=dev),
        "status": _status(dev),
    }
    if tree is not None:
        out["node_tokens"] = torch.empty((B, tree.T), dtype=torch.int32, device=dev)
        out["node_q"] = torch.empty((B, tree.T), dtype=torch.float32, device=dev)
    if want_logits:
        out["logits"] = torch.empty((B, K, V), dtype=torch.float32, device=dev)
    if want_probs:
        out["probs"] = torch.empty((B, K, V), dtype=torch.float32, device=dev)
    if want_hres:
        out["h_res"] = torch.empty((B, K, d), dtype=h.dtype, device=dev)
    nb = _b.medusa_heads_workspace_size(B, d, V, K, dt)
    ws = _ws(nb, dev)
    _b.medusa_heads(h, W_res, W_head, B, d, V, K, dt, tree, root_token, out["topk_idx"], out["topk_prob"],
                    out.get("node_tokens"), out.get("node_q"), out.get("h_res"), out.get("logits"),
                    out.get("probs"), ws, nb, out["status"])
    return out


def tree_attention(q, k_tree, v_tree, k_cache, v_cache, prefix_len, tree: Tree, scale: float = 0.0,
                   max_prefix: int = 0, want_lse: bool = False) -> Dict[str, torch.Tensor]:
    """Tree attention; q [B,T,Hq,D], k/v_tree [B,T,Hkv,D], caches
    [B,Hkv,S_max,D], prefix_len [B] int32."""
    B, T, Hq, D = q.shape
    Hkv = k_tree.shape[2]
    S_max = k_cache.shape[2]
    dev = q.device
    dt = _b.dtype_code(q.dtype)
    out = {"out": torch.empty_like(q), "status": _status(dev)}
    if want_lse:
        out["lse"] = torch.empty((B, T, Hq), dtype=torch.float32, device=dev)
    nb = _b.tree_attention_workspace_size(B, Hq, Hkv, D, S_max, max_prefix, tree, dt)
    ws = _ws(nb, dev)
    _b.tree_attention(q, k_tree, v_tree, k_cache, v_cache, prefix_len, B, Hq, Hkv, D, S_max, max_prefix, scale, dt,
                      tree, out["out"], out.get("lse"), ws, nb, out["status"])
    return out


def tree_verify(mode: int, target: torch.Tensor, node_tokens: torch.Tensor, tree: Tree,
                q: Optional[torch.Tensor] = None, q_row: Optional[torch.Tensor] = None, seed: int = 0,
                step: int = 0, max_path: Optional[int] = None) -> Dict[str, torch.Tensor]:
    """Greedy (target = logits [B,T,V]) or stochastic (target = p [B,T,V]
    fp32, q [B,q_rows,V] fp32, optional q_row [T]) verification."""
    B, T, V = target.shape
    dev = target.device
    max_path = max_path or tree.max_depth
    out = {
        "accept_path": torch.empty((B, max_path), dtype=torch.int32, device=dev),
        "accept_len": torch.empty((B,), dtype=torch.int32, device=dev),
        "bonus": torch.empty((B,), dtype=torch.int32, device=dev),
        "status": _status(dev),
    }
    nb = _b.tree_verify_workspace_size(mode, B, V, tree)
    ws = _ws(nb, dev)
    q_rows = q.shape[1] if q is not None else 0
    _b.tree_verify(mode, target, _b.dtype_code(target.dtype), q, q_rows, q_row, node_tokens, B, V, tree, seed, step,
                   out["accept_path"], max_path, out["accept_len"], out["bonus"], ws, nb, out["status"])
    return out


def tree_verify_logits(logits: torch.Tensor, temperature: float, q: torch.Tensor, node_tokens: torch.Tensor,
                       tree: Tree, q_row: Optional[torch.Tensor] = None, seed: int = 0, step: int = 0,
                       max_path: Optional[int] = None) -> Dict[str, torch.Tensor]:
    """Stochastic verification reading the target's logits [B,T,V] (f32 or
    bf16) at a temperature; q [B,q_rows,V] fp32, optional q_row."""
    B, T, V = logits.shape
    dev = logits.device
    max_path = max_path or tree.max_depth
    out = {
        "accept_path": torch.empty((B, max_path), dtype=torch.int32, device=dev),
        "accept_len": torch.empty((B,), dtype=torch.int32, device=dev),
        "bonus": torch.empty((B,), dtype=torch.int32, device=dev),
        "status": _status(dev),
    }
    nb = _b.tree_verify_workspace_size(_b.STOCHASTIC, B, V, tree)
    ws = _ws(nb, dev)
    _b.tree_verify_logits(logits, _b.dtype_code(logits.dtype), temperature, q, q.shape[1], q_row, node_tokens, B, V,
                          tree, seed, step, out["accept_path"], max_path, out["accept_len"], out["bonus"], ws, nb,
                          out["status"])
    return out


def tree_attention_incache(q, k_cache, v_cache, prefix_len, tree: Tree, scale: float = 0.0, max_prefix: int = 0,
                           want_lse: bool = False) -> Dict[str, torch.Tensor]:
    """Tree attention with the tree's K/V in the cache rows right after each
    prefix: k_cache/v_cache [B,Hkv,S_max,D]."""
    B, T, Hq, D = q.shape
    _, Hkv, S_max, _ = k_cache.shape
    dev = q.device
    dt = _b.dtype_code(q.dtype)
    out = {"out": torch.empty_like(q), "status": _status(dev)}
    if want_lse:
        out["lse"] = torch.empty((B, T, Hq), dtype=torch.float32, device=dev)
    nb = _b.tree_attention_incache_workspace_size(B, Hq, Hkv, D, S_max, max_prefix, tree, dt)
    ws = _ws(nb, dev)
    _b.tree_attention_incache(q, k_cache, v_cache, prefix_len, B, Hq, Hkv, D, S_max, max_prefix, scale, dt, tree,
                              out["out"], out.get("lse"), ws, nb, out["status"])
    return out


def kv_compact(k_caches, v_caches, accept_path, accept_len, prefix_len, T: int,
               new_prefix_len: Optional[torch.Tensor] = None) -> Dict[str, torch.Tensor]:
    """Compact the accepted path's rows (already in the cache after each
    prefix) in place, in every layer of the lists k_caches / v_caches
    ([B,Hkv,S_max,D] each) in one launch; returns new_prefix_len."""
    B, Hkv, S_max, D = k_caches[0].shape
    dev = k_caches[0].device
    if new_prefix_len is None:
        new_prefix_len = torch.empty_like(prefix_len)
    kp, vp = _b.layer_pointers(k_caches, dev), _b.layer_pointers(v_caches, dev)
    st = _status(dev)
    _b.kv_compact(kp, vp, len(k_caches), accept_path, accept_path.shape[1], accept_len, prefix_len, new_prefix_len, B,
                  T, Hkv, D, S_max, _b.dtype_code(k_caches[0].dtype), st)
    return {"new_prefix_len": new_prefix_len, "status": st}


def kv_commit(k_cache, v_cache, k_tree, v_tree, accept_path, accept_len, prefix_len,
              new_prefix_len: Optional[torch.Tensor] = None) -> Dict[str, torch.Tensor]:
    """Append the accepted path's K/V in place; returns new_prefix_len (a new
    tensor unless one is given, which may be prefix_len itself)."""
    B, Hkv, S_max, D = k_cache.shape
    T = k_tree.shape[1]
    dev = k_cache.device
    if new_prefix_len is None:
        new_prefix_len = torch.empty_like(prefix_len)
    st = _status(dev)
    _b.kv_commit(k_cache, v_cache, k_tree, v_tree, accept_path, accept_path.shape[1], accept_len, prefix_len,
                 new_prefix_len, B, T, Hkv, D, S_max, _b.dtype_code(k_cache.dtype), st)
    return {"new_prefix_len": new_prefix_len, "status": st}


def tree_attention_paged(q, k_tree, v_tree, k_pages, v_pages, block_table, prefix_len, tree: Tree,
                         scale: float = 0.0, max_prefix: int = 0, want_lse: bool = False) -> Dict[str, torch.Tensor]:
    """Tree attention over a paged cache: page pools k/v_pages
    [num_pages,Hkv,page_size,D], block_table [B,max_pages] int32."""
    B, T, Hq, D = q.shape
    Hkv = k_tree.shape[2]
    num_pages, _, page_size, _ = k_pages.shape
    max_pages = block_table.shape[1]
    dev = q.device
    dt = _b.dtype_code(q.dtype)
    out = {"out": torch.empty_like(q), "status": _status(dev)}
    if want_lse:
        out["lse"] = torch.empty((B, T, Hq), dtype=torch.float32, device=dev)
    nb = _b.tree_attention_paged_workspace_size(B, Hq, Hkv, D, max_prefix, max_pages, page_size, tree, dt)
    ws = _ws(nb, dev)
    _b.tree_attention_paged(q, k_tree, v_tree, k_pages, v_pages, block_table, max_pages, page_size, num_pages,
                            prefix_len, B, Hq, Hkv, D, max_prefix, scale, dt, tree, out["out"], out.get("lse"), ws,
                            nb, out["status"])
    return out


def kv_commit_paged(k_pages, v_pages, k_tree, v_tree, block_table, accept_path, accept_len, prefix_len,
                    new_prefix_len: Optional[torch.Tensor] = None) -> Dict[str, torch.Tensor]:
    """Append the accepted path's K/V into the page pools through the block table."""
    num_pages, Hkv, page_size, D = k_pages.shape
    B, T = k_tree.shape[0], k_tree.shape[1]
    dev = k_pages.device
    if new_prefix_len is None:
        new_prefix_len = torch.empty_like(prefix_len)
    st = _status(dev)
    _b.kv_commit_paged(k_pages, v_pages, k_tree, v_tree, block_table, block_table.shape[1], page_size, num_pages,
                       accept_path, accept_path.shape[1], accept_len, prefix_len, new_prefix_len, B, T, Hkv, D,
                       _b.dtype_code(k_pages.dtype), st)
    return {"new_prefix_len": new_prefix_len, "status": st}


class MedusaStep:
    """All buffers of one decode step of a fixed shape, allocated once.

    ``run`` issues the four library calls on the current stream:
    medusa_heads -> tree_attention -> tree_verify -> kv_commit, with tree
    attention on a second stream (joined back before verification) unless
    ``overlap`` is False.  The new
    prefix lengths go to ``new_prefix_len`` (pass the same tensor as
    ``prefix_len`` to advance in place).  ``parents`` is one parent list, or
    one per sequence.  With ``page_size`` > 0 the cache is a page pool
    [num_pages, Hkv, page_size, D] read and written through a block table
    [B, max_pages] (pass it as ``block_table``), and the paged calls run.
    With ``temperature`` > 0 (stochastic mode) the target passed to
    ``verify``/``run`` is the target's logits, read by tree_verify_logits.
    With ``tree_in_cache`` the tree's K/V are expected in the (contiguous)
    cache right after each prefix: attention runs tree_attention_incache and
    the commit is kv_compact over ``k_layers``/``v_layers`` (every layer's
    cache; the attended layer's cache among them) in one launch."""

    def __init__(self, *, B: int, d: int, V: int, K: int, Hq: int, Hkv: int, D: int, S_max: int,
                 parents, dtype: torch.dtype, mode: int = _b.GREEDY, max_prefix: int = 0,
                 q_rows: int = 0, device=None, page_size: int = 0, max_pages: int = 0, num_pages: int = 0,
                 temperature: float = 0.0, tree_in_cache: bool = False, overlap: bool = True,
                 attention_sms: int = 0):
        dev = torch.device(device) if device is not None else torch.device("cuda", torch.cuda.current_device())
        self.B, self.d, self.V, self.K = B, d, V, K
        self.Hq, self.Hkv, self.D, self.S_max, self.max_prefix = Hq, Hkv, D, S_max, max_prefix
        self.dt = _b.dtype_code(dtype)
        self.mode = mode
        self.temperature = temperature
        if temperature > 0 and mode != _b.STOCHASTIC:
            raise ValueError("a temperature applies to stochastic verification only")
        self.tree = Tree(parents)
        T = self.T = self.tree.T
        self.max_path = self.tree.max_depth
        self.q_rows = q_rows
        i32, f32 = torch.int32, torch.float32
        self.topk_idx = torch.empty((B, K, _b.TOPK), dtype=i32, device=dev)
        self.topk_prob = torch.empty((B, K, _b.TOPK), dtype=f32, device=dev)
        self.node_tokens = torch.empty((B, T), dtype=i32, device=dev)
        self.node_q = torch.empty((B, T), dtype=f32, device=dev)
        self.attn_out = torch.empty((B, T, Hq, D), dtype=dtype, device=dev)
        self.accept_path = torch.empty((B, self.max_path), dtype=i32, device=dev)
        self.accept_len = torch.empty((B,), dtype=i32, device=dev)
        self.bonus = torch.empty((B,), dtype=i32, device=dev)
        self.status = torch.zeros(1, dtype=i32, device=dev)
        self.ws_heads_n = _b.medusa_heads_workspace_size(B, d, V, K, self.dt)
        self.page_size, self.max_pages, self.num_pages = page_size, max_pages, num_pages
        self.tree_in_cache = tree_in_cache
        self._layer_ptrs = {}
        # run() with attention_sms > 0: the heads kernel leaves that many SMs
        # free and tree attention runs on them without key splits, during the
        # heads' weight stream instead of after it
        self.attention_sms = attention_sms if overlap else 0
        self._sms = torch.cuda.get_device_properties(dev).multi_processor_count
        # run(): tree attention (which reads none of the heads' outputs) on a
        # second stream, so its CTAs take the SMs the heads kernel frees while
        # that kernel's last CTA still merges
        # (the heads on a higher-priority stream: when both calls become ready
        # at once, the heads kernel, which needs every SM, is dispatched first)
        self._side = torch.cuda.Stream(device=dev) if overlap else None
        self._hp = torch.cuda.Stream(device=dev, priority=-1) if overlap else None
        # greedy verification's scan of the target rows reads neither: a third stream
        self._side2 = torch.cuda.Stream(device=dev) if overlap else None
        if tree_in_cache and page_size > 0:
            raise ValueError("the tree-in-cache layout is for contiguous caches")
        if tree_in_cache:
            self.ws_attn_n = _b.tree_attention_incache_workspace_size(B, Hq, Hkv, D, S_max, max_prefix, self.tree,
                                                                      self.dt)
        elif page_size > 0:
            self.ws_attn_n = _b.tree_attention_paged_workspace_size(B, Hq, Hkv, D, max_prefix, max_pages, page_size,
                                                                    self.tree, self.dt)
        else:
            self.ws_attn_n = _b.tree_attention_workspace_size(B, Hq, Hkv, D, S_max, max_prefix, self.tree, self.dt)
        self.ws_verify_n = _b.tree_verify_workspace_size(mode, B, V, self.tree)
        self.ws_heads = _ws(self.ws_heads_n, dev)
        self.ws_attn = _ws(self.ws_attn_n, dev)
        self.ws_verify = _ws(self.ws_verify_n, dev)

    def heads(self, h, W_res, W_head, root_token, probs_out=None):
        _b.medusa_heads(h, W_res, W_head, self.B, self.d, self.V, self.K, self.dt, self.tree, root_token,
                        self.topk_idx, self.topk_prob, self.node_tokens, self.node_q, None, None, probs_out,
                        self.ws_heads, self.ws_heads_n, self.status)

    def attention(self, q, k_tree, v_tree, k_cache, v_cache, prefix_len, block_table=None):
        if self.tree_in_cache:
            _b.tree_attention_incache(q, k_cache, v_cache, prefix_len, self.B, self.Hq, self.Hkv, self.D, self.S_max,
                                      self.max_prefix, 0.0, self.dt, self.tree, self.attn_out, None, self.ws_attn,
                                      self.ws_attn_n, self.status)
            return
        if self.page_size > 0:
            _b.tree_attention_paged(q, k_tree, v_tree, k_cache, v_cache, block_table, self.max_pages, self.page_size,
                                    self.num_pages, prefix_len, self.B, self.Hq, self.Hkv, self.D, self.max_prefix,
                                    0.0, self.dt, self.tree, self.attn_out, None, self.ws_attn, self.ws_attn_n,
                                    self.status)
            return
        _b.tree_attention(q, k_tree, v_tree, k_cache, v_cache, prefix_len, self.B, self.Hq, self.Hkv, self.D,
                          self.S_max, self.max_prefix, 0.0, self.dt, self.tree, self.attn_out, None, self.ws_attn,
                          self.ws_attn_n, self.status)

    def verify(self, target, q=None, q_row=None, seed: int = 0, step: int = 0, node_tokens=None):
        tgt_dt = _b.dtype_code(target.dtype)
        if self.temperature > 0:
            _b.tree_verify_logits(target, tgt_dt, self.temperature, q, self.q_rows, q_row,
                                  self.node_tokens if node_tokens is None else node_tokens, self.B, self.V, self.tree,
                                  seed, step, self.accept_path, self.max_path, self.accept_len, self.bonus,
                                  self.ws_verify, self.ws_verify_n, self.status)
            return
        _b.tree_verify(self.mode, target, tgt_dt, q, self.q_rows if q is not None else 0, q_row,
                       self.node_tokens if node_tokens is None else node_tokens, self.B, self.V, self.tree, seed,
                       step, self.accept_path, self.max_path, self.accept_len, self.bonus, self.ws_verify,
                       self.ws_verify_n, self.status)

    def verify_commit(self, target, k_cache, v_cache, k_tree, v_tree, prefix_len, new_prefix_len, block_table=None,
                      node_tokens=None):
        """Greedy verification and the commit as run() issues them, in order on
        the current stream: the row scan, then the walk that commits the path
        it finds (one launch)."""
        _b.tree_verify_greedy_rows(target, _b.dtype_code(target.dtype), self.B, self.V, self.tree, self.ws_verify,
                                   self.ws_verify_n)
        paged = self.page_size > 0
        _b.tree_verify_greedy_walk_commit(self.node_tokens if node_tokens is None else node_tokens, self.B, self.V,
                                          self.tree, self.accept_path, self.max_path, self.accept_len, self.bonus,
                                          self.ws_verify, self.ws_verify_n, k_cache, v_cache, k_tree, v_tree,
                                          prefix_len, new_prefix_len, self.Hkv, self.D, self.S_max,
                                          block_table if paged else None, self.max_pages, self.page_size,
                                          self.num_pages, self.dt, self.status)

    def layer_pointers(self, k_layers, v_layers):
        """Device pointer arrays of the layers' caches, built once per list
        (build them before capturing a graph)."""
        key = tuple(c.data_ptr() for c in k_layers) + tuple(c.data_ptr() for c in v_layers)
        if key not in self._layer_ptrs:
            dev = k_layers[0].device
            self._layer_ptrs[key] = (_b.layer_pointers(k_layers, dev), _b.layer_pointers(v_layers, dev))
        return self._layer_ptrs[key]

    def compact(self, k_layers, v_layers, prefix_len, new_prefix_len):
        kp, vp = self.layer_pointers(k_layers, v_layers)
        _b.kv_compact(kp, vp, len(k_layers), self.accept_path, self.max_path, self.accept_len, prefix_len,
                      new_prefix_len, self.B, self.T, self.Hkv, self.D, self.S_max, self.dt, self.status)

    def commit(self, k_cache, v_cache, k_tree, v_tree, prefix_len, new_prefix_len, block_table=None,
               k_layers=None, v_layers=None):
        if self.tree_in_cache:
            self.compact(k_layers if k_layers is not None else [k_cache],
                         v_layers if v_layers is not None else [v_cache], prefix_len, new_prefix_len)
            return
        if self.page_size > 0:
            _b.kv_commit_paged(k_cache, v_cache, k_tree, v_tree, block_table, self.max_pages, self.page_size,
                               self.num_pages, self.accept_path, self.max_path, self.accept_len, prefix_len,
                               new_prefix_len, self.B, self.T, self.Hkv, self.D, self.dt, self.status)
            return
        _b.kv_commit(k_cache, v_cache, k_tree, v_tree, self.accept_path, self.max_path, self.accept_len, prefix_len,
                     new_prefix_len, self.B, self.T, self.Hkv, self.D, self.S_max, self.dt, self.status)

    def capture(self, **run_kwargs) -> "torch.cuda.CUDAGraph":
        """A CUDA graph of ``run(**run_kwargs)`` (the same buffers every
        replay): one launch per step instead of the four calls' host work.
        The buffers must stay allocated while the graph is used."""
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            self.run(**run_kwargs)
        return g

    def run(self, *, h, W_res, W_head, root_token, q, k_tree, v_tree, k_cache, v_cache, prefix_len, new_prefix_len,
            target, q_draft=None, q_row=None, seed: int = 0, step: int = 0, node_tokens=None, block_table=None,
            k_layers=None, v_layers=None):
        if self._side is None:
            self.heads(h, W_res, W_head, root_token)
            self.attention(q, k_tree, v_tree, k_cache, v_cache, prefix_len, block_table)
        else:
            main = torch.cuda.current_stream(self._side.device)
            greedy_split = self.mode == _b.GREEDY and self.temperature <= 0
            self._hp.wait_stream(main)        # every call sees everything issued before the step
            self._side.wait_stream(main)
            reserve = 0 < self.attention_sms < self._sms
            if reserve:
                _b.set_launch_shape(self._sms - self.attention_sms, 1)
            try:
                with torch.cuda.stream(self._hp):
                    self.heads(h, W_res, W_head, root_token)
                with torch.cuda.stream(self._side):
                    self.attention(q, k_tree, v_tree, k_cache, v_cache, prefix_len, block_table)
            finally:
                if reserve:
                    _b.set_launch_shape(0, 0)
            if greedy_split:
                self._side2.wait_stream(main)
                with torch.cuda.stream(self._side2):
                    _b.tree_verify_greedy_rows(target, _b.dtype_code(target.dtype), self.B, self.V, self.tree,
                                               self.ws_verify, self.ws_verify_n)
                main.wait_stream(self._side2)
            main.wait_stream(self._hp)        # the walk (or the whole verification) and commit after all
            main.wait_stream(self._side)
            tokens = self.node_tokens if node_tokens is None else node_tokens
            if greedy_split and not self.tree_in_cache:
                # the walk and the commit of the path it finds: one launch
                paged = self.page_size > 0
                _b.tree_verify_greedy_walk_commit(tokens, self.B, self.V, self.tree, self.accept_path, self.max_path,
                                                  self.accept_len, self.bonus, self.ws_verify, self.ws_verify_n,
                                                  k_cache, v_cache, k_tree, v_tree, prefix_len, new_prefix_len,
                                                  self.Hkv, self.D, self.S_max, block_table if paged else None,
                                                  self.max_pages, self.page_size, self.num_pages, self.dt,
                                                  self.status)
                return
            if greedy_split:
                _b.tree_verify_greedy_walk(tokens, self.B, self.V, self.tree, self.accept_path, self.max_path,
                                           self.accept_len, self.bonus, self.ws_verify, self.ws_verify_n)
            else:
                self.verify(target, q_draft, q_row, seed, step, node_tokens)
            self.commit(k_cache, v_cache, k_tree, v_tree, prefix_len, new_prefix_len, block_table, k_layers,
                        v_layers)
            return
        self.verify(target, q_draft, q_row, seed, step, node_tokens)
        self.commit(k_cache, v_cache, k_tree, v_tree, prefix_len, new_prefix_len, block_table, k_layers, v_layers)
