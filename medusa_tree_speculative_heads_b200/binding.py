"""ctypes binding of libmedusa.so (argument marshalling only).

Every function has the name and argument order of its C entry point in
include/medusa.h.  Tensors are torch CUDA tensors (or None for nullable
pointers); the current torch stream of the current device is used unless a
``stream`` is given.  Non-zero return codes raise :class:`MedusaError` with
the library's message.  There is no fallback: if the library was not built,
the first call raises.
"""
from __future__ import annotations

import ctypes
import os
import re
from typing import Optional, Sequence

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmedusa.so")
HEADER = os.path.join(os.path.dirname(_HERE), "include", "medusa.h")

MEDUSA_OK = 0
MEDUSA_ERR_INVALID_ARG = -1
MEDUSA_ERR_UNSUPPORTED = -2
MEDUSA_ERR_WORKSPACE = -3
MEDUSA_ERR_CUDA = -4

STATUS_BAD_TOKEN = 1
STATUS_CACHE_OVERFLOW = 2
STATUS_BAD_PREFIX = 4
STATUS_NO_MASS = 8
STATUS_TIMEOUT = 16
STATUS_BAD_PAGE = 32
STATUS_BAD_LAYER = 64

F32, BF16 = 0, 1
GREEDY, STOCHASTIC = 0, 1
TOPK = 8
MAX_TREE = 128

_lib = None


class MedusaError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"[{code}] {msg}")
        self.code = code


def lib() -> ctypes.CDLL:
    """Load libmedusa.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libmedusa.so not built ({LIB_PATH}); run medusa_tree_speculative_heads_b200/build.py")
        L = ctypes.CDLL(LIB_PATH)
        vp, i32, u32, u64, sz, f32 = (ctypes.c_void_p, ctypes.c_int, ctypes.c_uint32, ctypes.c_uint64, ctypes.c_size_t,
                                      ctypes.c_float)
        L.medusa_last_error.restype = ctypes.c_char_p
        L.medusa_last_error.argtypes = []
        L.medusa_version.restype = i32
        L.medusa_debug_set_wait_limit.argtypes = [u64]
        L.medusa_debug_set_wait_limit.restype = None
        L.medusa_set_launch_shape.argtypes = [i32, i32]
        L.medusa_tree_create.argtypes = [vp, i32, ctypes.POINTER(vp)]
        L.medusa_tree_destroy.argtypes = [vp]
        L.medusa_tree_info.argtypes = [vp, vp, vp, vp]
        L.medusa_tree_create_ragged.argtypes = [vp, vp, i32, ctypes.POINTER(vp)]
        L.medusa_tree_ntrees.argtypes = [vp, vp, vp]
        L.medusa_heads_workspace_size.argtypes = [i32, i32, i32, i32, i32]
        L.medusa_heads_workspace_size.restype = sz
        L.medusa_heads.argtypes = [vp, vp, vp, i32, i32, i32, i32, i32, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz,
                                   vp, vp]
        L.medusa_heads_noalloc.argtypes = [vp, vp, vp, i32, i32, i32, i32, i32, vp, vp, vp, vp, vp, vp, vp, vp,
                                           vp, vp, vp]
        L.tree_attention_workspace_size.argtypes = [i32, i32, i32, i32, i32, i32, vp, i32]
        L.tree_attention_workspace_size.restype = sz
        L.tree_attention.argtypes = [vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, f32, i32, vp, vp, vp, vp,
                                     sz, vp, vp]
        L.tree_verify_workspace_size.argtypes = [i32, i32, i32, vp]
        L.tree_verify_workspace_size.restype = sz
        L.tree_verify.argtypes = [i32, vp, i32, vp, i32, vp, vp, i32, i32, vp, u64, u32, vp, i32, vp, vp, vp, sz, vp,
                                  vp]
        L.tree_verify_greedy_rows.argtypes = [vp, i32, i32, i32, vp, vp, sz, vp]
        L.tree_verify_greedy_walk.argtypes = [vp, i32, i32, vp, vp, i32, vp, vp, vp, sz, vp]
        L.tree_verify_greedy_walk_commit.argtypes = [vp, i32, i32, vp, vp, i32, vp, vp, vp, sz, vp, vp, vp, vp, vp,
                                                     vp, i32, i32, i32, vp, i32, i32, i32, i32, vp, vp]
        L.tree_verify_logits.argtypes = [vp, i32, ctypes.c_double, vp, i32, vp, vp, i32, i32, vp, u64, u32, vp, i32,
                                         vp, vp, vp, sz, vp, vp]
        L.kv_commit.argtypes = [vp, vp, vp, vp, vp, i32, vp, vp, vp, i32, i32, i32, i32, i32, i32, vp, vp]
        L.medusa_heads_shard_workspace_size.argtypes = [i32, i32, i32, i32, i32]
        L.medusa_heads_shard_workspace_size.restype = sz
        L.medusa_heads_shard.argtypes = [vp, vp, vp, i32, i32, i32, i32, i32, i32, vp, vp, sz, vp, vp]
        L.medusa_heads_merge.argtypes = [vp, i32, i32, i32, i32, vp, vp, vp, vp, vp, vp, vp, vp]
        L.tree_attention_incache_workspace_size.argtypes = [i32, i32, i32, i32, i32, i32, vp, i32]
        L.tree_attention_incache_workspace_size.restype = sz
        L.tree_attention_incache.argtypes = [vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, f32, i32, vp, vp, vp, vp,
                                             sz, vp, vp]
        L.kv_compact.argtypes = [vp, vp, i32, vp, i32, vp, vp, vp, i32, i32, i32, i32, i32, i32, vp, vp]
        L.tree_attention_paged_workspace_size.argtypes = [i32, i32, i32, i32, i32, i32, i32, vp, i32]
        L.tree_attention_paged_workspace_size.restype = sz
        L.tree_attention_paged.argtypes = [vp, vp, vp, vp, vp, vp, i32, i32, i32, vp, i32, i32, i32, i32, i32, f32,
                                           i32, vp, vp, vp, vp, sz, vp, vp]
        L.kv_commit_paged.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, vp, i32, vp, vp, vp, i32, i32, i32, i32, i32,
                                      vp, vp]
        _lib = L
    return _lib


def declared_functions() -> list:
    """Names of the functions include/medusa.h declares."""
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s*([a-z_][a-z0-9_]*)\s*\(", src,
                                 flags=re.M)))


def _check(rc: int):
    if rc != MEDUSA_OK:
        raise MedusaError(rc, lib().medusa_last_error().decode())


def _p(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    if isinstance(stream, torch.cuda.Stream):
        stream = stream.cuda_stream
    return ctypes.c_void_p(int(stream))


def dtype_code(t: torch.dtype) -> int:
    if t == torch.float32:
        return F32
    if t == torch.bfloat16:
        return BF16
    raise TypeError(f"unsupported dtype {t}")


def version() -> int:
    return lib().medusa_version()


def set_launch_shape(heads_ctas: int, attention_splits: int) -> None:
    """medusa_set_launch_shape for later calls from this thread (0, 0: default)."""
    _check(lib().medusa_set_launch_shape(int(heads_ctas), int(attention_splits)))


def set_wait_limit(ns: int) -> None:
    """medusa_debug_set_wait_limit: limit of the kernels' pipeline waits for
    later calls (0: the default of about two seconds; 1: give up at once)."""
    lib().medusa_debug_set_wait_limit(ctypes.c_uint64(int(ns)))


class Tree:
    """Owner of a medusa_tree handle (created on the current device): one
    parent list (a tree shared by every sequence) or a list of parent lists
    (one tree per sequence, medusa_tree_create_ragged)."""

    def __init__(self, parents):
        h = ctypes.c_void_p()
        if len(parents) > 0 and hasattr(parents[0], "__len__"):
            flat = [int(x) for p in parents for x in p]
            offs = [0]
            for p in parents:
                offs.append(offs[-1] + len(p))
            arr = (ctypes.c_int32 * max(len(flat), 1))(*flat)
            off = (ctypes.c_int32 * len(offs))(*offs)
            _check(lib().medusa_tree_create_ragged(arr, off, len(parents), ctypes.byref(h)))
            self.parents = [[int(x) for x in p] for p in parents]
        else:
            arr = (ctypes.c_int32 * len(parents))(*[int(x) for x in parents])
            _check(lib().medusa_tree_create(arr, len(parents), ctypes.byref(h)))
            self.parents = [int(x) for x in parents]
        self.handle = h
        T, dep, mc = ctypes.c_int(), ctypes.c_int(), ctypes.c_int()
        _check(lib().medusa_tree_info(h, ctypes.byref(T), ctypes.byref(dep), ctypes.byref(mc)))
        self.T, self.max_depth, self.max_children = T.value, dep.value, mc.value
        n = ctypes.c_int()
        _check(lib().medusa_tree_ntrees(h, ctypes.byref(n), None))
        each = (ctypes.c_int32 * n.value)()
        _check(lib().medusa_tree_ntrees(h, ctypes.byref(n), each))
        self.ntrees, self.T_each = n.value, list(each)

    def close(self):
        if self.handle:
            _check(lib().medusa_tree_destroy(self.handle))
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def medusa_heads_workspace_size(B: int, d: int, V: int, K: int, dt: int) -> int:
    return lib().medusa_heads_workspace_size(B, d, V, K, dt)


def medusa_heads(h, W_res, W_head, B, d, V, K, dt, tree: Optional[Tree], root_token, topk_idx, topk_prob,
                 node_tokens, node_q, h_res_out, logits_out, probs_out, workspace, workspace_bytes, status,
                 stream=None):
    _check(lib().medusa_heads(_p(h), _p(W_res), _p(W_head), B, d, V, K, dt, tree.handle if tree else None,
                              _p(root_token), _p(topk_idx), _p(topk_prob), _p(node_tokens), _p(node_q),
                              _p(h_res_out), _p(logits_out), _p(probs_out), _p(workspace), workspace_bytes,
                              _p(status), _stream(stream)))


def medusa_heads_noalloc(h, W_res, W_head, B, d, V, K, dt, tree: Optional[Tree], root_token, topk_idx, topk_prob,
                         node_tokens, node_q, h_res_out, logits_out, probs_out, status, stream=None):
    """medusa_heads for callers that cannot allocate device memory: the
    scratch is a fixed array inside the library (see include/medusa.h)."""
    _check(lib().medusa_heads_noalloc(_p(h), _p(W_res), _p(W_head), B, d, V, K, dt, tree.handle if tree else None,
                                      _p(root_token), _p(topk_idx), _p(topk_prob), _p(node_tokens), _p(node_q),
                                      _p(h_res_out), _p(logits_out), _p(probs_out), _p(status), _stream(stream)))


def tree_attention_workspace_size(B, Hq, Hkv, D, S_max, max_prefix, tree: Tree, dt) -> int:
    return lib().tree_attention_workspace_size(B, Hq, Hkv, D, S_max, max_prefix, tree.handle, dt)


def tree_attention(q, k_tree, v_tree, k_cache, v_cache, prefix_len, B, Hq, Hkv, D, S_max, max_prefix, scale, dt,
                   tree: Tree, out, lse, workspace, workspace_bytes, status, stream=None):
    _check(lib().tree_attention(_p(q), _p(k_tree), _p(v_tree), _p(k_cache), _p(v_cache), _p(prefix_len), B, Hq,
                                Hkv, D, S_max, max_prefix, float(scale), dt, tree.handle, _p(out), _p(lse),
                                _p(workspace), workspace_bytes, _p(status), _stream(stream)))


def tree_verify_workspace_size(mode, B, V, tree: Tree) -> int:
    return lib().tree_verify_workspace_size(mode, B, V, tree.handle)


def tree_verify(mode, target, target_dt, q, q_rows, q_row, node_tokens, B, V, tree: Tree, seed, step, accept_path,
                max_path, accept_len, bonus, workspace, workspace_bytes, status, stream=None):
    _check(lib().tree_verify(mode, _p(target), target_dt, _p(q), q_rows, _p(q_row), _p(node_tokens), B, V,
                             tree.handle, ctypes.c_uint64(seed & (2**64 - 1)), ctypes.c_uint32(step & 0xFFFFFFFF),
                             _p(accept_path), max_path, _p(accept_len), _p(bonus), _p(workspace), workspace_bytes,
                             _p(status), _stream(stream)))


def tree_verify_greedy_rows(target, target_dt, B, V, tree: Tree, workspace, workspace_bytes, stream=None):
    _check(lib().tree_verify_greedy_rows(_p(target), target_dt, B, V, tree.handle, _p(workspace), workspace_bytes,
                                         _stream(stream)))


def tree_verify_greedy_walk(node_tokens, B, V, tree: Tree, accept_path, max_path, accept_len, bonus, workspace,
                            workspace_bytes, stream=None):
    _check(lib().tree_verify_greedy_walk(_p(node_tokens), B, V, tree.handle, _p(accept_path), max_path,
                                         _p(accept_len), _p(bonus), _p(workspace), workspace_bytes, _stream(stream)))


def tree_verify_greedy_walk_commit(node_tokens, B, V, tree: Tree, accept_path, max_path, accept_len, bonus, workspace,
                                   workspace_bytes, k_cache, v_cache, k_tree, v_tree, prefix_len, new_prefix_len, Hkv,
                                   D, S_max, block_table, max_pages, page_size, num_pages, dt, status, stream=None):
    _check(lib().tree_verify_greedy_walk_commit(_p(node_tokens), B, V, tree.handle, _p(accept_path), max_path,
                                                _p(accept_len), _p(bonus), _p(workspace), workspace_bytes,
                                                _p(k_cache), _p(v_cache), _p(k_tree), _p(v_tree), _p(prefix_len),
                                                _p(new_prefix_len), Hkv, D, S_max, _p(block_table), max_pages,
                                                page_size, num_pages, dt, _p(status), _stream(stream)))


def tree_verify_logits(logits, logits_dt, temperature, q, q_rows, q_row, node_tokens, B, V, tree: Tree, seed, step,
                       accept_path, max_path, accept_len, bonus, workspace, workspace_bytes, status, stream=None):
    _check(lib().tree_verify_logits(_p(logits), logits_dt, float(temperature), _p(q), q_rows, _p(q_row),
                                    _p(node_tokens), B, V, tree.handle, ctypes.c_uint64(seed & (2**64 - 1)),
                                    ctypes.c_uint32(step & 0xFFFFFFFF), _p(accept_path), max_path, _p(accept_len),
                                    _p(bonus), _p(workspace), workspace_bytes, _p(status), _stream(stream)))


PARTIAL_BYTES = 72   # sizeof(medusa_head_partial): m, l, 8 logits, 8 int32 ids


def medusa_heads_shard_workspace_size(B, d, V_shard, K, dt) -> int:
    return lib().medusa_heads_shard_workspace_size(B, d, V_shard, K, dt)


def medusa_heads_shard(h, W_res, W_head_shard, B, d, V_shard, v_offset, K, dt, partial_out, workspace,
                       workspace_bytes, status, stream=None):
    _check(lib().medusa_heads_shard(_p(h), _p(W_res), _p(W_head_shard), B, d, V_shard, v_offset, K, dt,
                                    _p(partial_out), _p(workspace), workspace_bytes, _p(status), _stream(stream)))


def medusa_heads_merge(partials, n_shards, B, K, V, tree: Optional[Tree], root_token, topk_idx, topk_prob,
                       node_tokens, node_q, status, stream=None):
    _check(lib().medusa_heads_merge(_p(partials), n_shards, B, K, V, tree.handle if tree is not None else None,
                                    _p(root_token), _p(topk_idx), _p(topk_prob), _p(node_tokens), _p(node_q),
                                    _p(status), _stream(stream)))


def tree_attention_incache_workspace_size(B, Hq, Hkv, D, S_max, max_prefix, tree: Tree, dt) -> int:
    return lib().tree_attention_incache_workspace_size(B, Hq, Hkv, D, S_max, max_prefix, tree.handle, dt)


def tree_attention_incache(q, k_cache, v_cache, prefix_len, B, Hq, Hkv, D, S_max, max_prefix, scale, dt, tree: Tree,
                           out, lse, workspace, workspace_bytes, status, stream=None):
    _check(lib().tree_attention_incache(_p(q), _p(k_cache), _p(v_cache), _p(prefix_len), B, Hq, Hkv, D, S_max,
                                        max_prefix, float(scale), dt, tree.handle, _p(out), _p(lse), _p(workspace),
                                        workspace_bytes, _p(status), _stream(stream)))


def kv_compact(k_ptrs, v_ptrs, n_layers, accept_path, max_path, accept_len, prefix_len, new_prefix_len, B, T, Hkv, D,
               S_max, dt, status, stream=None):
    """k_ptrs, v_ptrs: device int64 tensors [n_layers] holding each layer's
    cache address (see layer_pointers)."""
    _check(lib().kv_compact(_p(k_ptrs), _p(v_ptrs), n_layers, _p(accept_path), max_path, _p(accept_len),
                            _p(prefix_len), _p(new_prefix_len), B, T, Hkv, D, S_max, dt, _p(status),
                            _stream(stream)))


def layer_pointers(caches, device) -> torch.Tensor:
    """A device int64 tensor of the caches' addresses (the pointer array
    kv_compact takes)."""
    return torch.tensor([c.data_ptr() for c in caches], dtype=torch.int64).to(device)


def kv_commit(k_cache, v_cache, k_tree, v_tree, accept_path, max_path, accept_len, prefix_len, new_prefix_len, B, T,
              Hkv, D, S_max, dt, status, stream=None):
    _check(lib().kv_commit(_p(k_cache), _p(v_cache), _p(k_tree), _p(v_tree), _p(accept_path), max_path,
                           _p(accept_len), _p(prefix_len), _p(new_prefix_len), B, T, Hkv, D, S_max, dt, _p(status),
                           _stream(stream)))


def tree_attention_paged_workspace_size(B, Hq, Hkv, D, max_prefix, max_pages, page_size, tree: Tree, dt) -> int:
    return lib().tree_attention_paged_workspace_size(B, Hq, Hkv, D, max_prefix, max_pages, page_size, tree.handle, dt)


def tree_attention_paged(q, k_tree, v_tree, k_pages, v_pages, block_table, max_pages, page_size, num_pages,
                         prefix_len, B, Hq, Hkv, D, max_prefix, scale, dt, tree: Tree, out, lse, workspace,
                         workspace_bytes, status, stream=None):
    _check(lib().tree_attention_paged(_p(q), _p(k_tree), _p(v_tree), _p(k_pages), _p(v_pages), _p(block_table),
                                      max_pages, page_size, num_pages, _p(prefix_len), B, Hq, Hkv, D, max_prefix,
                                      float(scale), dt, tree.handle, _p(out), _p(lse), _p(workspace), workspace_bytes,
                                      _p(status), _stream(stream)))


def kv_commit_paged(k_pages, v_pages, k_tree, v_tree, block_table, max_pages, page_size, num_pages, accept_path,
                    max_path, accept_len, prefix_len, new_prefix_len, B, T, Hkv, D, dt, status, stream=None):
    _check(lib().kv_commit_paged(_p(k_pages), _p(v_pages), _p(k_tree), _p(v_tree), _p(block_table), max_pages,
                                 page_size, num_pages, _p(accept_path), max_path, _p(accept_len), _p(prefix_len),
                                 _p(new_prefix_len), B, T, Hkv, D, dt, _p(status), _stream(stream)))
