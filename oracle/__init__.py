"""fp64 CPU oracle of one Medusa speculative decode step (ctypes wrapper).

TEST INFRASTRUCTURE ONLY: the tests, the package's smoke check and the
benchmark's timed CPU baseline use it; the product path never does.  The
arithmetic lives in ``oracle.c`` (plain C, fp64, loops); this module only
builds it with gcc and marshals torch/numpy buffers.  It imports nothing from
the CUDA package.

Parity status: every function here is pinned by ``tests/test_oracle.py``
(hand computations, closed forms, brute force, library cross-checks,
statistical tests); none is "parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Sequence

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_LIB_OMP = os.path.join(_HERE, "liboracle_omp.so")   # the same source built with OpenMP
_lib = None
_lib_omp = None
_use_omp = False
_CFLAGS = ["-O2", "-std=gnu11", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared"]

F32, BF16 = 0, 1


def build(force: bool = False) -> str:
    """Compile oracle.c with gcc (no FMA contraction) into liboracle.so, and
    the same source with OpenMP into liboracle_omp.so.  The OpenMP build only
    shares independent output elements (rows, vocabulary entries) among
    threads; each element's arithmetic is the serial build's, so the two give
    bit-identical results."""
    for out, extra in ((_LIB, []), (_LIB_OMP, ["-fopenmp"])):
        if force or not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(_SRC):
            subprocess.check_call(["gcc"] + _CFLAGS + extra + ["-o", out + ".tmp", _SRC, "-lm"])
            os.replace(out + ".tmp", out)
    return _LIB


def lib():
    global _lib, _lib_omp
    if _use_omp:
        if _lib_omp is None:
            build()
            _lib_omp = configure(ctypes.CDLL(_LIB_OMP))
        return _lib_omp
    if _lib is None:
        build()
        _lib = configure(ctypes.CDLL(_LIB))
    return _lib


def use_openmp(on: bool = True) -> None:
    """Route later calls to the OpenMP build (on) or the serial one (off)."""
    global _use_omp
    _use_omp = bool(on)


def threads() -> int:
    """Threads the build currently in use runs its parallel loops on."""
    return int(lib().orc_threads())


def configure(L):
    """Declares the argument and result types of every oracle function on a
    loaded copy of the library (the tests also load deliberately broken
    builds of oracle.c through it)."""
    vp, i32, i64, u32, u64, dbl = (ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_uint32,
                                   ctypes.c_uint64, ctypes.c_double)
    L.orc_tree_mask.argtypes = [vp, i32, vp]
    L.orc_tree_shape.argtypes = [vp, i32, vp, vp]
    L.orc_product_tree.argtypes = [vp, i32, vp, i32]
    L.orc_heads.argtypes = [vp, vp, vp, i32, i32, i32, i32, i32, i32, i32, i32, vp, vp, vp]
    L.orc_threads.argtypes = []
    L.orc_threads.restype = i32
    L.orc_heads.restype = None
    L.orc_topk.argtypes = [vp, i32, i32, vp]
    L.orc_topk.restype = None
    L.orc_tree_fill.argtypes = [vp, i32, i32, i32, i32, vp, vp, vp, vp, vp]
    L.orc_tree_attention.argtypes = [vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, i32, dbl, vp,
                                     i32, vp, vp, vp]
    L.orc_verify_greedy.argtypes = [vp, i32, vp, i32, i32, i32, vp, i32, vp, vp, vp]
    L.orc_philox4x32_10.argtypes = [vp, vp, vp]
    L.orc_philox4x32_10.restype = None
    L.orc_verify_stochastic.argtypes = [vp, vp, i32, vp, vp, i32, i32, i32, vp, u64, u32, i32, vp, vp, vp,
                                        vp, i32]
    L.orc_verify_stochastic_logits.argtypes = [vp, i32, dbl, vp, i32, vp, vp, i32, i32, i32, vp, u64, u32,
                                               i32, vp, vp, vp, vp, i32]
    L.orc_softmax_temperature.argtypes = [vp, i32, dbl, vp]
    L.orc_softmax_temperature.restype = None
    L.orc_kv_compact.argtypes = [vp, vp, i32, vp, i32, vp, vp, vp, i32, i32, i32, i32, i32, i32, vp]
    L.orc_kv_compact.restype = None
    L.orc_kv_commit.argtypes = [vp, vp, vp, vp, vp, i32, vp, vp, vp, i32, i32, i32, i32, i32, i32, vp]
    L.orc_kv_commit.restype = None
    L.orc_gather_pages.argtypes = [vp, vp, i32, i32, i32, vp, i32, i32, i32, i32, i32, vp]
    L.orc_gather_pages.restype = i32
    L.orc_kv_commit_paged.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, vp, i32, vp, vp, vp, i32, i32, i32, i32,
                                      i32, vp]
    L.orc_kv_commit_paged.restype = None
    L.orc_residual.argtypes = [vp, vp, i32, vp, vp]
    L.orc_residual.restype = u64
    L.orc_round_bf16.argtypes = [dbl]
    L.orc_round_bf16.restype = dbl
    return L


# ----------------------------------------------------------------------------
# marshalling helpers
# ----------------------------------------------------------------------------

def _raw(t):
    """(contiguous numpy array of the raw elements, dtype code)."""
    if isinstance(t, torch.Tensor):
        t = t.detach().cpu().contiguous()
        if t.dtype == torch.bfloat16:
            return t.view(torch.int16).numpy(), BF16
        if t.dtype == torch.float32:
            return t.numpy(), F32
        raise TypeError(f"oracle takes fp32/bf16 tensors, got {t.dtype}")
    a = np.ascontiguousarray(t)
    if a.dtype == np.float32:
        return a, F32
    raise TypeError(f"oracle takes fp32 arrays, got {a.dtype}")


def _i32(x) -> np.ndarray:
    if isinstance(x, torch.Tensor):
        x = x.detach().cpu().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.int32))


def _f32(x) -> np.ndarray:
    if isinstance(x, torch.Tensor):
        x = x.detach().cpu().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float32))


def _p(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


# ----------------------------------------------------------------------------
# tree
# ----------------------------------------------------------------------------

def tree_mask(parents: Sequence[int]) -> np.ndarray:
    par = _i32(parents)
    T = len(par)
    anc = np.zeros((T, T), dtype=np.uint8)
    if lib().orc_tree_mask(_p(par), T, _p(anc)) != 0:
        raise ValueError("bad parent array")
    return anc


def tree_shape(parents: Sequence[int]):
    par = _i32(parents)
    T = len(par)
    depth = np.zeros(T, np.int32)
    rank = np.zeros(T, np.int32)
    if lib().orc_tree_shape(_p(par), T, _p(depth), _p(rank)) != 0:
        raise ValueError("not a single-rooted topologically ordered tree")
    return depth, rank


def product_tree(branching: Sequence[int], cap: int = 4096) -> np.ndarray:
    s = _i32(branching)
    par = np.zeros(cap, np.int32)
    n = lib().orc_product_tree(_p(s), len(s), _p(par), cap)
    if n < 0:
        raise ValueError("tree too large")
    return par[:n].copy()


# ----------------------------------------------------------------------------
# heads
# ----------------------------------------------------------------------------

def heads(h, W_res, W_head, b_only: int = -1, k_only: int = -1, want_hk=True, want_probs=True,
          exact_hk: bool = False):
    """Returns dict of fp64 arrays hk [B,K,d], logits [B,K,V], probs [B,K,V]
    (rows not selected by b_only/k_only are NaN).  For bf16 inputs h^(k) is
    rounded to bf16 before the vocabulary projection, unless exact_hk keeps
    its exact fp64 value."""
    hr, dt = _raw(h)
    wr, dt2 = _raw(W_res)
    wh, dt3 = _raw(W_head)
    assert dt == dt2 == dt3
    B, d = h.shape
    K, V, _ = W_head.shape
    hk = np.full((B, K, d), np.nan) if want_hk else None
    logits = np.full((B, K, V), np.nan)
    probs = np.full((B, K, V), np.nan) if want_probs else None
    lib().orc_heads(_p(hr), _p(wr), _p(wh), dt, B, d, V, K, b_only, k_only, 0 if exact_hk else 1, _p(hk), _p(logits),
                    _p(probs))
    return {"hk": hk, "logits": logits, "probs": probs}


def round_bf16(x: float) -> float:
    return lib().orc_round_bf16(float(x))


def topk(x: np.ndarray, s: int) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float64)
    idx = np.zeros(s, np.int32)
    lib().orc_topk(_p(x), x.shape[0], s, _p(idx))
    return idx


def tree_fill(parents, root_token, topk_idx, topk_p):
    par = _i32(parents)
    ti = _i32(topk_idx)
    tp = np.ascontiguousarray(topk_p, dtype=np.float64)
    B, K, S = ti.shape
    T = len(par)
    rt = _i32(root_token)
    tok = np.zeros((B, T), np.int32)
    nq = np.zeros((B, T), np.float64)
    if lib().orc_tree_fill(_p(par), T, B, K, S, _p(rt), _p(ti), _p(tp), _p(tok), _p(nq)) != 0:
        raise ValueError("tree does not fit the heads")
    return tok, nq


# ----------------------------------------------------------------------------
# attention
# ----------------------------------------------------------------------------

def tree_attention(q, k_tree, v_tree, k_cache, v_cache, prefix_len, parents, scale: float = 0.0,
                   rows: Optional[np.ndarray] = None):
    """Returns (out [nrows, D] fp64, lse [nrows] fp64); rows: int array
    [n, 3] of (b, i, h), or None for all rows in (b, i, h) order."""
    qa, dt = _raw(q)
    kt, _ = _raw(k_tree)
    vt, _ = _raw(v_tree)
    kc, _ = _raw(k_cache)
    vc, _ = _raw(v_cache)
    B, T, Hq, D = q.shape
    Hkv = k_tree.shape[2]
    S_max = k_cache.shape[2]
    pl = _i32(prefix_len)
    par = _i32(parents)
    r = None if rows is None else _i32(rows).reshape(-1, 3)
    n = B * T * Hq if r is None else r.shape[0]
    out = np.zeros((n, D))
    lse = np.zeros(n)
    rc = lib().orc_tree_attention(_p(qa), _p(kt), _p(vt), _p(kc), _p(vc), _p(pl), dt, B, T, Hq, Hkv, D, S_max,
                                  float(scale), _p(par), n, _p(r), _p(out), _p(lse))
    if rc != 0:
        raise ValueError("bad attention arguments")
    return out, lse


def tree_rows_from_cache(cache, prefix_len, T: int):
    """The tree's K or V [B, T, Hkv, D] when they sit in the cache [B, Hkv,
    S_max, D] at rows prefix_len[b] .. prefix_len[b] + T - 1 (rows past S_max
    read as zeros)."""
    c = cache.detach().cpu()
    B, Hkv, S_max, D = c.shape
    out = torch.zeros((B, T, Hkv, D), dtype=c.dtype)
    for b in range(B):
        S = int(prefix_len[b])
        n = max(0, min(T, S_max - S))
        out[b, :n] = c[b, :, S:S + n].transpose(0, 1)
    return out


def tree_attention_incache(q, k_cache, v_cache, prefix_len, parents, scale: float = 0.0,
                           rows: Optional[np.ndarray] = None):
    """tree_attention with the tree's K/V read from the cache rows right after
    each prefix."""
    T = q.shape[1]
    kt = tree_rows_from_cache(k_cache, prefix_len, T)
    vt = tree_rows_from_cache(v_cache, prefix_len, T)
    return tree_attention(q, kt, vt, k_cache, v_cache, prefix_len, parents, scale, rows)


# ----------------------------------------------------------------------------
# verification
# ----------------------------------------------------------------------------

def verify_greedy(logits, node_tokens, parents, max_path: int):
    la, dt = _raw(logits)
    B, T, V = logits.shape
    nt = _i32(node_tokens)
    par = _i32(parents)
    path = np.zeros((B, max_path), np.int32)
    ln = np.zeros(B, np.int32)
    bonus = np.zeros(B, np.int32)
    if lib().orc_verify_greedy(_p(la), dt, _p(nt), B, T, V, _p(par), max_path, _p(path), _p(ln),
                               _p(bonus)) != 0:
        raise ValueError("bad verify arguments")
    return path, ln, bonus


def philox4x32_10(ctr: Sequence[int], key: Sequence[int]) -> np.ndarray:
    c = np.asarray(ctr, dtype=np.uint32)
    k = np.asarray(key, dtype=np.uint32)
    out = np.zeros(4, np.uint32)
    lib().orc_philox4x32_10(_p(c), _p(k), _p(out))
    return out


def residual(P, Q):
    """(out fp64 [V], W uint64 [V], S) of the quantised residual."""
    Pa = np.ascontiguousarray(P, dtype=np.float64)
    Qa = _f32(Q)
    V = Pa.shape[0]
    out = np.zeros(V)
    W = np.zeros(V, np.uint64)
    S = lib().orc_residual(_p(Pa), _p(Qa), V, _p(out), _p(W))
    return out, W, int(S)


def verify_stochastic(p, q, node_tokens, parents, seed: int, step: int, max_path: int, q_row=None, b0: int = 0):
    """Rows of p, q, node_tokens are sequences b0, b0+1, ... of the batch (the
    sequence index selects the Philox counter)."""
    pa = _f32(p)
    qa = _f32(q)
    B, T, V = pa.shape
    Qrows = qa.shape[1]
    nt = _i32(node_tokens)
    par = _i32(parents)
    qr = None if q_row is None else _i32(q_row)
    path = np.zeros((B, max_path), np.int32)
    ln = np.zeros(B, np.int32)
    bonus = np.zeros(B, np.int32)
    status = np.zeros(1, np.int32)
    rc = lib().orc_verify_stochastic(_p(pa), _p(qa), Qrows, _p(qr), _p(nt), B, T, V, _p(par),
                                     ctypes.c_uint64(seed & (2**64 - 1)), ctypes.c_uint32(step & 0xFFFFFFFF),
                                     max_path, _p(path), _p(ln), _p(bonus), _p(status), int(b0))
    if rc != 0:
        raise ValueError("bad verify arguments")
    return path, ln, bonus, int(status[0])


def softmax_temperature(z, temperature: float):
    """fp64 P = softmax((z - max z) / tau) of one logits row (numpy f64)."""
    za = np.ascontiguousarray(np.asarray(z, dtype=np.float64))
    out = np.empty_like(za)
    lib().orc_softmax_temperature(_p(za), za.shape[0], ctypes.c_double(1.0 / temperature), _p(out))
    return out


def verify_stochastic_logits(logits, temperature: float, q, node_tokens, parents, seed: int, step: int,
                             max_path: int, q_row=None, b0: int = 0):
    """verify_stochastic with every visited node's target distribution taken
    as softmax(logits row / temperature) in fp64 (logits f32 or bf16 torch)."""
    lg = logits.detach().cpu().contiguous()
    dt = BF16 if lg.dtype == torch.bfloat16 else F32
    if dt == F32:
        lg = lg.float()
    qa = _f32(q)
    B, T, V = lg.shape
    Qrows = qa.shape[1]
    nt = _i32(node_tokens)
    par = _i32(parents)
    qr = None if q_row is None else _i32(q_row)
    path = np.zeros((B, max_path), np.int32)
    ln = np.zeros(B, np.int32)
    bonus = np.zeros(B, np.int32)
    status = np.zeros(1, np.int32)
    rc = lib().orc_verify_stochastic_logits(ctypes.c_void_p(lg.data_ptr()), dt, ctypes.c_double(temperature),
                                            _p(qa), Qrows, _p(qr), _p(nt), B, T, V, _p(par),
                                            ctypes.c_uint64(seed & (2**64 - 1)), ctypes.c_uint32(step & 0xFFFFFFFF),
                                            max_path, _p(path), _p(ln), _p(bonus), _p(status), int(b0))
    if rc != 0:
        raise ValueError("bad verify arguments")
    return path, ln, bonus, int(status[0])


# ----------------------------------------------------------------------------
# commit
# ----------------------------------------------------------------------------

def kv_commit(k_cache, v_cache, k_tree, v_tree, path, length, prefix_len):
    """Returns (k_cache', v_cache', new_prefix_len, status) as new torch
    tensors; inputs untouched."""
    kc = k_cache.detach().cpu().contiguous().clone()
    vc = v_cache.detach().cpu().contiguous().clone()
    kt = k_tree.detach().cpu().contiguous()
    vt = v_tree.detach().cpu().contiguous()
    B, Hkv, S_max, D = kc.shape
    T = kt.shape[1]
    pa = _i32(path)
    max_path = pa.shape[1]
    ln = _i32(length)
    pl = _i32(prefix_len)
    npl = np.zeros(B, np.int32)
    status = np.zeros(1, np.int32)
    esize = kc.element_size()
    lib().orc_kv_commit(ctypes.c_void_p(kc.data_ptr()), ctypes.c_void_p(vc.data_ptr()),
                        ctypes.c_void_p(kt.data_ptr()), ctypes.c_void_p(vt.data_ptr()), _p(pa), max_path, _p(ln),
                        _p(pl), _p(npl), B, Hkv, D, S_max, T, esize, _p(status))
    return kc, vc, npl, int(status[0])


def kv_compact(k_layers, v_layers, path, length, prefix_len, T: int):
    """Returns (k_layers', v_layers', new_prefix_len, status): new torch
    tensors (the layers stacked [n_layers, B, Hkv, S_max, D]); inputs
    untouched."""
    kc = torch.stack([x.detach().cpu() for x in k_layers]).contiguous().clone()
    vc = torch.stack([x.detach().cpu() for x in v_layers]).contiguous().clone()
    n_layers, B, Hkv, S_max, D = kc.shape
    pa = _i32(path)
    max_path = pa.shape[1]
    ln = _i32(length)
    pl = _i32(prefix_len)
    npl = np.zeros(B, np.int32)
    status = np.zeros(1, np.int32)
    lib().orc_kv_compact(ctypes.c_void_p(kc.data_ptr()), ctypes.c_void_p(vc.data_ptr()), n_layers, _p(pa), max_path,
                         _p(ln), _p(pl), _p(npl), B, Hkv, D, S_max, T, kc.element_size(), _p(status))
    return kc, vc, npl, int(status[0])


# ----------------------------------------------------------------------------
# paged KV cache
# ----------------------------------------------------------------------------

def gather_pages(pages, table, n_pos, S_max: int, fill=None):
    """Contiguous cache [B, Hkv, S_max, D] (torch, pages' dtype) holding
    positions s < n_pos[b] of each sequence read through the block table;
    other entries are `fill` (zeros when None)."""
    pg = pages.detach().cpu().contiguous()
    num_pages, Hkv, page_size, D = pg.shape
    tb = _i32(table)
    B, max_pages = tb.shape
    npos = _i32(n_pos)
    cache = torch.zeros((B, Hkv, S_max, D), dtype=pg.dtype) if fill is None else \
        torch.full((B, Hkv, S_max, D), fill, dtype=pg.dtype)
    rc = lib().orc_gather_pages(ctypes.c_void_p(pg.data_ptr()), _p(tb), max_pages, page_size, num_pages, _p(npos),
                                B, Hkv, D, S_max, pg.element_size(), ctypes.c_void_p(cache.data_ptr()))
    if rc != 0:
        raise ValueError("block table does not cover the positions")
    return cache


def kv_commit_paged(k_pages, v_pages, k_tree, v_tree, table, path, length, prefix_len):
    """Returns (k_pages', v_pages', new_prefix_len, status); inputs untouched."""
    kp = k_pages.detach().cpu().contiguous().clone()
    vp_ = v_pages.detach().cpu().contiguous().clone()
    kt = k_tree.detach().cpu().contiguous()
    vt = v_tree.detach().cpu().contiguous()
    num_pages, Hkv, page_size, D = kp.shape
    B, T = kt.shape[0], kt.shape[1]
    tb = _i32(table)
    pa = _i32(path)
    ln = _i32(length)
    pl = _i32(prefix_len)
    npl = np.zeros(B, np.int32)
    status = np.zeros(1, np.int32)
    lib().orc_kv_commit_paged(ctypes.c_void_p(kp.data_ptr()), ctypes.c_void_p(vp_.data_ptr()),
                              ctypes.c_void_p(kt.data_ptr()), ctypes.c_void_p(vt.data_ptr()), _p(tb), tb.shape[1],
                              page_size, num_pages, _p(pa), pa.shape[1], _p(ln), _p(pl), _p(npl), B, Hkv, D, T,
                              kp.element_size(), _p(status))
    return kp, vp_, npl, int(status[0])
