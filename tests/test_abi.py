"""Host-side checks of the C ABI that need no GPU: the library builds, loads
and exports every function include/medusa.h declares, and argument errors
are reported by return code before anything reaches the device."""
import ctypes
import os
import re

import pytest

from medusa_tree_speculative_heads_b200 import binding as B
from medusa_tree_speculative_heads_b200 import build as build_mod


@pytest.fixture(scope="module")
def lib():
    build_mod.build()
    return B.lib()


def test_header_declares_the_four_step_calls():
    names = B.declared_functions()
    for n in ("medusa_heads", "tree_attention", "tree_verify", "kv_commit", "medusa_tree_create",
              "medusa_tree_destroy", "medusa_last_error"):
        assert n in names, n


def test_library_exports_every_declared_symbol(lib):
    missing = [n for n in B.declared_functions() if not hasattr(lib, n)]
    assert not missing, missing
    assert lib.medusa_version() == 100


def test_sm100a_only():
    src = open(build_mod.__file__).read()
    assert "arch=compute_100a,code=sm_100a" in src


def test_tree_create_rejects_bad_parents(lib):
    h = ctypes.c_void_p()
    for parents, code in (([0, 0], B.MEDUSA_ERR_INVALID_ARG), ([-1, 1], B.MEDUSA_ERR_INVALID_ARG),
                          ([-1, 0, -1], B.MEDUSA_ERR_INVALID_ARG), ([-1, 0, 5], B.MEDUSA_ERR_INVALID_ARG),
                          ([-1] + list(range(128)), B.MEDUSA_ERR_UNSUPPORTED)):
        arr = (ctypes.c_int32 * len(parents))(*parents)
        assert lib.medusa_tree_create(arr, len(parents), ctypes.byref(h)) == code
        assert lib.medusa_last_error()
    assert lib.medusa_tree_create(None, 3, ctypes.byref(h)) == B.MEDUSA_ERR_INVALID_ARG


def test_ragged_tree_create_rejects_bad_trees(lib):
    # validation happens on the host, before any device allocation
    h = ctypes.c_void_p()

    def create(trees):
        flat = [x for t in trees for x in t]
        offs = [0]
        for t in trees:
            offs.append(offs[-1] + len(t))
        arr = (ctypes.c_int32 * max(len(flat), 1))(*flat)
        off = (ctypes.c_int32 * len(offs))(*offs)
        return lib.medusa_tree_create_ragged(arr, off, len(trees), ctypes.byref(h))

    assert create([[-1, 0], [-1, 1]]) == B.MEDUSA_ERR_INVALID_ARG
    assert b"tree 1" in lib.medusa_last_error()
    assert create([[-1, 0, 0], [-1] + list(range(128))]) == B.MEDUSA_ERR_UNSUPPORTED
    assert b"tree 1" in lib.medusa_last_error()
    assert create([[-1], []]) == B.MEDUSA_ERR_INVALID_ARG  # an empty tree
    off = (ctypes.c_int32 * 2)(0, 1)
    arr = (ctypes.c_int32 * 1)(-1)
    assert lib.medusa_tree_create_ragged(arr, off, 0, ctypes.byref(h)) == B.MEDUSA_ERR_INVALID_ARG
    bad = (ctypes.c_int32 * 2)(1, 2)
    assert lib.medusa_tree_create_ragged(arr, bad, 1, ctypes.byref(h)) == B.MEDUSA_ERR_INVALID_ARG
    assert lib.medusa_tree_create_ragged(None, off, 1, ctypes.byref(h)) == B.MEDUSA_ERR_INVALID_ARG


def test_null_and_size_errors_before_launch(lib):
    # no tensor touches the device: every one of these fails validation first
    assert lib.medusa_heads(None, None, None, 1, 8, 8, 1, 1, None, None, None, None, None, None, None, None, None,
                            None, 0, None, None) == B.MEDUSA_ERR_INVALID_ARG
    assert b"NULL" in lib.medusa_last_error()
    fake = ctypes.c_void_p(0x1000)
    assert lib.medusa_heads(fake, fake, fake, 1, 12, 8, 1, 1, None, None, fake, fake, None, None, None, None, None,
                            fake, 1 << 30, None, None) == B.MEDUSA_ERR_INVALID_ARG  # d % 8 != 0 for bf16
    assert lib.medusa_heads(fake, fake, fake, 1, 16, 8, 1, 7, None, None, fake, fake, None, None, None, None, None,
                            fake, 1 << 30, None, None) == B.MEDUSA_ERR_UNSUPPORTED  # unknown dtype
    assert lib.medusa_heads(fake, fake, fake, 1, 16, 8, 1, 1, None, None, fake, fake, None, None, None, None, None,
                            fake, 16, None, None) == B.MEDUSA_ERR_WORKSPACE
    assert lib.tree_attention(None, None, None, None, None, None, 1, 4, 4, 64, 64, 0, 0.0, 1, None, None, None, None,
                              0, None, None) == B.MEDUSA_ERR_INVALID_ARG
    assert lib.tree_verify(0, None, 1, None, 0, None, None, 1, 8, None, 0, 0, None, 1, None, None, None, 0, None,
                           None) == B.MEDUSA_ERR_INVALID_ARG
    assert lib.kv_commit(fake, fake, fake, fake, fake, 1, fake, fake, fake, 1, 7, 2, 12, 16, 1, None,
                         None) == B.MEDUSA_ERR_INVALID_ARG  # a 24-byte row is not a multiple of 16


def test_workspace_queries_are_pure(lib):
    a = lib.medusa_heads_workspace_size(1, 4096, 128256, 4, 1)
    b = lib.medusa_heads_workspace_size(1, 4096, 128256, 4, 1)
    assert a == b and a > 0
    assert lib.medusa_heads_workspace_size(0, 4096, 128256, 4, 1) == 0


def test_paged_calls_validate_before_launch(lib):
    # every one of these fails on the host, before any device work
    fake = ctypes.c_void_p(0x1000)
    nul = None
    # NULL block table
    assert lib.tree_attention_paged(fake, fake, fake, fake, fake, nul, 4, 16, 8, fake, 1, 4, 2, 128, 0, ctypes.c_float(0),
                                    1, nul, fake, nul, fake, 1 << 20, nul, nul) == B.MEDUSA_ERR_INVALID_ARG
    assert b"NULL" in lib.medusa_last_error()
    assert lib.kv_commit_paged(fake, fake, fake, fake, nul, 4, 16, 8, fake, 3, fake, fake, fake, 1, 7, 2, 128, 1, nul,
                               nul) == B.MEDUSA_ERR_INVALID_ARG
    # bad page geometry
    assert lib.kv_commit_paged(fake, fake, fake, fake, fake, 4, 0, 8, fake, 3, fake, fake, fake, 1, 7, 2, 128, 1, nul,
                               nul) == B.MEDUSA_ERR_INVALID_ARG
    assert lib.kv_commit_paged(fake, fake, fake, fake, fake, 0, 16, 8, fake, 3, fake, fake, fake, 1, 7, 2, 128, 1,
                               nul, nul) == B.MEDUSA_ERR_INVALID_ARG
    # a K/V row that is not a multiple of 16 bytes
    assert lib.kv_commit_paged(fake, fake, fake, fake, fake, 4, 16, 8, fake, 3, fake, fake, fake, 1, 7, 2, 4, 1, nul,
                               nul) == B.MEDUSA_ERR_INVALID_ARG
    # unknown dtype
    assert lib.kv_commit_paged(fake, fake, fake, fake, fake, 4, 16, 8, fake, 3, fake, fake, fake, 1, 7, 2, 128, 9, nul,
                               nul) == B.MEDUSA_ERR_UNSUPPORTED
    # the paged workspace query mirrors the contiguous one's domain
    assert lib.tree_attention_paged_workspace_size(1, 4, 2, 96, 0, 4, 16, nul, 1) == 0
    assert lib.tree_attention_paged_workspace_size(1, 4, 2, 128, 0, 0, 16, nul, 1) == 0


def test_newer_calls_validate_before_launch(lib):
    # every failure here is found on the host, before any device work
    fake = ctypes.c_void_p(0x1000)
    other = ctypes.c_void_p(0x2000)
    nul = None
    INV, UNS, WS = B.MEDUSA_ERR_INVALID_ARG, B.MEDUSA_ERR_UNSUPPORTED, B.MEDUSA_ERR_WORKSPACE
    # kv_compact: NULL arrays, aliased prefix lengths, sizes, row alignment, dtype
    args = dict(kc=fake, vc=fake, nl=4, path=fake, mp=5, ln=fake, pl=fake, npl=other, B_=2, T=8, Hkv=2, D=128,
                S=64, dt=1)

    def compact(**kw):
        a = {**args, **kw}
        return lib.kv_compact(a["kc"], a["vc"], a["nl"], a["path"], a["mp"], a["ln"], a["pl"], a["npl"], a["B_"],
                              a["T"], a["Hkv"], a["D"], a["S"], a["dt"], nul, nul)
    assert compact(kc=nul) == INV
    assert compact(npl=fake) == INV and b"alias" in lib.medusa_last_error()
    assert compact(nl=0) == INV and compact(nl=70000) == INV
    assert compact(mp=129) == INV and compact(T=129) == INV
    assert compact(D=4) == INV                                  # 8-byte rows
    assert compact(dt=7) == UNS
    assert compact(kc=ctypes.c_void_p(0x1008)) == INV           # the pointer array itself misaligned
    # sharded heads
    part = fake
    assert lib.medusa_heads_shard(fake, fake, fake, 1, 64, 100, 0, 2, 1, nul, fake, 1 << 30, nul, nul) == INV
    assert lib.medusa_heads_shard(fake, fake, fake, 1, 64, 100, -1, 2, 1, part, fake, 1 << 30, nul, nul) == INV
    assert lib.medusa_heads_shard(fake, fake, fake, 1, 60, 100, 0, 2, 1, part, fake, 1 << 30, nul, nul) == INV
    assert lib.medusa_heads_shard(fake, fake, fake, 1, 64, 100, 0, 17, 1, part, fake, 1 << 30, nul, nul) == INV
    assert lib.medusa_heads_shard(fake, fake, fake, 1, 64, 100, 0, 2, 1, part, fake, 16, nul, nul) == WS
    assert lib.medusa_heads_shard(fake, fake, fake, 1, 64, 100, 0, 2, 5, part, fake, 1 << 30, nul, nul) == UNS
    assert lib.medusa_heads_shard_workspace_size(1, 64, 0, 2, 1) == 0
    assert lib.medusa_heads_shard_workspace_size(1, 64, 100, 2, 1) >= lib.medusa_heads_workspace_size(1, 64, 100, 2, 1)
    assert lib.medusa_heads_merge(nul, 2, 1, 2, 100, nul, nul, fake, fake, nul, nul, nul, nul) == INV
    assert lib.medusa_heads_merge(fake, 0, 1, 2, 100, nul, nul, fake, fake, nul, nul, nul, nul) == INV
    assert lib.medusa_heads_merge(ctypes.c_void_p(0x1004), 2, 1, 2, 100, nul, nul, fake, fake, nul, nul, nul,
                                  nul) == INV
    # tree K/V in the cache, logits verify, two-launch greedy verify: NULLs and a missing tree
    assert lib.tree_attention_incache(nul, fake, fake, fake, 1, 4, 2, 128, 256, 0, ctypes.c_float(0), 1, nul, fake,
                                      nul, fake, 1 << 20, nul, nul) == INV
    assert lib.tree_attention_incache(fake, fake, fake, fake, 1, 4, 2, 128, 256, 0, ctypes.c_float(0), 1, nul, fake,
                                      nul, fake, 1 << 20, nul, nul) == INV           # tree NULL
    assert lib.tree_verify_logits(nul, 1, ctypes.c_double(1.0), fake, 4, nul, fake, 1, 100, nul, 0, 0, fake, 4,
                                  fake, fake, fake, 1 << 20, nul, nul) == INV
    assert lib.tree_verify_logits(fake, 5, ctypes.c_double(1.0), fake, 4, nul, fake, 1, 100, nul, 0, 0, fake, 4,
                                  fake, fake, fake, 1 << 20, nul, nul) == INV        # tree NULL comes first
    assert lib.tree_verify_greedy_rows(nul, 1, 1, 100, nul, fake, 1 << 20, nul) == INV
    assert lib.tree_verify_greedy_rows(fake, 5, 1, 100, nul, fake, 1 << 20, nul) == UNS
    assert lib.tree_verify_greedy_walk(nul, 1, 100, nul, fake, 4, fake, fake, fake, 1 << 20, nul) == INV
    assert lib.tree_verify_greedy_walk(fake, 1, 100, nul, fake, 4, fake, fake, fake, 1 << 20, nul) == INV
    # the launch shape refuses negative values and is restored by (0, 0)
    assert lib.medusa_set_launch_shape(-1, 0) == INV
    assert lib.medusa_set_launch_shape(100, 1) == 0 and lib.medusa_set_launch_shape(0, 0) == 0
    # the walk with its commit: NULL cache arguments, then a missing tree
    wc = lib.tree_verify_greedy_walk_commit
    wc.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int,
                   ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p,
                   ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int,
                   ctypes.c_int, ctypes.c_int, ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                   ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p]
    assert wc(fake, 1, 100, nul, fake, 4, fake, fake, fake, 1 << 20, nul, fake, fake, fake, fake, fake, 8, 128, 256,
              nul, 0, 0, 0, 1, nul, nul) == INV
    assert wc(fake, 1, 100, nul, fake, 4, fake, fake, fake, 1 << 20, fake, fake, fake, fake, fake, fake, 8, 128, 256,
              nul, 0, 0, 0, 1, nul, nul) == INV                                       # tree NULL
    assert lib.tree_attention_incache_workspace_size(1, 4, 2, 96, 256, 0, nul, 1) == 0


def test_header_is_plain_c(tmp_path):
    # the boundary is a C ABI: the header compiles as C11 and as C++17 with
    # every warning on, and needs no CUDA or torch header
    inc = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include")
    src = tmp_path / "use.c"
    src.write_text('#include "medusa.h"\nint f(void) { return MEDUSA_TOPK + (int)sizeof(medusa_head_partial); }\n')
    import subprocess
    subprocess.check_call(["gcc", "-std=c11", "-Wall", "-Wextra", "-Werror", "-fsyntax-only", "-I", inc, str(src)])
    cpp = tmp_path / "use.cpp"
    cpp.write_text(src.read_text())
    subprocess.check_call(["g++", "-std=c++17", "-Wall", "-Wextra", "-Werror", "-fsyntax-only", "-I", inc, str(cpp)])
