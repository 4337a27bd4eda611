"""medusa_heads_noalloc: the heads entry point for callers that cannot
allocate device memory.

Such callers exist: a plug-in running inside a framework that owns every byte
of GPU memory and offers it no allocator, or a decode loop that must never
call cudaMalloc/cudaFree because those calls synchronise the device.  The
variant keeps its scratch in a fixed array inside the library.  Here it must
give the same results as medusa_heads with a caller-supplied workspace, on
two calls in a row (the second runs on whatever the first left behind in the
shared array), and refuse sizes whose scratch would not fit.

This file is named to be collected last, so a run that stops at the first
failure has run every other test before it.
"""
import pytest
import torch

from medusa_tree_speculative_heads_b200 import binding as B
from medusa_tree_speculative_heads_b200 import inputs as I
from medusa_tree_speculative_heads_b200.binding import MedusaError, Tree

pytestmark = pytest.mark.gpu


def _outs(w, T):
    dev = "cuda"
    return {
        "topk_idx": torch.full((w.B, w.K, B.TOPK), -7, dtype=torch.int32, device=dev),
        "topk_prob": torch.full((w.B, w.K, B.TOPK), -7.0, device=dev),
        "node_tokens": torch.full((w.B, T), -7, dtype=torch.int32, device=dev),
        "node_q": torch.full((w.B, T), -7.0, device=dev),
        "h_res": torch.empty((w.B, w.K, w.d), dtype=w.torch_dtype, device=dev),
        "logits": torch.empty((w.B, w.K, w.V), device=dev),
        "probs": torch.empty((w.B, w.K, w.V), device=dev),
        "status": torch.zeros(1, dtype=torch.int32, device=dev),
    }


def _call(fn_noalloc, w, inp, tree, o):
    args = (inp["h"], inp["W_res"], inp["W_head"], w.B, w.d, w.V, w.K, B.dtype_code(w.torch_dtype), tree,
            inp["root_token"], o["topk_idx"], o["topk_prob"], o["node_tokens"], o["node_q"], o["h_res"], o["logits"],
            o["probs"])
    if fn_noalloc:
        B.medusa_heads_noalloc(*args, o["status"])
    else:
        nb = B.medusa_heads_workspace_size(w.B, w.d, w.V, w.K, B.dtype_code(w.torch_dtype))
        ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
        B.medusa_heads(*args, ws, nb, o["status"])


def _same(a, b):
    # the same kernels on the same inputs with the same workspace layout: every
    # output must be bit-identical (a value perturbed by stale scratch would
    # still pass a float tolerance)
    for k in ("topk_idx", "topk_prob", "node_tokens", "node_q", "logits", "probs", "h_res", "status"):
        assert torch.equal(a[k], b[k]), k


@pytest.mark.parametrize("name,kw,tree", [
    ("tiny", {}, (2, 2)),
    ("llama8b", dict(V=32000), (4, 4, 2, 2)),
    ("llama8b", dict(B=3, d=1024, V=5000, K=2), (4, 2)),
])
def test_noalloc_matches_workspace_entry_point_twice(name, kw, tree):
    w0 = I.scaled(I.WORKLOADS[name], **kw)
    parents = I.product_tree_parents(tree)
    t = Tree(parents)
    for call in range(2):
        w = I.scaled(w0, seed=w0.seed + 100 * call)   # different inputs on the second call
        inp = {k: v.cuda() for k, v in I.head_inputs(w).items()}
        mine, ref = _outs(w, t.T), _outs(w, t.T)
        _call(True, w, inp, t, mine)
        _call(False, w, inp, t, ref)
        torch.cuda.synchronize()
        _same(mine, ref)
        assert int(mine["status"].item()) == 0


def test_noalloc_refuses_sizes_beyond_its_scratch():
    # 64 sequences x 4 heads x 128256 logits need far more than the fixed
    # array; the call must refuse before touching any pointer (NULLs here)
    with pytest.raises(MedusaError) as e:
        B.medusa_heads_noalloc(None, None, None, 64, 4096, 128256, 4, B.BF16, None, None, None, None, None, None,
                               None, None, None, None)
    assert e.value.code == B.MEDUSA_ERR_UNSUPPORTED
    assert "scratch" in str(e.value)
