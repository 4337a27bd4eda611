"""Shared checks for the GPU parity tests (tolerances from the stated
bounds: bf16 inputs with fp32 accumulation max-abs <= 1e-2 and relative L2
<= 5e-3; fp32 max-abs <= 1e-4; discrete outputs bit-exact)."""
import numpy as np
import torch

BF16_MAX_ABS = 1e-2
BF16_REL_L2 = 5e-3
F32_MAX_ABS = 1e-4


def assert_float_parity(gpu, ref, dtype, what=""):
    g = np.asarray(gpu.detach().float().cpu().numpy() if isinstance(gpu, torch.Tensor) else gpu, dtype=np.float64)
    r = np.asarray(ref, dtype=np.float64)
    assert g.shape == r.shape, (what, g.shape, r.shape)
    err = np.abs(g - r)
    assert np.isfinite(g).all(), f"{what}: non-finite GPU values"
    max_abs = float(err.max()) if err.size else 0.0
    if dtype == torch.float32:
        assert max_abs <= F32_MAX_ABS, f"{what}: max abs err {max_abs:.3g} > {F32_MAX_ABS}"
    else:
        rel = float(np.linalg.norm(g - r) / max(np.linalg.norm(r), 1e-30))
        assert max_abs <= BF16_MAX_ABS, f"{what}: max abs err {max_abs:.3g} > {BF16_MAX_ABS}"
        assert rel <= BF16_REL_L2, f"{what}: rel L2 err {rel:.3g} > {BF16_REL_L2}"
    return max_abs


def float_tol(dtype):
    return F32_MAX_ABS if dtype == torch.float32 else BF16_MAX_ABS


def check_topk(gpu_idx, ref_logits, eps):
    """The GPU's top list against the oracle's fp64 logits: entries must be
    distinct and, at every rank, have an oracle logit within eps of the
    oracle's value at that rank (so where the oracle's order is separated by
    more than the float tolerance, the ids are equal).  Returns the number of
    ranks whose id differs from the oracle's own stable sort."""
    import oracle
    ref_logits = np.asarray(ref_logits, dtype=np.float64)
    s = len(gpu_idx)
    want = oracle.topk(ref_logits, s)
    g = [int(x) for x in gpu_idx]
    assert len(set(g)) == len(g), f"duplicate ids {g}"
    mismatches = 0
    for r in range(s):
        if g[r] != int(want[r]):
            mismatches += 1
            assert 0 <= g[r] < len(ref_logits)
            assert abs(ref_logits[g[r]] - ref_logits[want[r]]) <= eps, (r, g[r], int(want[r]))
    return mismatches


def assert_top_lists_exact(out):
    """Every (sequence, head) top list equals the oracle's top-s run on the
    kernel's own fp32 logits (missing entries -1 when V < 8)."""
    import oracle
    lg = out["logits"].double().cpu().numpy()
    ti = out["topk_idx"].cpu().numpy()
    B, K, S = ti.shape
    for b in range(B):
        for k in range(K):
            assert np.array_equal(ti[b, k], oracle.topk(lg[b, k], S)), (b, k)


def to_dev(d, device="cuda"):
    return {k: (v.to(device) if isinstance(v, torch.Tensor) else v) for k, v in d.items()}
