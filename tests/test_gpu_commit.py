"""kv_commit on the GPU against the oracle: bit-exact cache contents."""
import numpy as np
import pytest
import torch

import oracle
from medusa_tree_speculative_heads_b200 import api
from medusa_tree_speculative_heads_b200 import binding as B

pytestmark = pytest.mark.gpu


def make(Bsz, Hkv, S_max, D, T, dtype, seed=0):
    g = torch.Generator().manual_seed(seed)
    kc = torch.randn((Bsz, Hkv, S_max, D), generator=g).to(dtype)
    vc = torch.randn((Bsz, Hkv, S_max, D), generator=g).to(dtype)
    kt = torch.randn((Bsz, T, Hkv, D), generator=g).to(dtype)
    vt = torch.randn((Bsz, T, Hkv, D), generator=g).to(dtype)
    return kc, vc, kt, vt


@pytest.mark.parametrize("dtype,D", [(torch.bfloat16, 128), (torch.float32, 64), (torch.bfloat16, 8)])
def test_commit_parity(dtype, D):
    Bsz, Hkv, S_max, T = 5, 3, 40, 9
    kc, vc, kt, vt = make(Bsz, Hkv, S_max, D, T, dtype)
    path = torch.tensor([[0, 3, 7, -1], [0, -1, -1, -1], [0, 1, 2, 8], [0, 4, -1, -1], [0, 2, 5, 6]],
                        dtype=torch.int32)
    ln = torch.tensor([3, 1, 4, 2, 4], dtype=torch.int32)
    pl = torch.tensor([10, 0, 36, 38, 37], dtype=torch.int32)   # last two overflow
    k2, v2, npl, st = oracle.kv_commit(kc, vc, kt, vt, path, ln, pl)
    d = {n: t.cuda() for n, t in dict(kc=kc, vc=vc, kt=kt, vt=vt, path=path, ln=ln, pl=pl).items()}
    out = api.kv_commit(d["kc"], d["vc"], d["kt"], d["vt"], d["path"], d["ln"], d["pl"])
    torch.cuda.synchronize()
    assert torch.equal(d["kc"].cpu(), k2) and torch.equal(d["vc"].cpu(), v2)
    assert np.array_equal(out["new_prefix_len"].cpu().numpy(), npl)
    assert int(out["status"].item()) == B.STATUS_CACHE_OVERFLOW


def test_commit_in_place_prefix_and_bad_ids():
    Bsz, Hkv, S_max, D, T = 3, 2, 16, 64, 5
    kc, vc, kt, vt = make(Bsz, Hkv, S_max, D, T, torch.bfloat16, 1)
    path = torch.tensor([[0, 1, 2], [0, 9, -1], [0, 4, -1]], dtype=torch.int32)   # node 9 >= T
    ln = torch.tensor([3, 2, 2], dtype=torch.int32)
    pl = torch.tensor([0, 3, 14], dtype=torch.int32)
    d = {n: t.cuda() for n, t in dict(kc=kc, vc=vc, kt=kt, vt=vt, path=path, ln=ln, pl=pl).items()}
    before = d["kc"].clone()
    out = api.kv_commit(d["kc"], d["vc"], d["kt"], d["vt"], d["path"], d["ln"], d["pl"], new_prefix_len=d["pl"])
    torch.cuda.synchronize()
    assert d["pl"].tolist() == [3, 3, 16]
    assert int(out["status"].item()) == B.STATUS_BAD_TOKEN
    assert torch.equal(d["kc"][1], before[1])                  # the bad sequence is untouched
    assert torch.equal(d["kc"][0, :, 0:3].cpu(), kt[0, [0, 1, 2]].transpose(0, 1))
    assert torch.equal(d["kc"][2, :, 14:16].cpu(), kt[2, [0, 4]].transpose(0, 1))
    assert torch.equal(d["kc"][0, :, 3:], before[0, :, 3:])   # slots past the commit keep their contents
