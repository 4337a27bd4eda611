"""One whole decode step (heads -> tree -> attention -> verify -> commit) on
the GPU against the same step run by the oracle."""
import numpy as np
import pytest
import torch

import oracle
from helpers import assert_float_parity, check_topk, float_tol
from medusa_tree_speculative_heads_b200 import inputs as I
from medusa_tree_speculative_heads_b200.api import MedusaStep

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name,attention_sms", [("tiny", 0), ("llama8b", 0), ("llama8b", 8)])
def test_whole_step_matches_oracle(name, attention_sms):
    # attention_sms = 8: the heads kernel on all but 8 SMs, tree attention
    # (no key splits) on those 8 during the weight stream
    w = I.WORKLOADS[name]
    parents = I.workload_tree(w)
    T = len(parents)
    hin = I.head_inputs(w)
    ain = I.attention_inputs(w, T)
    # ---- oracle step ----
    ref = oracle.heads(hin["h"], hin["W_res"], hin["W_head"], want_hk=False)
    otop = np.stack([np.stack([oracle.topk(ref["logits"][b, k], 8) for k in range(w.K)]) for b in range(w.B)])
    otok, _ = oracle.tree_fill(parents, hin["root_token"], otop,
                               np.take_along_axis(ref["probs"], otop, axis=-1))
    logits = I.boosted_target_logits(w, parents, torch.from_numpy(otok))
    o_att, _ = oracle.tree_attention(ain["q"], ain["k_tree"], ain["v_tree"], ain["k_cache"], ain["v_cache"],
                                     ain["prefix_len"], parents)
    maxd = int(max(oracle.tree_shape(parents)[0]))
    opath, olen, obonus = oracle.verify_greedy(logits, otok, parents, maxd)
    okc, ovc, onpl, ost = oracle.kv_commit(ain["k_cache"], ain["v_cache"], ain["k_tree"], ain["v_tree"], opath, olen,
                                           ain["prefix_len"])
    # ---- GPU step ----
    d = {k: v.cuda() for k, v in {**hin, **ain}.items()}
    st = MedusaStep(B=w.B, d=w.d, V=w.V, K=w.K, Hq=w.Hq, Hkv=w.Hkv, D=w.D, S_max=w.S_max, parents=parents,
                    dtype=w.torch_dtype, max_prefix=w.max_prefix, attention_sms=attention_sms)
    new_pl = torch.empty_like(d["prefix_len"])
    st.run(h=d["h"], W_res=d["W_res"], W_head=d["W_head"], root_token=d["root_token"], q=d["q"], k_tree=d["k_tree"],
           v_tree=d["v_tree"], k_cache=d["k_cache"], v_cache=d["v_cache"], prefix_len=d["prefix_len"],
           new_prefix_len=new_pl, target=logits.cuda())
    torch.cuda.synchronize()
    assert int(st.status.item()) == 0
    ti = st.topk_idx.cpu().numpy()
    chain = dict(path=st.accept_path.cpu().numpy(), len=st.accept_len.cpu().numpy(), bonus=st.bonus.cpu().numpy(),
                 npl=new_pl.cpu().numpy(), kc=d["k_cache"].cpu(), vc=d["v_cache"].cpu())
    mism = sum(check_topk(ti[b, k], ref["logits"][b, k], float_tol(w.torch_dtype)) for b in range(w.B)
               for k in range(w.K))
    assert_float_parity(st.attn_out.float().cpu().reshape(-1, w.D), o_att, w.torch_dtype, "attention")
    # verify and commit on identical inputs: the oracle's node tokens
    kc2, vc2 = ain["k_cache"].cuda(), ain["v_cache"].cuda()
    pl2 = torch.empty_like(d["prefix_len"])
    st.verify(logits.cuda(), node_tokens=torch.from_numpy(otok).cuda())
    st.commit(kc2, vc2, d["k_tree"], d["v_tree"], d["prefix_len"], pl2)
    torch.cuda.synchronize()
    assert np.array_equal(st.accept_path.cpu().numpy(), opath)
    assert np.array_equal(st.accept_len.cpu().numpy(), olen)
    assert np.array_equal(st.bonus.cpu().numpy(), obonus)
    assert np.array_equal(pl2.cpu().numpy(), onpl)
    assert torch.equal(kc2.cpu(), okc) and torch.equal(vc2.cpu(), ovc)
    # the GPU's own chain, when every top-s decision matched the oracle's
    if mism == 0:
        assert np.array_equal(st.node_tokens.cpu().numpy(), otok)
        assert np.array_equal(chain["path"], opath)
        assert np.array_equal(chain["len"], olen)
        assert np.array_equal(chain["bonus"], obonus)
        assert np.array_equal(chain["npl"], onpl)
        assert torch.equal(chain["kc"], okc) and torch.equal(chain["vc"], ovc)


@pytest.mark.parametrize("name", ["llama8b_small", "stoch_small", "stoch_logits_small", "llama8b_reserved"])
def test_graph_replay_equals_eager_step(name):
    # the step captured in a CUDA graph and replayed gives the eager step's
    # results bit for bit (the kernels are deterministic)
    if name.startswith("llama8b"):
        w = I.scaled(I.WORKLOADS["llama8b"], B=2, d=512, V=3001, prefix=300)
    else:
        w = I.scaled(I.WORKLOADS["stoch_b64"], B=3, V=900)
    parents = I.workload_tree(w)
    T = len(parents)
    from medusa_tree_speculative_heads_b200 import binding as Bnd
    mode = Bnd.STOCHASTIC if w.stochastic else Bnd.GREEDY
    tau = I.STOCH_TEMPERATURE if name == "stoch_logits_small" else 0.0
    # "reserved": the heads kernel leaves 8 SMs to tree attention (the launch
    # shape is recorded into the graph with the kernels)
    step = MedusaStep(B=w.B, d=w.d, V=w.V, K=w.K, Hq=w.Hq, Hkv=w.Hkv, D=w.D, S_max=w.S_max, parents=parents,
                      dtype=w.torch_dtype, device="cuda", mode=mode, q_rows=T, temperature=tau,
                      attention_sms=8 if name.endswith("reserved") else 0)
    hin = {k: v.cuda() for k, v in I.head_inputs(w).items()}
    ain = {k: v.cuda() for k, v in I.attention_inputs(w, T).items()}
    if w.stochastic:
        sd = {k: v.cuda() for k, v in I.stochastic_inputs(w, parents).items()}
        target, q_draft, tok = sd["p"], sd["q"], sd["node_tokens"]
        if tau > 0:   # the step reads the target's bf16 logits
            target = sd["logits"].bfloat16()
    else:
        target = torch.randn((w.B, T, w.V), generator=torch.Generator().manual_seed(2)).to(w.torch_dtype).cuda()
        q_draft = tok = None
    new_pl = torch.empty_like(ain["prefix_len"])
    k0, v0 = ain["k_cache"].clone(), ain["v_cache"].clone()
    kw = dict(h=hin["h"], W_res=hin["W_res"], W_head=hin["W_head"], root_token=hin["root_token"], q=ain["q"],
              k_tree=ain["k_tree"], v_tree=ain["v_tree"], k_cache=ain["k_cache"], v_cache=ain["v_cache"],
              prefix_len=ain["prefix_len"], new_prefix_len=new_pl, target=target, q_draft=q_draft,
              node_tokens=tok, step=5)
    step.run(**kw)
    torch.cuda.synchronize()
    eager = [x.clone() for x in (step.node_tokens, step.attn_out, step.accept_path, step.accept_len, step.bonus,
                                 new_pl, ain["k_cache"])]
    ain["k_cache"].copy_(k0)
    ain["v_cache"].copy_(v0)
    for x in (step.node_tokens, step.attn_out, step.accept_path, step.accept_len, step.bonus, new_pl):
        x.zero_()
    g = step.capture(**kw)
    torch.cuda.synchronize()
    ain["k_cache"].copy_(k0)  # capture does not run the kernels; replay twice from the same state
    ain["v_cache"].copy_(v0)
    g.replay()
    g.replay()
    torch.cuda.synchronize()
    assert int(step.status.item()) == 0
    replay = (step.node_tokens, step.attn_out, step.accept_path, step.accept_len, step.bonus, new_pl, ain["k_cache"])
    for a, b in zip(eager, replay):
        assert torch.equal(a, b)
    if tau > 0:
        maxd = int(max(oracle.tree_shape(parents)[0]))
        path, ln, bonus, _ = oracle.verify_stochastic_logits(target, tau, q_draft, tok, parents, 0, 5, maxd)
        assert np.array_equal(step.accept_path.cpu().numpy(), path)
        assert np.array_equal(step.accept_len.cpu().numpy(), ln) and np.array_equal(step.bonus.cpu().numpy(), bonus)


@pytest.mark.parametrize("name", ["llama8b_small", "stoch_small"])
def test_overlapped_step_equals_the_calls_in_order(name):
    # run() with attention (and greedy verification's row scan) on side
    # streams gives the in-order step's results bit for bit
    if name == "llama8b_small":
        w = I.scaled(I.WORKLOADS["llama8b"], B=2, d=512, V=3001, prefix=300)
    else:
        w = I.scaled(I.WORKLOADS["stoch_b64"], B=3, V=900)
    parents = I.workload_tree(w)
    T = len(parents)
    from medusa_tree_speculative_heads_b200 import binding as Bnd
    mode = Bnd.STOCHASTIC if w.stochastic else Bnd.GREEDY
    hin = {k: v.cuda() for k, v in I.head_inputs(w).items()}
    ain = {k: v.cuda() for k, v in I.attention_inputs(w, T).items()}
    if w.stochastic:
        sd = {k: v.cuda() for k, v in I.stochastic_inputs(w, parents).items()}
        target, q_draft, tok = sd["p"], sd["q"], sd["node_tokens"]
    else:
        target = torch.randn((w.B, T, w.V), generator=torch.Generator().manual_seed(2)).to(w.torch_dtype).cuda()
        q_draft = tok = None
    results = []
    for overlap in (False, True):
        step = MedusaStep(B=w.B, d=w.d, V=w.V, K=w.K, Hq=w.Hq, Hkv=w.Hkv, D=w.D, S_max=w.S_max, parents=parents,
                          dtype=w.torch_dtype, device="cuda", mode=mode, q_rows=T, overlap=overlap)
        kc, vc = ain["k_cache"].clone(), ain["v_cache"].clone()
        new_pl = torch.empty_like(ain["prefix_len"])
        step.run(h=hin["h"], W_res=hin["W_res"], W_head=hin["W_head"], root_token=hin["root_token"], q=ain["q"],
                 k_tree=ain["k_tree"], v_tree=ain["v_tree"], k_cache=kc, v_cache=vc, prefix_len=ain["prefix_len"],
                 new_prefix_len=new_pl, target=target, q_draft=q_draft, node_tokens=tok, step=3)
        torch.cuda.synchronize()
        assert int(step.status.item()) == 0
        results.append([x.clone() for x in (step.node_tokens, step.attn_out, step.accept_path, step.accept_len,
                                            step.bonus, new_pl, kc, vc)])
    for a, b in zip(*results):
        assert torch.equal(a, b)
