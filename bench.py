#!/usr/bin/env python
"""Benchmark of one Medusa speculative decode step on B200.

A step is the whole hot path over one batch: medusa_heads (residual block,
LM-head projection, softmax statistics, top-8, tree fill) -> tree_attention
(one layer) -> tree_verify (greedy) -> kv_commit, on the 8B-shaped workload
(B=1, d=4096, V=128256, K=4 heads, top-s (4,4,2,2) = 117 nodes, 32/8 heads,
head_dim 128, prefix 2048), bf16 with fp32 accumulation, synthetic seeded
inputs and random weights.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl mine|reference]

Prints one JSON line (rank 0).  Multi-GPU runs (torchrun) are independent
replicas, one per GPU: the step has no cross-sequence exchange.
"""
from __future__ import annotations

import argparse
import datetime
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

METRIC = "Medusa verify steps/s (8B shape, 117-node tree); tree-attn HBM GB/s vs peak"
UNIT = "steps/s"
W_E2E = 10   # untimed end-to-end steps first (the first copies from fresh pinned buffers run slower)
WORKLOAD = "llama8b"
# DRAM bytes (read + write) per launch of the heads kernel, from an ncu capture
# of the same kernel at V=32000 (1184.480 MB read + 3.802 MB written against
# 1182.802 MB algorithmic), scaled to the workload's algorithmic bytes; only for
# the workload whose launch configuration (B=1, d=4096, K=4) was captured.
HEADS_DRAM_BYTES = {"llama8b": 4336918528 * (1184480000 + 3802112) / 1182801920}
OVERRIDDEN = set()   # workloads whose sizes --override replaced (no captured traffic applies)


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# ----------------------------------------------------------------------------
# clocks during the timed region
# ----------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) >= 9:
                rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[j] for r in rows for j in range(4) if r[5 + j].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


# ----------------------------------------------------------------------------
# oracle timing (the CPU baseline / reference arm)
# ----------------------------------------------------------------------------

class OracleSample:
    """A bounded sample of the step, run by the fp64 oracle on the host: the
    residual block of every head, the LM-head rows of a `fraction` slice of
    the vocabulary, the attention of a `fraction` of the query rows, greedy
    verification over the full tree and the commit.  Inputs are drawn once
    (not timed); run() returns (seconds, fraction of a full step's work).
    Workloads with a tree per sequence run the tree calls sequence by
    sequence; a paged cache is read through its block table (the oracle's
    page gather) and committed through it."""

    def __init__(self, w, fraction: float, seed: int = 0):
        import numpy as np

        from medusa_tree_speculative_heads_b200 import inputs as I
        self.w = w
        self.parents = I.workload_tree(w)
        self.trees = I.sequence_trees(w)
        T = self.T = max(len(t) for t in self.trees)
        self.Vs = max(8, int(round(w.V * fraction)))
        self.ws = I.scaled(w, V=self.Vs)
        self.hin = I.head_inputs(self.ws)
        self.ain = I.attention_inputs(w, T)
        self.pc = (I.paged_cache(w, w.page_size, self.ain["prefix_len"], room=T, capacity=w.max_prefix + T)
                   if w.page_size else None)
        if w.tree_in_cache:   # the tree's K/V after each prefix, as the GPU path holds them
            for b, tr in enumerate(self.trees):
                S = int(self.ain["prefix_len"][b])
                self.ain["k_cache"][b, :, S:S + len(tr)] = self.ain["k_tree"][b, :len(tr)].transpose(0, 1)
                self.ain["v_cache"][b, :, S:S + len(tr)] = self.ain["v_tree"][b, :len(tr)].transpose(0, 1)
        n_rows = w.B * T * w.Hq
        nr = max(1, int(round(n_rows * fraction)))
        g = np.random.default_rng(seed)
        rid = g.choice(n_rows, size=nr, replace=False)
        rows = np.stack([rid // (T * w.Hq), (rid // w.Hq) % T, rid % w.Hq], axis=1)
        # rows of nodes past a sequence's own tree are not part of the step
        self.rows = rows[[r[1] < len(self.trees[r[0]]) for r in rows]]
        # the residual block and verification/commit run whole; the LM head
        # and attention (all but ~2% of the work) are sampled at `fraction`
        lm = w.K * w.V * w.d
        att = n_rows * (w.prefix + 5) * w.D * 2
        res = w.K * w.d * w.d
        self.frac = (res + lm * self.Vs / w.V + att * nr / n_rows) / (res + lm + att)
        self.logits = None
        # stochastic workloads verify the harness's drafted tokens against its
        # target (probabilities, or logits at the temperature), whole
        self.sd = I.stochastic_inputs(w, self.parents) if w.stochastic else None

    def run(self):
        import numpy as np

        import oracle
        from medusa_tree_speculative_heads_b200 import inputs as I
        w, hin, ain, trees, T = self.w, self.hin, self.ain, self.trees, self.T
        ragged = w.ragged_trees is not None
        t0 = time.perf_counter()
        ref = oracle.heads(hin["h"], hin["W_res"], hin["W_head"], want_hk=False)
        otop = np.stack([np.stack([oracle.topk(ref["logits"][b, k], 8) for k in range(w.K)]) for b in range(w.B)])
        otp = np.take_along_axis(ref["probs"], otop, axis=-1)
        if ragged:
            otok = np.full((w.B, T), -1, np.int32)
            for b in range(w.B):
                tb, _ = oracle.tree_fill(trees[b], hin["root_token"][b:b + 1], otop[b:b + 1], otp[b:b + 1])
                otok[b, :len(trees[b])] = tb[0]
        else:
            otok, _ = oracle.tree_fill(self.parents, hin["root_token"], otop, otp)
        t1 = time.perf_counter()
        if self.logits is None and self.sd is None:   # the target model's logits: input generation, not timed
            self.logits = I.boosted_target_logits(self.ws, self.parents, torch.from_numpy(otok))
        t2 = time.perf_counter()
        kc, vc = ain["k_cache"], ain["v_cache"]
        if self.pc is not None:   # the prefix read through the block table
            kc = oracle.gather_pages(self.pc["k_pages"], self.pc["block_table"], ain["prefix_len"], w.S_max)
            vc = oracle.gather_pages(self.pc["v_pages"], self.pc["block_table"], ain["prefix_len"], w.S_max)
        if ragged:
            for b in range(w.B):
                rb = self.rows[self.rows[:, 0] == b].copy()
                if len(rb) == 0:
                    continue
                rb[:, 0] = 0
                Tb = len(trees[b])
                oracle.tree_attention(ain["q"][b:b + 1, :Tb], ain["k_tree"][b:b + 1, :Tb], ain["v_tree"][b:b + 1, :Tb],
                                      kc[b:b + 1], vc[b:b + 1], ain["prefix_len"][b:b + 1], trees[b], rows=rb)
        elif w.tree_in_cache:
            oracle.tree_attention_incache(ain["q"], kc, vc, ain["prefix_len"], self.parents, rows=self.rows)
        else:
            oracle.tree_attention(ain["q"], ain["k_tree"], ain["v_tree"], kc, vc, ain["prefix_len"], self.parents,
                                  rows=self.rows)
        maxd = max(int(max(oracle.tree_shape(t)[0])) for t in (trees if ragged else [self.parents]))
        if ragged:
            path = np.full((w.B, maxd), -1, np.int32)
            ln = np.zeros(w.B, np.int32)
            for b in range(w.B):
                Tb = len(trees[b])
                pb, lb, _ = oracle.verify_greedy(self.logits[b:b + 1, :Tb], otok[b:b + 1, :Tb], trees[b], maxd)
                path[b], ln[b] = pb[0], lb[0]
        elif self.sd is not None:
            sd = self.sd
            if w.temperature > 0:
                path, ln, _, _ = oracle.verify_stochastic_logits(sd["logits"].bfloat16(), w.temperature, sd["q"],
                                                                 sd["node_tokens"], self.parents, 0, 0, maxd)
            else:
                path, ln, _, _ = oracle.verify_stochastic(sd["p"], sd["q"], sd["node_tokens"], self.parents, 0, 0,
                                                          maxd)
        else:
            path, ln, _ = oracle.verify_greedy(self.logits, otok, self.parents, maxd)
        if self.pc is not None:
            oracle.kv_commit_paged(self.pc["k_pages"], self.pc["v_pages"], ain["k_tree"], ain["v_tree"],
                                   self.pc["block_table"], path, ln, ain["prefix_len"])
        elif w.tree_in_cache:
            oracle.kv_compact([ain["k_cache"]] * w.layers, [ain["v_cache"]] * w.layers, path, ln, ain["prefix_len"],
                              T)
        else:
            oracle.kv_commit(ain["k_cache"], ain["v_cache"], ain["k_tree"], ain["v_tree"], path, ln,
                             ain["prefix_len"])
        t3 = time.perf_counter()
        return (t1 - t0) + (t3 - t2), self.frac


def time_oracle(w, fraction: float, budget_s: float, min_steps: float, omp: bool):
    """Time the oracle (serial or OpenMP build) on whole steps of workload w
    (fraction 1) or a sampled slice; returns (steps/s, seconds, steps' worth
    of work, threads used)."""
    import oracle
    oracle.build()
    oracle.use_openmp(omp)
    try:
        sample = OracleSample(w, fraction)
        tt, ff = 0.0, 0.0
        while tt < budget_s and ff < min_steps:
            t1, f1 = sample.run()
            tt += t1
            ff += f1
        return ff / tt, tt, ff, oracle.threads()
    finally:
        oracle.use_openmp(False)


def run_reference(args, rank, world):
    """The reference arm: the fp64 oracle (its OpenMP build, every host core)
    runs whole steps of the same workload -- W untimed, then K timed -- and
    the line reports what was timed: K whole steps."""
    from medusa_tree_speculative_heads_b200 import inputs as I
    if rank != 0:
        return
    w = I.WORKLOADS[args.workload]
    import oracle
    oracle.build()
    oracle.use_openmp(True)
    sample = OracleSample(w, 1.0, seed=1)
    for _ in range(args.warmup):
        sample.run()
    tot_t = 0.0
    for _ in range(args.steps):
        t, f = sample.run()
        assert f == 1.0
        tot_t += t
    cores = oracle.threads()
    oracle.use_openmp(False)
    value = args.steps / tot_t
    desc = (f"{args.steps} whole steps of the workload (after {args.warmup} untimed), timed one by one: the fp64 "
            f"oracle's OpenMP build on {cores} host threads; the target logits are inputs, drawn outside the timing")
    out = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000.0 * tot_t / args.steps,
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
           "config": config_dict(w, world),
           "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": desc},
           "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


# ----------------------------------------------------------------------------
# the CUDA path
# ----------------------------------------------------------------------------

def max_over_ranks(x: float, world: int, device) -> float:
    """The slowest rank's value (timings are max-reduced across ranks)."""
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(world: int, steps: int, seconds: float) -> float:
    """Steps per second of the whole job: every rank ran `steps` steps of its
    own replica; the job took as long as its slowest rank."""
    return world * steps / seconds


def config_dict(w, world):
    from medusa_tree_speculative_heads_b200 import inputs as I
    Ts = [len(t) for t in I.sequence_trees(w)]
    T = max(Ts)
    if w.ragged_trees:
        tree = f"a random tree per sequence {w.ragged_trees} ({min(Ts)}..{max(Ts)} nodes, mean {sum(Ts) / len(Ts):.0f})"
    else:
        tree = f"top-s {w.topk}" if w.topk else f"random tree {w.random_tree}"
    if w.page_size:
        tree += f", KV in pages of {w.page_size} via a block table"
    if w.tree_in_cache:
        tree += (f", tree K/V appended to the cache after each prefix, commit = in-place compaction of "
                 f"{w.layers} layers' caches in one launch")
    prefix = f"prefix U[{w.prefix_range[0]}, {w.prefix_range[1]}]" if w.prefix_range else f"prefix {w.prefix}"
    if w.stochastic:
        verify = ("stochastic verify from bf16 logits at temperature " + f"{w.temperature}" if w.temperature > 0
                  else "stochastic verify from fp32 probabilities")
    else:
        verify = f"greedy verify, match prob {w.match_prob}"
    head_gb = w.K * (w.d * w.d + w.V * w.d) * (2 if w.dtype == "bf16" else 4) / 1e9
    shape = tree if w.ragged_trees else f"{tree} -> {T}-node tree"
    return {"workload": (f"{w.name}: B={w.B} d={w.d} V={w.V} K={w.K} heads, {shape}, "
                         f"{w.Hq}/{w.Hkv} heads head_dim {w.D}, {prefix}, {verify}, one attention layer"),
            "global_batch": w.B * world, "seq_len": w.max_prefix, "parallelism": f"replicas x{world}",
            "l2": f"inputs larger than L2: each step streams {head_gb:.2f} GB of head weights through the 126 MB L2"}


def launches_per_step(w):
    """Library kernels per step as MedusaStep.run issues it.  medusa_heads is
    one cooperative kernel on the bf16 tensor-core path (B <= 64), else
    residual + per-8-sequence LM and merge kernels; tree attention is one
    kernel (the tensor-core kernel merges its key splits in-cluster; the
    mma.sync path adds a combine kernel); greedy verification is the row scan
    plus the walk, which also commits unless the commit is the all-layer
    compaction; stochastic verification is one kernel, then the commit."""
    if w.dtype == "bf16" and w.B <= 64 and w.d % 8 == 0:
        heads = 1
    elif w.B == 1:
        heads = 1
    else:
        heads = 1 + 2 * ((w.B + 7) // 8)
    G = w.Hq // w.Hkv
    tc = w.dtype == "bf16" and w.D in (64, 128) and G <= 16 and (G & (G - 1)) == 0 and \
        (w.page_size == 0 or w.page_size % 64 == 0 or w.page_size in (8, 16, 32))
    attn = 1 if (w.dtype != "bf16" or tc) else 2
    if w.stochastic:
        tail = 2
    else:
        tail = 3 if w.tree_in_cache else 2
    return heads + attn + tail


class StepCtx:
    """One workload's decode step on the device: seeded inputs resident in
    HBM, a MedusaStep, and the step's calls (overlapped as MedusaStep.run
    issues them, or the four calls in order)."""

    def __init__(self, w, dev):
        from medusa_tree_speculative_heads_b200 import binding as Bnd
        from medusa_tree_speculative_heads_b200 import inputs as I
        from medusa_tree_speculative_heads_b200.api import MedusaStep
        self.w, self.dev = w, dev
        self.parents = I.workload_tree(w)       # one parent list, or one per sequence
        self.seq_trees = I.sequence_trees(w)
        T = self.T = max(len(t) for t in self.seq_trees)
        self.hin = hin = I.head_inputs(w, device="cuda")
        self.ain = ain = I.attention_inputs(w, T, device="cuda")
        self.block_table = None
        paged = {}
        if w.page_size:
            # the cache as a page pool read through a block table
            pc = I.paged_cache(w, w.page_size, ain["prefix_len"].cpu(), room=T, device="cuda",
                               capacity=w.max_prefix + T)
            ain["k_cache"], ain["v_cache"], self.block_table = pc["k_pages"], pc["v_pages"], pc["block_table"]
            paged = dict(page_size=w.page_size, max_pages=self.block_table.shape[1], num_pages=pc["k_pages"].shape[0])
        self.k_layers = self.v_layers = None
        if w.tree_in_cache:
            # the tree's K/V appended to each sequence's cache after its prefix
            # (the target model's layers would write them there); every other
            # layer's cache is compacted in the same launch
            for b, tr in enumerate(self.seq_trees):
                S = int(ain["prefix_len"][b])
                ain["k_cache"][b, :, S:S + len(tr)] = ain["k_tree"][b, :len(tr)].transpose(0, 1)
                ain["v_cache"][b, :, S:S + len(tr)] = ain["v_tree"][b, :len(tr)].transpose(0, 1)
            self.k_layers = [ain["k_cache"]] + [ain["k_cache"].clone() for _ in range(w.layers - 1)]
            self.v_layers = [ain["v_cache"]] + [ain["v_cache"].clone() for _ in range(w.layers - 1)]
            ain["k_tree"] = ain["v_tree"] = None
        mode = Bnd.STOCHASTIC if w.stochastic else Bnd.GREEDY
        self.step = step = MedusaStep(B=w.B, d=w.d, V=w.V, K=w.K, Hq=w.Hq, Hkv=w.Hkv, D=w.D, S_max=w.S_max,
                                      parents=self.parents, dtype=w.torch_dtype, max_prefix=w.max_prefix,
                                      device=dev, mode=mode, q_rows=T, temperature=w.temperature,
                                      tree_in_cache=w.tree_in_cache, **paged)
        self.q_draft = self.vtok = None
        if w.stochastic:
            # the target's and the draft's distributions and the drafted tokens
            # (children drawn from q at their parent) come from the harness
            sd = I.stochastic_inputs(w, self.parents, device="cuda")
            self.logits, self.q_draft, self.vtok = sd["p"], sd["q"], sd["node_tokens"]
            if w.temperature > 0:   # the target's bf16 logits, read at the temperature
                self.logits = sd["logits"].bfloat16()
        else:
            # the target model's logits (outside this path) are synthesised once
            # from the tree the heads propose, with the workload's match probability
            step.heads(hin["h"], hin["W_res"], hin["W_head"], hin["root_token"])
            torch.cuda.synchronize()
            self.logits = I.boosted_target_logits(w, self.parents, step.node_tokens.cpu(), device="cuda")
        self.new_pl = torch.empty_like(ain["prefix_len"])

    def run_kwargs(self, src=None):
        """Arguments of MedusaStep.run; `src` replaces the per-step inputs
        (h, root token, q, tree K/V, target, draft, drafted tokens)."""
        hin, ain, src = self.hin, self.ain, src or {}
        return dict(h=src.get("h", hin["h"]), W_res=hin["W_res"], W_head=hin["W_head"],
                    root_token=src.get("root_token", hin["root_token"]), q=src.get("q", ain["q"]),
                    k_tree=src.get("k_tree", ain["k_tree"]), v_tree=src.get("v_tree", ain["v_tree"]),
                    k_cache=ain["k_cache"], v_cache=ain["v_cache"], prefix_len=ain["prefix_len"],
                    new_prefix_len=self.new_pl, target=src.get("target", self.logits),
                    q_draft=src.get("q_draft", self.q_draft), node_tokens=src.get("tokens", self.vtok),
                    block_table=self.block_table, k_layers=self.k_layers, v_layers=self.v_layers)

    def run_step(self):
        self.step.run(**self.run_kwargs())

    @property
    def fused_commit(self):
        """Greedy verification commits in the walk's launch (run() does that
        unless the commit is the all-layer compaction)."""
        return not self.w.stochastic and not self.w.tree_in_cache

    def stages(self, i):
        """The step's calls in order on the current stream, as run() issues
        them: heads, attention, verification (with the commit fused into the
        walk in greedy mode), and the commit when it is a separate call."""
        st, hin, ain = self.step, self.hin, self.ain
        calls = [lambda: st.heads(hin["h"], hin["W_res"], hin["W_head"], hin["root_token"]),
                 lambda: st.attention(ain["q"], ain["k_tree"], ain["v_tree"], ain["k_cache"], ain["v_cache"],
                                      ain["prefix_len"], self.block_table)]
        if self.fused_commit:
            calls.append(lambda: st.verify_commit(self.logits, ain["k_cache"], ain["v_cache"], ain["k_tree"],
                                                  ain["v_tree"], ain["prefix_len"], self.new_pl, self.block_table))
        else:
            calls += [lambda: st.verify(self.logits, self.q_draft, None, 0, i, self.vtok),
                      lambda: st.commit(ain["k_cache"], ain["v_cache"], ain["k_tree"], ain["v_tree"],
                                        ain["prefix_len"], self.new_pl, self.block_table, self.k_layers,
                                        self.v_layers)]
        return calls

    def algorithmic(self):
        """Algorithmic bytes of the heads and of tree attention, and the
        attention's FLOPs over visible (query, key) pairs only."""
        w = self.w
        elt = 2 if w.dtype == "bf16" else 4
        heads_bytes = (w.K * w.d * w.d + w.K * w.V * w.d) * elt + w.B * w.d * elt
        Sb = [int(x) for x in self.ain["prefix_len"].cpu()]
        Ts = [len(t) for t in self.seq_trees]
        attn_bytes = (2 * w.Hkv * sum(Sb) * w.D + 2 * sum(Ts) * w.Hq * w.D + 2 * sum(Ts) * w.Hkv * w.D) * elt
        anc = {}
        for tr in self.seq_trees:  # visible (node, tree node) pairs of each distinct tree
            key = tuple(tr)
            if key not in anc:
                anc[key] = sum(1 for i in range(len(tr)) for j in range(len(tr)) if _is_anc(tr, i, j))
        attn_flops = 4 * w.D * w.Hq * sum(Ts[b] * Sb[b] + anc[tuple(self.seq_trees[b])] for b in range(w.B))
        return heads_bytes, attn_bytes, attn_flops


L2_FLUSH_BYTES = 256 << 20   # twice the 126 MB L2


def measure_stages(ctx, K, flush):
    """Each of K repetitions: an L2 flush (a 256 MB memset, untimed), then the
    step's calls in order on one stream, each bracketed by CUDA events.
    Returns the median time of each stage (s) and the mean in-order step (s)."""
    n = len(ctx.stages(0))
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(n + 1)] for _ in range(K)]
    for i in range(K):
        flush.zero_()
        calls = ctx.stages(i)
        ev[i][0].record()
        for j, call in enumerate(calls):
            call()
            ev[i][j + 1].record()
    torch.cuda.synchronize()
    stage = [statistics.median(ev[i][j].elapsed_time(ev[i][j + 1]) for i in range(K)) / 1000.0 for j in range(n)]
    serial = statistics.mean(ev[i][0].elapsed_time(ev[i][n]) for i in range(K)) / 1000.0
    return stage, serial


def stage_dict(ctx, stage):
    """stage_us keys: the commit is reported with verification when the walk
    does it (one launch)."""
    d = {"medusa_heads": stage[0] * 1e6, "tree_attention": stage[1] * 1e6}
    if ctx.fused_commit:
        d["tree_verify+kv_commit"] = stage[2] * 1e6
    else:
        d["tree_verify"] = stage[2] * 1e6
        d["kv_compact" if ctx.w.tree_in_cache else "kv_commit"] = stage[3] * 1e6
    return d


def measure_steps(ctx, K, world, dev, barrier):
    """K back-to-back steps as MedusaStep.run issues them, CUDA events on the
    launching stream, barrier and synchronize on both sides; the slowest
    rank's time (s)."""
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    e0.record()
    for _ in range(K):
        ctx.run_step()
    e1.record()
    torch.cuda.synchronize()
    barrier()
    return max_over_ranks(e0.elapsed_time(e1) / 1000.0, world, dev)


def attention_roofline(attn_bytes, attn_flops, t_attn, pk):
    gbs = attn_bytes / t_attn / 1e9
    tflops = attn_flops / t_attn / 1e12
    bound = "tensor" if attn_flops / (pk["bf16_tflops"] * 1e12) > attn_bytes / (pk["hbm_gbs"] * 1e9) else "hbm"
    return {"us": t_attn * 1e6, "algorithmic_bytes": attn_bytes, "algorithmic_flops": attn_flops, "hbm_gbs": gbs,
            "hbm_frac": gbs / pk["hbm_gbs"], "tflops": tflops, "tc_frac": tflops / pk["bf16_tflops"], "bound": bound}


def choose_attention_sms(ctx, args):
    """SMs the heads kernel leaves to tree attention during its weight stream
    (MedusaStep attention_sms): --attention-sms N, or with "auto" the fastest
    of 0, 4, 8 and 16 over a few timed steps (the same computation every
    time; only the launch shape differs)."""
    if args.attention_sms != "auto":
        return int(args.attention_sms)
    best, best_t = 0, None
    for R in (0, 4, 8, 16):
        ctx.step.attention_sms = R
        for _ in range(3):
            ctx.run_step()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        e0.record()
        for _ in range(8):
            ctx.run_step()
        e1.record()
        torch.cuda.synchronize()
        t = e0.elapsed_time(e1)
        print(f"attention_sms {R}: {1000.0 * t / 8:.1f} us per step", file=sys.stderr, flush=True)
        if best_t is None or t < best_t * 0.995:
            best, best_t = R, t
    ctx.step.attention_sms = best
    return best


def measure_config(name, args, world, dev, barrier, flush, pk):
    """A compact measurement of another workload (same protocol, fewer steps)."""
    from medusa_tree_speculative_heads_b200 import inputs as I
    w = I.WORKLOADS[name]
    ctx = StepCtx(w, dev)
    K = max(5, min(args.steps, 30))
    for _ in range(max(args.warmup, 3)):
        ctx.run_step()
    torch.cuda.synchronize()
    R = choose_attention_sms(ctx, args)
    stage, serial = measure_stages(ctx, K, flush)
    t = measure_steps(ctx, K, world, dev, barrier)
    hb, ab, af = ctx.algorithmic()
    out = {"workload": config_dict(w, world)["workload"], "steps": K, "value": whole_job_rate(world, K, t),
           "unit": UNIT, "ms_per_step": 1000.0 * t / K, "serial_ms_per_step": 1000.0 * serial,
           "stage_us": stage_dict(ctx, stage),
           "medusa_heads": {"gbs": hb / stage[0] / 1e9, "hbm_frac": hb / stage[0] / 1e9 / pk["hbm_gbs"]},
           "tree_attention": attention_roofline(ab, af, stage[1], pk),
           "mean_accept_len": float(ctx.step.accept_len.float().mean().item()),
           "attention_sms": R, "status": int(ctx.step.status.item())}
    del ctx
    torch.cuda.empty_cache()
    return out


def run_mine(args, rank, world, local_rank):
    import torch.distributed as dist

    from medusa_tree_speculative_heads_b200 import build as build_mod
    from medusa_tree_speculative_heads_b200 import inputs as I

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)
    if rank == 0:
        build_mod.build()
    if world > 1:
        dist.barrier()

    def barrier():
        if world > 1:
            dist.barrier()

    w = I.WORKLOADS[args.workload]
    ctx = StepCtx(w, dev)
    step, hin, ain = ctx.step, ctx.hin, ctx.ain
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    for _ in range(max(args.warmup, 3)):
        ctx.run_step()
    torch.cuda.synchronize()
    attention_sms = choose_attention_sms(ctx, args)
    K = args.steps
    clocks = ClockSampler(local_rank)
    clocks.start()
    time.sleep(0.3)
    # ---- per-stage breakdown: the four calls in order, an L2 flush before each
    # repetition, median of K ----
    stage, serial_s = measure_stages(ctx, K, flush)
    # ---- device-timed steps (the value): the step as MedusaStep.run issues
    # it, tree attention on a second stream overlapping the heads' tail; each
    # step streams the heads' weights, far more than the 126 MB L2 ----
    t = measure_steps(ctx, K, world, dev, barrier)
    clk = clocks.stop()
    value = whole_job_rate(world, K, t)
    assert int(step.status.item()) == 0, "device status set during the benchmark"
    mean_len = float(step.accept_len.float().mean().item())

    # ---- end to end through the public API with host buffers ----
    # every step copies its own inputs from pinned host memory (h, root token,
    # the tree's Q/K/V and the target logits) and reads its results back; the
    # copies run on a second stream into two alternating device buffers, so the
    # next step's upload overlaps this step's compute, as a serving loop would
    names_in = ["h", "root_token", "q"] + ([] if w.tree_in_cache else ["k_tree", "v_tree"])
    host_in = {n: (hin if n in hin else ain)[n].cpu().pin_memory() for n in names_in}
    host_in["target"] = ctx.logits.cpu().pin_memory()
    if w.stochastic:
        host_in["q_draft"] = ctx.q_draft.cpu().pin_memory()
        host_in["tokens"] = ctx.vtok.cpu().pin_memory()
    dev_in = [{n: torch.empty_like(host_in[n], device=dev) for n in host_in} for _ in range(2)]
    outs = [step.accept_path, step.accept_len, step.bonus, step.node_tokens]   # int32, read back every step
    n_out = sum(o.numel() for o in outs)
    stage_out = [torch.empty(n_out, dtype=torch.int32, device=dev) for _ in range(2)]
    host_out = [torch.empty(n_out, dtype=torch.int32).pin_memory() for _ in range(2)]
    h2d = sum(x.numel() * x.element_size() for x in host_in.values())
    d2h = host_out[0].numel() * host_out[0].element_size()
    main_stream = torch.cuda.current_stream()
    copy_stream = torch.cuda.Stream(device=dev)
    # this machine's host-to-device rate for the step's uploads alone (median of 5)
    rates = []
    for _ in range(5):
        c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(copy_stream):
            c0.record(copy_stream)
            for n in host_in:
                dev_in[0][n].copy_(host_in[n], non_blocking=True)
            c1.record(copy_stream)
        c1.synchronize()
        rates.append(h2d / (c0.elapsed_time(c1) / 1000.0) / 1e9)
    h2d_gbs = statistics.median(rates)
    copied = [torch.cuda.Event(), torch.cuda.Event()]
    used = [torch.cuda.Event(), torch.cuda.Event()]
    for e in used:
        e.record(main_stream)
    # the results are packed into one buffer per slot on the compute stream
    # (one small kernel) and read back on a stream of their own: four small
    # device-to-host copies on the compute stream cost ~50 us of every step,
    # each a DMA with its own latency, that the next step need not wait for
    d2h_stream = torch.cuda.Stream(device=dev)
    packed = [torch.cuda.Event(), torch.cuda.Event()]
    read = [torch.cuda.Event(), torch.cuda.Event()]
    for e in read:
        e.record(d2h_stream)

    # one CUDA graph per input slot: a step is one graph launch on the host
    graphs, e2e_mode = None, "cuda-graph"
    try:
        torch.cuda.synchronize()
        graphs = [step.capture(**ctx.run_kwargs(dev_in[slot])) for slot in range(2)]
        torch.cuda.synchronize()
    except Exception as exc:  # capture unsupported here: the four calls are issued eagerly
        graphs, e2e_mode = None, f"eager ({type(exc).__name__})"
        torch.cuda.synchronize()

    def e2e_step(i):
        slot = i & 1
        with torch.cuda.stream(copy_stream):
            copy_stream.wait_event(used[slot])        # the step that last read this buffer is done
            for n in host_in:
                dev_in[slot][n].copy_(host_in[n], non_blocking=True)
            copied[slot].record(copy_stream)
        main_stream.wait_event(copied[slot])
        if graphs is not None:
            graphs[slot].replay()
        else:
            step.run(**ctx.run_kwargs(dev_in[slot]))
        used[slot].record(main_stream)
        main_stream.wait_event(read[slot])  # this slot's previous read-back is done
        torch.cat([o.view(-1) for o in outs], out=stage_out[slot])
        packed[slot].record(main_stream)
        d2h_stream.wait_event(packed[slot])
        with torch.cuda.stream(d2h_stream):
            host_out[slot].copy_(stage_out[slot], non_blocking=True)
            read[slot].record(d2h_stream)

    for i in range(W_E2E):
        e2e_step(i)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    e0.record()
    for i in range(K):
        e2e_step(i)
    for e in read:  # every step's results are on the host
        main_stream.wait_event(e)
    e1.record()
    torch.cuda.synchronize()
    barrier()
    t_e2e = max_over_ranks(e0.elapsed_time(e1) / 1000.0, world, dev)
    value_e2e = whole_job_rate(world, K, t_e2e)
    del graphs

    # ---- roofline of the dominant stage (the heads) and of tree attention ----
    pk = peaks()
    heads_bytes, attn_bytes, attn_flops = ctx.algorithmic()
    heads_gbs = heads_bytes / stage[0] / 1e9
    att = attention_roofline(attn_bytes, attn_flops, stage[1], pk)
    # the roofline object describes the step's dominant kernel: the heads
    # kernel (HBM-bound weight stream) or, at long contexts, tree attention,
    # bound by whichever of its HBM bytes and tensor-core FLOPs takes longer
    if stage[1] > stage[0]:
        if att["bound"] == "tensor":
            roofline = {"kernel": "tree_attention", "bound": "tensor", "achieved": att["tflops"],
                        "peak": pk["bf16_tflops"], "unit": "TFLOP/s", "frac": att["tc_frac"],
                        "peak_source": pk["source"], "algorithmic_flops": attn_flops, "traffic": None}
        else:
            roofline = {"kernel": "tree_attention", "bound": "hbm", "achieved": att["hbm_gbs"],
                        "peak": pk["hbm_gbs"], "unit": "GB/s", "frac": att["hbm_frac"], "peak_source": pk["source"],
                        "algorithmic_bytes": attn_bytes, "traffic": None}
    else:
        roofline = {"kernel": "medusa_heads (residual GEMV + LM-head GEMV with softmax/top-8 + merge)",
                    "bound": "hbm", "achieved": heads_gbs, "peak": pk["hbm_gbs"], "unit": "GB/s",
                    "frac": heads_gbs / pk["hbm_gbs"], "peak_source": pk["source"],
                    "algorithmic_bytes": heads_bytes,
                    "traffic": HEADS_DRAM_BYTES.get(w.name) if w.name not in OVERRIDDEN else None}
    roofline["timing"] = "median of the heads stage over K in-order repetitions, each after a 256 MB L2 flush"
    out = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K, "warmup": args.warmup,
        "ms_per_step": 1000.0 * t / K, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": w.dtype, "data": ("synthetic (seeded random weights and activations; stochastic verify on Zipf-"
                                   "ranked target and draft distributions)" if w.stochastic else
                                   "synthetic (seeded random weights and activations; target logits synthesised "
                                   f"from the proposed tree with match probability {w.match_prob})"),
        "config": {**config_dict(w, world),
                   "launch": (f"heads kernel on {torch.cuda.get_device_properties(dev).multi_processor_count - attention_sms}"
                              f" SMs, tree attention (no key splits) on the other {attention_sms} during the weight "
                              f"stream" if attention_sms else
                              "heads kernel on every SM, tree attention after it (key splits merged in-cluster)")},
        "roofline": roofline,
        "tree_attention": att,
        "stage_us": stage_dict(ctx, stage),
        "timing": ("value: K back-to-back steps as MedusaStep.run issues them (attention overlapped with the heads' "
                   "tail), CUDA events on the launching stream; stage_us and serial_ms_per_step: the step's calls in "
                   "order (greedy: the row scan, then the walk that also commits, one launch), median (stages) / "
                   "mean (step) of K repetitions, each after a 256 MB L2 flush"),
        "serial_ms_per_step": 1000.0 * serial_s,
        "mean_accept_len": mean_len,
        **({"kv_compact": {"layers": w.layers, "us": stage[-1] * 1e6,
                           "moved_bytes": 2 * 2 * w.layers * w.Hkv * w.D * (2 if w.dtype == "bf16" else 4) *
                           int(step.accept_len.sum().item()),
                           "note": "read + write of the accepted rows' K and V in every layer, one launch"}}
           if w.tree_in_cache else {}),
        "tokens_per_s": value * w.B * (mean_len + 1),
        "e2e": {"value": value_e2e, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "mode": e2e_mode, "h2d_gbs_measured": h2d_gbs,
                "note": "inputs copied from pinned host memory every step; the upload hides behind compute only "
                        "when h2d_bytes_per_step / h2d_gbs_measured is below the step time"},
        "gpu_launches": K * launches_per_step(w),
        "clocks": clk,
    }
    del ctx
    torch.cuda.empty_cache()
    # ---- the other configurations, each measured the same way (fewer steps) ----
    names = [n for n in args.configs.split(",") if n and n not in (w.name, "none")]
    if names:
        out["configs"] = {n: measure_config(n, args, world, dev, barrier, flush, pk) for n in names}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        frac = 1.0 / 16 if w.stochastic else 1.0   # B=64: a vocabulary / query-row slice keeps it to seconds
        v_omp, t_omp, f_omp, cores = time_oracle(w, frac, 10.0, 10.0, True)
        v_one, t_one, f_one, _ = time_oracle(w, frac, 10.0, 3.0, False)
        what = ("whole steps of the same workload" if frac == 1.0 else
                "steps' worth of work (residual blocks whole, LM-head rows of a 1/16 vocabulary slice, 1/16 of the "
                "attention rows, verification and commit whole; steps/s scaled by the sampled fraction)")
        out["cpu_baseline"] = {"value": v_omp, "unit": UNIT, "cores": cores, "kind": "oracle",
                               "sample": (f"{f_omp:.2f} {what}: the fp64 oracle's OpenMP build on {cores} host "
                                          f"threads ({t_omp:.1f} s)"),
                               "single_thread": {"value": v_one, "unit": UNIT, "cores": 1,
                                                 "sample": f"{f_one:.2f} {what}, serial build ({t_one:.1f} s)"}}
    if rank == 0:
        print(json.dumps(out), flush=True)
    if world > 1:
        dist.destroy_process_group()


def _is_anc(parents, i, j):
    while i != -1:
        if i == j:
            return True
        i = parents[i]
    return False


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="mine", choices=["mine", "reference"])
    ap.add_argument("--workload", default=WORKLOAD)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--attention-sms", default="auto",
                    help="SMs left to tree attention during the heads' weight stream (a number, or auto)")
    ap.add_argument("--configs", default="tiny,llama70b_b8,long32k,long128k,stoch_b64",
                    help="other workloads measured compactly into the line's 'configs' object ('none' for none)")
    ap.add_argument("--override", action="append", default=[],
                    help="replace a workload size, e.g. --override V=32000 (profiling a smaller case)")
    args = ap.parse_args()
    from medusa_tree_speculative_heads_b200 import inputs as I
    for ov in args.override:
        key, val = ov.split("=")
        I.WORKLOADS[args.workload] = I.scaled(I.WORKLOADS[args.workload], **{key: int(val)})
        OVERRIDDEN.add(args.workload)
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local_rank = int(os.environ.get("LOCAL_RANK", 0))
    if args.impl == "reference":
        run_reference(args, rank, world)
    else:
        run_mine(args, rank, world, local_rank)


if __name__ == "__main__":
    main()
