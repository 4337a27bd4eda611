"""The oracle's pins catch plausible mistakes: each case builds a copy of
oracle.c with one planted error (a dropped term, a wrong sign or index, a
flipped tie rule, a wrong constant), loads it in place of the real oracle, and
requires at least one of the pins aimed at that part to fail.  CPU only."""
import ctypes
import os
import subprocess

import pytest

import oracle
import test_oracle as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "oracle.c")

# (what is planted, the exact source text, its replacement, the pins that must catch it)
MUTANTS = [
    ("SiLU gate dropped", "hk[o] = z * sig + load(h, dtype, (size_t)b * d + o);",
     "hk[o] = z + load(h, dtype, (size_t)b * d + o);",
     [pins.test_heads_hand_d4_case_b_silu_ln3, pins.test_heads_silu_limits]),
    ("residual + h dropped", "hk[o] = z * sig + load(h, dtype, (size_t)b * d + o);", "hk[o] = z * sig;",
     [pins.test_heads_hand_d4_case_a, pins.test_heads_hand_d4_case_b_silu_ln3]),
    ("attention scale 1/D instead of 1/sqrt(D)", "if (scale <= 0.0) scale = 1.0 / sqrt((double)D);",
     "if (scale <= 0.0) scale = 1.0 / (double)D;",
     [pins.test_attention_chain_tree_is_causal_attention, pins.test_attention_single_node_is_decode_attention]),
    ("mask without the node itself", "for (int cur = i; cur != -1; cur = parent[cur])",
     "for (int cur = parent[i]; cur != -1; cur = parent[cur])", [pins.test_mask_guide_5_candidates]),
    ("argmax ties to the highest index", "        if (t > best) {", "        if (t >= best) {",
     [pins.test_greedy_argmax_ties_lowest_index]),
    ("top-k ties to the highest index", "if (best < 0 || x[i] > x[best]) best = i;",
     "if (best < 0 || x[i] >= x[best]) best = i;", [pins.test_topk_equals_stable_sort]),
    ("h^(k) not rounded to bf16 for bf16 inputs", "if (dtype == ORC_BF16 && round_hk) hk[o] = orc_round_bf16(hk[o]);",
     "if (0) hk[o] = orc_round_bf16(hk[o]);",
     [pins.test_heads_hand_d4_case_c_bf16_activation, pins.test_heads_bf16_stores_hk_as_bf16]),
    ("residual with the sign flipped", "double diff = P[y] - (double)Q[y];", "double diff = (double)Q[y] - P[y];",
     [pins.test_residual_normalises_and_closed_form]),
    ("acceptance test inverted", "if (uc * (double)Q[x] < P[x]) {", "if (uc * (double)Q[x] > P[x]) {",
     [pins.test_stochastic_one_hot_draft_closed_form]),
    ("Philox Weyl constant off by one", "const uint32_t W0 = 0x9E3779B9u,", "const uint32_t W0 = 0x9E3779B8u,",
     [pins.test_philox_known_answers]),
    ("temperature dropped", "P[y] = exp((z[y] - m) * inv_tau);", "P[y] = exp(z[y] - m);",
     [lambda o: pins.test_softmax_temperature_vs_scipy(o, 0.7),
      pins.test_stochastic_logits_temperature_scaling_and_shift]),
    ("compaction without the prefix offset", "blk + (size_t)(S + path[(size_t)b * max_path + t]) * row",
     "blk + (size_t)(path[(size_t)b * max_path + t]) * row", [pins.test_kv_compact_hand_example]),
    ("page slot from the page number", "+ s % page_size) * D * esize;", "+ s / page_size) * D * esize;",
     [pins.test_gather_pages_identity_table_is_a_reshape]),
    ("tree fill ignores the sibling rank", "size_t e = ((size_t)b * K + (depth[i] - 2)) * S + rank[i];",
     "size_t e = ((size_t)b * K + (depth[i] - 2)) * S + 0;", [pins.test_tree_fill_product_tree]),
    ("kv-head of a q-head taken modulo", "int g = h / G;", "int g = h % Hkv;",
     [pins.test_attention_product_tree_vs_sdpa_with_path_mask]),
    ("deepest accepted node: highest index on ties", "if (acc[c] && depth[c] > depth[best]) best = c;",
     "if (acc[c] && depth[c] >= depth[best]) best = c;",
     [pins.test_greedy_equally_deep_nodes_take_the_lowest_index]),
    ("acceptance without the parent's", "acc[c] = acc[parent[c]] && node_tokens[(size_t)b * T + c] == pred[parent[c]];",
     "acc[c] = node_tokens[(size_t)b * T + c] == pred[parent[c]];", [pins.test_greedy_vs_brute_force]),
    ("children tried in reverse order", "for (int c = u + 1; c < T; ++c) {", "for (int c = T - 1; c > u; --c) {",
     [pins.test_stochastic_draft_equals_target_accepts_all]),
    ("the accepted child keeps its parent's target row",
     "++L;\n                    load_row(src, (size_t)b * T + u, V, P);", "++L;",
     [lambda o: pins.test_stochastic_first_token_follows_target(o, 1)]),
    ("attention's V from the tree row of the wrong kv-head",
     "size_t voff = (((size_t)b * T + j) * Hkv + g) * D;", "size_t voff = (((size_t)b * T + j) * Hkv + 0) * D;",
     [pins.test_attention_product_tree_vs_sdpa_with_path_mask]),
    ("attention reads one prefix key too many",
     "        int n = 0;\n        for (int j = 0; j < S; ++j) {", "        int n = 0;\n        for (int j = 0; j <= S; ++j) {",
     [pins.test_attention_chain_tree_is_causal_attention, pins.test_attention_single_node_is_decode_attention]),
    ("compaction accepts a repeated node", "if (n <= prev || n >= T) ok = 0;", "if (n < prev || n >= T) ok = 0;",
     [pins.test_kv_compact_refusals]),
    ("paged commit writes every row into the prefix's last page",
     "int page = table[(size_t)b * max_pages + (S + t) / page_size];",
     "int page = table[(size_t)b * max_pages + S / page_size];",
     [pins.test_paged_commit_equals_contiguous_commit_through_the_table]),
    ("commit one row late", "size_t dst = ((((size_t)b * Hkv + g) * S_max) + S + t) * D * esize;",
     "size_t dst = ((((size_t)b * Hkv + g) * S_max) + S + t + 1) * D * esize;",
     [pins.test_kv_commit_exact_and_canaries]),
]


def _build_mutant(tmp_path, old, new):
    src = open(SRC).read()
    assert src.count(old) == 1, f"the planted site must be unique: {old!r}"
    path = tmp_path / "oracle_mutant.c"
    path.write_text(src.replace(old, new))
    so = tmp_path / "liboracle_mutant.so"
    subprocess.check_call(["gcc", "-O2", "-std=gnu11", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared",
                           "-o", str(so), str(path), "-lm"])
    return oracle.configure(ctypes.CDLL(str(so)))


@pytest.mark.parametrize("what,old,new,catchers", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_a_planted_mistake(tmp_path, monkeypatch, what, old, new, catchers):
    for pin in catchers:   # the real oracle passes the pins
        pin(oracle)
    monkeypatch.setattr(oracle, "_lib", _build_mutant(tmp_path, old, new))
    failed = 0
    for pin in catchers:
        try:
            pin(oracle)
        except (AssertionError, ValueError):
            failed += 1
    assert failed > 0, f"no pin caught: {what}"
