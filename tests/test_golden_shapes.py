"""The workloads carry the shape constants the pages state (tests/golden)."""
import json
import math
import os

from compressed_sparse_kv_04_b200 import configs

G = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "v4_pro_attention_shapes.json")))


def v(name):
    return G[name]["value"]


def test_pro_shapes_in_workloads():
    for w in (configs.CSA_128K, configs.CSA_1M, configs.CSA_PREFILL):
        assert (w.m, w.H_I, w.D_I, w.k) == (v("csa_ratio_m"), v("indexer_heads"), v("indexer_head_dim"), v("top_k"))
    for w in (configs.CSA_128K, configs.HCA_1M, configs.CSA_1M, configs.CSA_PREFILL):
        assert (w.H, w.D, w.rope_dim, w.W) == (v("query_heads"), v("head_dim"), v("rope_dims"), v("window"))
    assert configs.HCA_1M.m == v("hca_ratio_m_prime")


def test_one_million_context_entry_counts():
    L = v("context_tokens")
    assert configs.CSA_1M.L == L and configs.HCA_1M.L == L
    n_csa = math.ceil(L / v("csa_ratio_m"))
    assert n_csa == configs.CSA_1M.N_c == 262144
    assert abs(n_csa - v("indexer_candidates_at_1m_approx")) / n_csa < 0.01
    assert configs.HCA_1M.N_c == 8192
    # The double reduction of CSA: n -> n/m -> k.
    assert n_csa // v("top_k") == 256


def test_flash_and_yarn_settings():
    w = configs.CSA_FLASH_128K
    assert (w.H, w.k) == (v("flash_query_heads"), v("flash_top_k"))
    assert (w.m, w.H_I, w.D_I, w.D, w.rope_dim, w.W) == (
        v("csa_ratio_m"), v("indexer_heads"), v("indexer_head_dim"), v("head_dim"), v("rope_dims"),
        v("window"))
    factor, beta_fast, beta_slow, original_len = w.yarn
    assert (factor, beta_fast, beta_slow) == (
        v("yarn_factor"), v("yarn_beta_fast"), v("yarn_beta_slow"))
    assert original_len * factor == v("context_tokens")
