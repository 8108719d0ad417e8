"""Host-only checks of the C ABI: the library builds, loads and exports every
symbol include/csa.h declares, and argument validation rejects bad calls
before anything reaches a device.  No test here passes a non-null device
pointer, so nothing can be launched.
"""
import ctypes as C
import os
import re

import pytest

from compressed_sparse_kv_04_b200 import binding
from compressed_sparse_kv_04_b200 import build as csa_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    csa_build.build()
    return binding.lib()


def declared_functions():
    names = []
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if not fn.endswith(".h"):
            continue
        text = open(os.path.join(ROOT, "include", fn)).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        for m in re.finditer(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s*([a-z_][a-z0-9_]*)\s*\(",
                             text, flags=re.M):
            names.append(m.group(1))
    return sorted(set(names))


def test_header_declares_the_six_entry_points():
    names = declared_functions()
    for n in ["hca_compress", "csa_compress", "lightning_index_topk", "sparse_mqa_decode",
              "dense_mqa_decode", "csa_prefill_chunk"]:
        assert n in names


def test_library_exports_every_declared_symbol(L):
    for name in declared_functions():
        assert hasattr(L, name), name
    assert set(binding.EXPORTS) <= set(declared_functions())


def test_version_and_error_string(L):
    assert L.csa_version() >= 100
    assert isinstance(L.csa_last_error(), bytes)


def P(**kw):
    base = dict(B=1, d=512, H=128, H_I=64, D_I=128, k=1024, window=128, rope_dim=64, m=4)
    base.update(kw)
    return binding.make_params(**base)


def test_null_params_rejected(L):
    assert L.hca_compress(None, None, 1, None, None, None, None, 0, 1, None, 1, None, None) == 1
    assert L.csa_workspace_bytes(None, 1, 1, 1) == 0


@pytest.mark.parametrize("kw,code", [(dict(d=256), 2), (dict(m=0), 2), (dict(m=200), 2),
                                     (dict(B=0), 1), (dict(eps=0.0), 1)])
def test_bad_shapes_rejected(L, kw, code):
    p = P(**kw)
    st = L.hca_compress(C.byref(p), None, 1, None, None, None, None, 0, 1, None, 1, None, None)
    assert st == code, binding.lib().csa_last_error()


def test_null_tensor_rejected_before_launch(L):
    p = P()
    st = L.lightning_index_topk(C.byref(p), 1, None, None, None, None, None, 1024, None, None,
                                None, None, None, 0, None, None)
    assert st == 1
    assert b"q_idx" in L.csa_last_error()


def test_indexer_shape_limits(L):
    for kw in (dict(D_I=96), dict(H_I=65), dict(k=2049), dict(k=0)):
        p = P(**kw)
        st = L.lightning_index_topk(C.byref(p), 1, None, None, None, None, None, 1024, None,
                                    None, None, None, None, 0, None, None)
        assert st == 2, kw


def test_attention_shape_limits(L):
    for kw in (dict(H=129), dict(rope_dim=63), dict(rope_dim=512), dict(rope_dim=128), dict(window=-1)):
        p = P(**kw)
        st = L.dense_mqa_decode(C.byref(p), None, None, None, 1, None, 1, None, None, None,
                                None, None, None, 0, None, None)
        assert st == 2, kw


def test_prefill_argument_checks(L):
    p = P(B=2)
    args = [None] * 2 + [1] + [None] * 8 + [1] + [None] * 10 + [None, 0, None, None]
    st = L.csa_prefill_chunk(C.byref(p), 0, 4, *args)
    assert st == 2  # B must be 1
    p = P(B=1)
    st = L.csa_prefill_chunk(C.byref(p), 3, 4, *args)
    assert st == 1  # P not a multiple of m


def test_hca_prefill_argument_checks(L):
    def call(p, P_, T, L_cap=1 << 20, N_cap=1 << 13):
        return L.hca_prefill_chunk(C.byref(p), P_, T, None, L_cap, None, None, None, None, N_cap,
                                   None, None, None, None, None, None, None, 0, None, None)
    assert call(P(B=2, m=128), 0, 4) == 2          # B must be 1
    p = P(B=1, m=128)
    assert call(p, 3, 4) == 1                      # P not a multiple of m
    assert call(p, 0, 0) == 1                      # T >= 1
    assert call(p, 0, 70000) == 2                  # T <= 65535
    assert call(p, 128, 10, L_cap=100) == 3        # P+T > L_cap
    assert call(p, 0, 300, L_cap=1024, N_cap=2) == 3  # ceil(300/128) > N_cap
    assert call(p, 0, 300, L_cap=1024, N_cap=3) == 1  # q is NULL
    assert L.csa_workspace_bytes(C.byref(p), 5, 4096, 544) > 0


def test_decode_step_argument_checks(L):
    p = P(B=2)
    n = [None] * 29
    n[0] = C.byref(p)
    n[4], n[13], n[26] = 1 << 12, 1 << 10, 0  # L_cap, N_cap, ws_bytes
    assert L.csa_decode_step(*n) == 1            # pos_q (and the rest) NULL
    p = P(B=2, k=4096)
    n[0] = C.byref(p)
    assert L.csa_decode_step(*n) in (1, 2)       # k outside 1..2048 or NULL pointers
    h = [None] * 19
    h[0] = C.byref(P(B=2, m=128))
    h[3], h[8], h[16] = 1 << 12, 32, 0
    assert L.hca_decode_step(*h) == 1            # NULL tensors
    assert L.csa_workspace_bytes(C.byref(P(B=8)), 6, 1, 32768) > \
        L.csa_workspace_bytes(C.byref(P(B=8)), 2, 1, 32768)
    assert L.csa_workspace_bytes(C.byref(P(B=8, m=128)), 7, 1, 8192) > 0


def test_workspace_sizes_are_monotone(L):
    p = P(B=8)
    a = L.csa_workspace_bytes(C.byref(p), 1, 1, 32768)
    b = L.csa_workspace_bytes(C.byref(p), 1, 1, 65536)
    assert 0 < a < b
    assert L.csa_workspace_bytes(C.byref(p), 2, 1, 32768) > 0
    assert L.csa_workspace_bytes(C.byref(p), 3, 1, 8192) > 0
    assert L.csa_workspace_bytes(C.byref(p), 9, 1, 8192) == 0


# ---------------------------------------------- YaRN frequency table (host) --
@pytest.mark.parametrize("args", [(64, 16.0, 32.0, 1.0, 65536.0), (32, 4.0, 32.0, 1.0, 4096.0),
                                  (64, 1.0, 32.0, 1.0, 4096.0), (64, 40.0, 16.0, 2.0, 1.0e6),
                                  (2, 16.0, 32.0, 1.0, 100.0)])
def test_yarn_table_matches_the_oracle(L, orc, args):
    import math

    import numpy as np
    tab, gain, scale = binding.rope_yarn(*args, d=512)
    assert np.allclose(tab, orc.yarn_inv_freq(*args), rtol=1e-14, atol=0)
    assert math.isclose(gain, orc.yarn_logit_gain(args[1]), rel_tol=1e-14)
    # The ready logit scale (binary32) is the gain over sqrt(d).
    ref = orc.yarn_logit_gain(args[1]) / math.sqrt(512)
    assert abs(scale - ref) <= ref * 2.0 ** -24
    _, _, s128 = binding.rope_yarn(*args, d=128)
    assert abs(s128 - 2 * ref) <= 2 * ref * 2.0 ** -24


@pytest.mark.parametrize("args,code", [((63, 16.0, 32.0, 1.0, 65536.0), 2),
                                       ((0, 16.0, 32.0, 1.0, 65536.0), 2),
                                       ((130, 16.0, 32.0, 1.0, 65536.0), 2),
                                       ((64, 0.5, 32.0, 1.0, 65536.0), 1),
                                       ((64, 16.0, 1.0, 1.0, 65536.0), 1),
                                       ((64, 16.0, 32.0, -1.0, 65536.0), 1),
                                       ((64, 16.0, 32.0, 1.0, 0.0), 1),
                                       ((64, 16.0, 32.0, 1.0, float("nan")), 1),
                                       ((64, float("inf"), 32.0, 1.0, 65536.0), 1)])
def test_yarn_argument_checks(L, args, code):
    with pytest.raises(binding.CsaError) as e:
        binding.rope_yarn(*args)
    assert e.value.status == code
    assert L.csa_rope_yarn(64, 1e4, 16.0, 32.0, 1.0, 65536.0, 512, None, None, None) == 1
    tab = (C.c_double * 32)()
    sc = C.c_float()
    assert L.csa_rope_yarn(64, 1e4, 16.0, 32.0, 1.0, 65536.0, 0, tab, None, C.byref(sc)) == 1
    assert L.csa_rope_yarn(64, 1e4, 16.0, 32.0, 1.0, 65536.0, 0, tab, None, None) == 0


# ------------------------------------------- bench accounting (no GPU) --
def test_step_algorithmic_bytes_per_query():
    """Per query of a decode step: indexer keys N (D_I + 4), gathered entries
    k d 2, window W d 2, newest-block compression (m d 2 + d 2 for the KV,
    m D_I 2 + D_I + 4 for the indexer), q and out H d 2 each, the indexer
    query H_I (D_I + 8), the selection k 4 written and read, its count; once
    per step (shared by the batch): the sinks H 4 and the pooling weights.
    The fp32 scores are implementation traffic (not counted)."""
    import sys
    sys.argv = ["bench"]
    import bench
    from compressed_sparse_kv_04_b200 import configs
    for w in (configs.CSA_128K, configs.CSA_1M):
        N, d, k, W, m, H, HI, DI = w.N_c, w.d, w.k, w.W, w.m, w.H, w.H_I, w.D_I
        per_q = (N * (DI + 4) + k * d * 2 + W * d * 2 + (m * d * 2 + d * 2) + (m * DI * 2 + DI + 4)
                 + 2 * H * d * 2 + HI * (DI + 8) + 2 * k * 4 + 4)
        weights = ((d + m) * 4 * 2 + H * 4) / w.B  # pooling weights and sinks, once per step
        got = bench.algorithmic_bytes(w)["step"] / w.B
        assert abs(got - (per_q + weights)) <= 8, (w.name, got, per_q + weights)
    w = configs.HCA_1M
    per_q = (w.N_c + w.W) * w.d * 2 + w.m * w.d * 2 + w.d * 2 + 2 * w.H * w.d * 2 + w.H * 4 / w.B
    got = bench.algorithmic_bytes(w)["step"] / w.B
    assert abs(got - per_q - (w.d + w.m) * 4 / w.B) <= 8, (got, per_q)


def test_params_for_applies_yarn_to_a_yarn_workload(L, orc):
    import math

    import numpy as np
    from compressed_sparse_kv_04_b200 import configs
    w = configs.CSA_FLASH_128K
    p = binding.params_for(w)
    tab = np.array([p.rope_inv_freq[j] for j in range(w.rope_dim // 2)])
    assert np.allclose(tab, orc.yarn_inv_freq(w.rope_dim, *w.yarn), rtol=1e-14, atol=0)
    ref = orc.yarn_logit_gain(w.yarn[0]) / math.sqrt(w.d)
    assert abs(p.softmax_scale - ref) <= ref * 2.0 ** -24
    plain = binding.params_for(configs.CSA_128K)
    assert not plain.rope_inv_freq and plain.softmax_scale == 0.0


# ------------------------------------------ grouped output projection (host) --
@pytest.mark.parametrize("shape,code", [((8, 128, 512, 16, 1024, 7168), 0),
                                        ((8, 128, 512, 12, 1024, 7168), 2),   # g does not divide H
                                        ((8, 128, 512, 16, 1000, 7168), 2),   # d_g % 128
                                        ((8, 128, 512, 16, 1024, 7000), 2),   # d % 128
                                        ((0, 128, 512, 16, 1024, 7168), 1),
                                        ((8, 128, 36, 16, 1024, 7168), 2)])   # (H/g)*D % 64
def test_grouped_out_proj_argument_checks(L, shape, code):
    n = L.grouped_out_proj_workspace_bytes(*shape)
    assert (n > 0) == (code == 0)
    # NULL tensors: the shape error wins, else the pointer check.
    st = L.grouped_out_proj(*shape, None, None, None, None, None, None, 0, None, None)
    assert st == (code if code else 1)


def test_grouped_out_proj_workspace_grows_with_tokens(L):
    a = L.grouped_out_proj_workspace_bytes(8, 128, 512, 16, 1024, 7168)
    b = L.grouped_out_proj_workspace_bytes(4096, 128, 512, 16, 1024, 7168)
    assert 0 < a < b
    # At least the bf16 intermediate y.
    assert b >= 4096 * 16 * 1024 * 2


def test_copy_entry_points_check_arguments(L):
    """csa_copy_async / csa_copy_rows_async refuse NULL addresses and pitches
    below the row before any copy is enqueued; empty copies do nothing."""
    import ctypes as C
    buf = (C.c_char * 64)()
    a = C.cast(buf, C.c_void_p)
    assert L.csa_copy_async(a, a, 0, None) == 0
    assert L.csa_copy_async(None, a, 16, None) == 1
    assert L.csa_copy_async(a, None, 16, None) == 1
    assert L.csa_copy_rows_async(a, 64, a, 64, 0, 3, None) == 0
    assert L.csa_copy_rows_async(a, 64, a, 64, 16, 0, None) == 0
    assert L.csa_copy_rows_async(a, 8, a, 64, 16, 2, None) == 1
    assert L.csa_copy_rows_async(a, 64, a, 8, 16, 2, None) == 1
    assert L.csa_copy_rows_async(None, 64, a, 64, 16, 2, None) == 1
    assert b"pitch" in L.csa_last_error() or b"NULL" in L.csa_last_error()


def test_prepared_copy_checks_its_tensors(L):
    """PreparedCopy wants equal shapes and dtypes and page-locked host
    memory (checked before the library is called)."""
    import torch
    a, b = torch.zeros(4, 8), torch.zeros(4, 9)
    with pytest.raises(ValueError):
        binding.PreparedCopy(a, b)
    with pytest.raises(ValueError):
        binding.PreparedCopy(a, a.clone())  # neither side on a device nor pinned


def test_prepared_copy_row_layout():
    """The (rows, row bytes, pitch) that PreparedCopy passes to
    csa_copy_rows_async: one row per first-dimension slice of a strided
    view, its bytes contiguous, the pitch the first dimension's stride."""
    import torch
    buf = torch.zeros(3, 37, 512, dtype=torch.bfloat16)
    assert binding._rows_of(buf[:, 11:12]) == (3, 1024, 37 * 512 * 2)
    assert binding._rows_of(buf[:, 5:9]) == (3, 4 * 1024, 37 * 512 * 2)
    host = torch.zeros(3, 1, 512, dtype=torch.bfloat16)
    assert binding._rows_of(host) == (3, 1024, 1024)
    assert binding._rows_of(torch.zeros(1, 7, dtype=torch.uint8)) == (1, 7, 7)
    with pytest.raises(ValueError):  # rows that are not contiguous
        binding._rows_of(buf[:, :, ::2])


def test_prepared_decode_steps_reject_host_tensors(L):
    """CsaDecodeStep / HcaDecodeStep check their tensors like the plain calls
    (host tensors are refused before anything reaches the library)."""
    import torch
    from compressed_sparse_kv_04_b200 import configs
    w = configs.scaled(configs.CSA_128K, B=1, L=64)
    p = binding.params_for(w)
    t = torch.zeros(16)
    with pytest.raises(ValueError):
        binding.CsaDecodeStep(p, t, t, t, t, None, t, t, t, t, t, t, t, t, t)
    with pytest.raises(ValueError):
        binding.HcaDecodeStep(p, t, t, t, None, t, t, t)
