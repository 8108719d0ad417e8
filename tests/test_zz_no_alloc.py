"""lightning_index_topk_static: the indexer + top-k call that keeps its scores
in the library's own device array and allocates nothing.

It exists for callers that cannot allocate device memory: code running under
a memory manager that has already reserved the GPU's memory, code that may
not stall the device, or code whose interface has no workspace to pass.  Its
results must be those of lightning_index_topk with a caller workspace.

This file is named so that pytest collects it last."""
import ctypes as C

import numpy as np
import pytest
import torch

from compressed_sparse_kv_04_b200 import binding, configs, synth

DEV = "cuda"
STATIC_SCORES = 1 << 21  # capacity of the library's array, in fp32 scores


def _keys(B, N, D_I, seed):
    g = torch.Generator(device="cpu").manual_seed(seed)
    x = (torch.randn(B, N, D_I, generator=g) * 64).clamp(-448, 448)
    codes = x.to(torch.float8_e4m3fn).view(torch.uint8)
    scale = torch.rand(B, N, generator=g) * 0.01 + 0.005
    return codes.to(DEV), scale.to(DEV)


def _both(w, N_cap, pos, seed):
    """Top-k of one input set through the workspace call and the static call."""
    B, Q = w.B, 1
    key, ks = _keys(B, N_cap, w.D_I, seed)
    qi = synth.queries(w, Q=Q, device=DEV)
    p = binding.params_for(w)
    pos_t = torch.as_tensor(pos, dtype=torch.int64, device=DEV).reshape(B, Q)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    ws = binding.workspace(p, binding.OP_INDEX_TOPK, Q, N_cap)
    ref_idx = torch.full((B, Q, p.k), -7, dtype=torch.int32, device=DEV)
    ref_cnt = torch.full((B, Q), -7, dtype=torch.int32, device=DEV)
    binding.lightning_index_topk(p, Q, qi["q_idx"], qi["q_scale"], qi["w"], key, ks, pos_t,
                                 ref_idx, ref_cnt, ws=ws, dev_status=status)
    idx = torch.full((B, Q, p.k), -9, dtype=torch.int32, device=DEV)
    cnt = torch.full((B, Q), -9, dtype=torch.int32, device=DEV)
    binding.lightning_index_topk_static(p, Q, qi["q_idx"], qi["q_scale"], qi["w"], key, ks, pos_t,
                                        idx, cnt, dev_status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    return ref_idx.cpu().numpy(), ref_cnt.cpu().numpy(), idx.cpu().numpy(), cnt.cpu().numpy()


@pytest.mark.gpu
def test_static_matches_workspace_call_twice():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    # First call: a batch of 8 at 128K tokens, every entry visible.
    w1 = configs.CSA_128K
    N1 = w1.N_c
    assert w1.B * N1 <= STATIC_SCORES
    r1 = _both(w1, N1, [[w1.L - 1]] * w1.B, seed=31)
    # Second call: another shape and ragged visible counts, so that rows are
    # shorter than the previous call's and the array still holds its scores.
    w2 = configs.scaled(configs.CSA_128K, B=3)
    N2 = 20000
    r2 = _both(w2, N2, [[4 * N2 - 1], [4 * 700 + 2], [4 * 9000 + 1]], seed=32)
    for ref_idx, ref_cnt, idx, cnt in (r1, r2):
        assert np.array_equal(cnt, ref_cnt)
        assert np.array_equal(idx, ref_idx)
    assert (r2[1].ravel() == [1024, 700, 1024]).all()


def test_static_rejects_oversize_before_any_launch():
    """Sizes beyond the array are refused with CSA_ERR_WORKSPACE (no device
    work, so this runs without a GPU too)."""
    L = binding.lib()
    w = configs.CSA_128K
    p = binding.params_for(w)
    N_cap = STATIC_SCORES // w.B + 1
    st = L.lightning_index_topk_static(C.byref(p), 1, None, None, None, None, None, N_cap, None,
                                       None, None, None, None)
    assert st == 4
    msg = L.csa_last_error().decode()
    assert "static buffer" in msg and str(STATIC_SCORES) in msg
