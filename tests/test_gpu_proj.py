"""GPU parity: grouped output projection (grouped_out_proj, tcgen05 bf16 GEMMs)
through the C ABI, against the fp64 oracle.

Layered checks: the intermediate y (bf16) against the oracle's exact y, one
bf16 rounding plus fp32 accumulation (|d| <= 2^-8 |y| + 1e-3); z against the
oracle's second projection of the GPU's own y, the same bound; and z end to
end (the oracle rounding y itself) within the attention tolerance (max abs
<= 2e-2, relative L2 <= 5e-3), since a y element that lands on the other
side of a bf16 rounding boundary moves z slightly.  Shapes cover ragged
token counts (one to several token tiles), split-K (small grids), the
V4-Pro shape (g = 16, d_g = 1024, 128 heads of 512) chained after the
sparse attention at the 128K decode shape, and the 4096-token prefill shape
on sampled rows."""
import math

import numpy as np
import pytest
import torch

from compressed_sparse_kv_04_b200 import binding, configs, synth
from gpuhelp import assert_attention_close, assert_bf16_storage_close, bits16

pytestmark = pytest.mark.gpu
DEV = "cuda"
D_MODEL = 7168  # the pages do not give d; see the entry point's documentation


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    binding.lib()


def weights(H, D, g, d_g, d_model, seed):
    gen = torch.Generator(device=DEV).manual_seed(seed)
    k1 = (H // g) * D
    w_g = (torch.randn(g, d_g, k1, generator=gen, device=DEV) / math.sqrt(k1)).to(torch.bfloat16)
    w_o = (torch.randn(d_model, g * d_g, generator=gen, device=DEV) /
           math.sqrt(g * d_g)).to(torch.bfloat16)
    return w_g, w_o


def run(o, w_g, w_o):
    T = o.shape[0]
    g, d_g, _ = w_g.shape
    y = torch.full((T, g * d_g), float("nan"), dtype=torch.bfloat16, device=DEV)
    z = torch.full((T, w_o.shape[0]), float("nan"), dtype=torch.bfloat16, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    binding.grouped_out_proj(o, w_g, w_o, z, y=y, dev_status=status)
    torch.cuda.synchronize()
    assert status.item() == 0, status.item()
    return y, z


def check(orc, o, w_g, w_o, y, z, rows=None, what=""):
    ob, wg, wo = bits16(o), bits16(w_g), bits16(w_o)
    yb, zv = bits16(y), z.double().cpu().numpy()
    if rows is not None:
        ob, yb, zv = ob[rows], yb[rows], zv[rows]
    y_exact, _ = orc.grouped_out_proj(ob, wg, wo, y_bf16=False)
    assert_bf16_storage_close(yb, y_exact, what + " y")
    _, z_chain = orc.grouped_out_proj(ob, wg, wo, y_in=yb)
    assert_bf16_storage_close(bits16(z)[rows] if rows is not None else bits16(z), z_chain,
                              what + " z (on the GPU's y)")
    _, z_ref = orc.grouped_out_proj(ob, wg, wo, y_bf16=True)
    assert np.isfinite(zv).all()
    assert_attention_close(zv, z_ref, what + " z end to end")


@pytest.mark.parametrize("T", [1, 8, 37, 300])
def test_proj_small_ragged(orc, T):
    H, D, g, d_g, d_model = 16, 128, 4, 128, 256
    o = synth.normal_bf16((T, H, D), 100 + T, "q", DEV)
    w_g, w_o = weights(H, D, g, d_g, d_model, 101 + T)
    y, z = run(o, w_g, w_o)
    check(orc, o, w_g, w_o, y, z, what=f"T={T}")


@pytest.mark.parametrize("T", [3, 16, 130])
def test_proj_split_k(orc, T):
    """Few output tiles and long inner dims: both projections split K (fp32
    partials summed by the reduce kernel)."""
    H, D, g, d_g, d_model = 16, 512, 2, 128, 128
    o = synth.normal_bf16((T, H, D), 200 + T, "q", DEV)
    w_g, w_o = weights(H, D, g, d_g, d_model, 201 + T)
    y, z = run(o, w_g, w_o)
    check(orc, o, w_g, w_o, y, z, what=f"split-K T={T}")


def test_proj_after_sparse_attention_128k_decode(orc):
    """The V4-Pro projection (g = 16, d_g = 1024, d = 7168) of the sparse
    attention output at the 128K decode shape (8 sequences x 128 heads x 512)."""
    w = configs.CSA_128K
    g = torch.Generator(device=DEV).manual_seed(40)
    kv_c = torch.randn(w.B, w.N_c, w.D, generator=g, device=DEV)
    kv_c = (kv_c / kv_c.pow(2).mean(-1, keepdim=True).sqrt()).to(torch.bfloat16)
    kv_tok = torch.randn(w.B, w.L, w.D, generator=g, device=DEV).to(torch.bfloat16)
    q = synth.normal_bf16((w.B, w.H, w.D), 41, "q", DEV)
    sink = synth.normal_f32((w.H,), 42, "sink", 1.0, DEV)
    rng = np.random.default_rng(43)
    sel = np.stack([np.sort(rng.choice(w.N_c, w.k, replace=False)) for _ in range(w.B)])
    sel = torch.from_numpy(sel.astype(np.int32)).to(DEV)
    cnt = torch.full((w.B,), w.k, dtype=torch.int32, device=DEV)
    p = binding.params_for(w)
    out = torch.empty(w.B, w.H, w.D, dtype=torch.bfloat16, device=DEV)
    ws = binding.workspace(p, binding.OP_SPARSE_MQA, 1, w.N_c)
    pos = torch.full((w.B,), w.L - 1, dtype=torch.int64, device=DEV)
    binding.sparse_mqa_decode(p, q, pos, kv_c, sel, cnt, kv_tok, sink, out, ws=ws)
    del kv_tok, kv_c
    w_g, w_o = weights(w.H, w.D, 16, 1024, D_MODEL, 44)
    y, z = run(out, w_g, w_o)
    check(orc, out, w_g, w_o, y, z, what="V4-Pro decode")


def test_proj_prefill_4096_sampled(orc):
    """4096 tokens (16 token tiles of 256), the V4-Pro weights; the oracle
    checks a sample of rows (tile edges and random rows)."""
    T, H, D = 4096, 128, 512
    o = synth.normal_bf16((T, H, D), 300, "q", DEV)
    w_g, w_o = weights(H, D, 16, 1024, D_MODEL, 301)
    y, z = run(o, w_g, w_o)
    rng = np.random.default_rng(302)
    rows = sorted({0, 1, 255, 256, 2047, T - 1, *rng.choice(T, 10, replace=False).tolist()})
    check(orc, o, w_g, w_o, y, z, rows=np.array(rows), what="prefill 4096")


def test_proj_without_y_output(orc):
    """y kept in the workspace (not returned): z is the same."""
    T, H, D, g, d_g, d_model = 8, 16, 128, 4, 128, 256
    o = synth.normal_bf16((T, H, D), 400, "q", DEV)
    w_g, w_o = weights(H, D, g, d_g, d_model, 401)
    _, z1 = run(o, w_g, w_o)
    z2 = torch.empty_like(z1)
    binding.grouped_out_proj(o, w_g, w_o, z2)
    torch.cuda.synchronize()
    assert torch.equal(z1, z2)
