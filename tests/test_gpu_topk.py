"""GPU parity of topk_select (exact top-k of indexer scores, ties to the lower
index, NaN lowest, -0 == +0) against the oracle's selection, bit for bit.

Scores are drawn here (seeded numpy) with the structures that stress a radix
select: wide random values, heavy duplicates, values one ulp apart, special
values (+-inf, NaN, signed zeros), constant rows; the visible count n of each
row spans n = 0, n < k, n = k, n = k + 1 and n = N_cap, over capacities that
give one to eight CTAs per row and ragged slices."""
import zlib

import numpy as np
import pytest
import torch

from compressed_sparse_kv_04_b200 import binding

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    binding.lib()


def make_scores(kind, rows, N, rng):
    if kind == "normal":
        s = rng.standard_normal((rows, N)).astype(np.float32) * 3
    elif kind == "dups":
        s = rng.integers(0, 6, (rows, N)).astype(np.float32)
    elif kind == "ulp":  # keys that differ in the lowest bits only
        s = (np.float32(1.5) + rng.integers(0, 4096, (rows, N)).astype(np.float32)
             * np.float32(2.0 ** -22)).astype(np.float32)
    elif kind == "special":
        s = rng.standard_normal((rows, N)).astype(np.float32)
        pick = rng.random((rows, N))
        s[pick < 0.05] = np.nan
        s[(pick >= 0.05) & (pick < 0.08)] = -np.inf
        s[(pick >= 0.08) & (pick < 0.09)] = np.inf
        s[(pick >= 0.09) & (pick < 0.20)] = 0.0
        s[(pick >= 0.20) & (pick < 0.30)] = -0.0
    elif kind == "const":
        s = np.full((rows, N), -2.25, np.float32)
    elif kind == "relu":  # what the indexer gives: many exact zeros, positive tail
        s = np.maximum(rng.standard_normal((rows, N)).astype(np.float32), 0) ** 2
    else:
        raise ValueError(kind)
    return s


def run_topk(scores_np, n_vis, k, m=4):
    rows, N = scores_np.shape
    p = binding.make_params(1, 512, 128, 64, 128, k, 128, 64, m)
    scores = torch.from_numpy(scores_np).to(DEV).reshape(1, rows, N)
    # pos such that (pos + 1) // m == n_vis
    pos = torch.tensor([[n * m - 1 if n > 0 else 0 for n in n_vis]], dtype=torch.int64, device=DEV)
    idx = torch.full((1, rows, k), -7, dtype=torch.int32, device=DEV)
    cnt = torch.full((1, rows), -7, dtype=torch.int32, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    binding.topk_select(p, rows, scores, pos, idx, cnt, dev_status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    nv = (pos.cpu().numpy()[0] + 1) // m
    assert np.array_equal(nv, np.minimum(np.array(n_vis), N))
    return idx.cpu().numpy()[0], cnt.cpu().numpy()[0], nv


def check(orc, scores_np, n_vis, k):
    got_idx, got_cnt, nv = run_topk(scores_np, n_vis, k)
    ridx, rcnt = orc.topk(scores_np.astype(np.float64), nv, k)
    assert np.array_equal(got_cnt, rcnt)
    bad = np.nonzero((got_idx != ridx).any(-1))[0]
    assert bad.size == 0, f"rows {bad[:8]} differ (n={nv[bad[:8]]})"


@pytest.mark.parametrize("N", [1, 1025, 4096, 5000, 32768, 40001, 131072, 262144])
@pytest.mark.parametrize("kind", ["normal", "dups", "ulp", "special", "const", "relu"])
def test_topk_select_structures(orc, N, kind):
    rng = np.random.default_rng(zlib.crc32(f"{N}-{kind}".encode()))
    k = 1024
    ns = sorted({0, 1, min(N, k - 1), min(N, k), min(N, k + 1), N, max(0, N - 1), (N * 2) // 3})
    s = make_scores(kind, len(ns), N, rng)
    check(orc, s, ns, k)


@pytest.mark.parametrize("k", [1, 7, 512, 1000])
def test_topk_select_small_k(orc, k):
    rng = np.random.default_rng(k)
    N = 50000
    ns = [N, N - 13, 3 * k + 1, k + 1, k]
    for kind in ("normal", "dups", "special"):
        check(orc, make_scores(kind, len(ns), N, rng), ns, k)


def test_topk_select_many_rows(orc):
    """More rows than SMs (one CTA per row, no spreading)."""
    rng = np.random.default_rng(5)
    N = 8192
    rows = 300
    ns = list(rng.integers(1000, N + 1, rows))
    check(orc, make_scores("normal", rows, N, rng), ns, 1024)


def test_topk_select_repeated_calls_same_result():
    rng = np.random.default_rng(6)
    s = make_scores("dups", 4, 131072, rng)
    a = run_topk(s, [131072] * 4, 1024)[0]
    b = run_topk(s, [131072] * 4, 1024)[0]
    assert np.array_equal(a, b)
    assert (np.diff(a, axis=-1) > 0).all()


@pytest.mark.parametrize("N", [4096, 32768, 262144])
def test_topk_select_k2048(orc, N):
    """The largest supported k, on the one-CTA-per-row and cluster paths."""
    rng = np.random.default_rng(N + 2048)
    k = 2048
    ns = sorted({min(N, k - 1), min(N, k), min(N, k + 1), N, (N * 2) // 3})
    for kind in ("normal", "dups", "relu"):
        check(orc, make_scores(kind, len(ns), N, rng), ns, k)


def test_topk_select_row_path_boundary(orc):
    """Capacities either side of the largest row the one-CTA kernel holds in
    shared memory, and a ragged capacity (scalar loads)."""
    rng = np.random.default_rng(77)
    for N in (46000, 47000, 48000, 33333):
        ns = [N, N - 1, 5000, 1025]
        check(orc, make_scores("normal", len(ns), N, rng), ns, 1024)
