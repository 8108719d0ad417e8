"""Helpers shared by the GPU parity tests (tensor <-> oracle array conversion,
tolerance checks).  Holds none of the method's arithmetic."""
import math

import numpy as np
import torch


# Largest errors seen by the checks below in this test session (printed in
# the terminal summary, so every GPU run reports its measured margins).
MAX_ERR = {}


def _record(key, value):
    if np.isfinite(value):
        MAX_ERR[key] = max(MAX_ERR.get(key, 0.0), float(value))


def bits16(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor (any device) -> numpy uint16 storage bits."""
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def bits8(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().view(torch.uint8).cpu().numpy()


def f32(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy()


def bf16_values(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def assert_bf16_storage_close(got_bits, ref_vals, what=""):
    """|gpu - oracle| <= 2^-8 |x| + 1e-3: one bf16 ulp of storage rounding plus
    fp32 accumulation, on values the oracle computes in fp64."""
    got = torch.from_numpy(np.ascontiguousarray(got_bits).view(np.int16)).view(torch.bfloat16)
    got = got.double().numpy()
    err = np.abs(got - ref_vals)
    bound = np.abs(ref_vals) * 2.0 ** -8 + 1e-3
    bad = err > bound
    assert not bad.any(), f"{what}: {bad.sum()} elements out of tolerance, max err {err.max():.3e}"


def attention_errors(got: np.ndarray, ref: np.ndarray):
    """(max abs error, relative L2 error)."""
    d = got.astype(np.float64) - ref.astype(np.float64)
    return float(np.abs(d).max()), float(np.linalg.norm(d) / max(np.linalg.norm(ref), 1e-30))


def assert_attention_close(got: np.ndarray, ref: np.ndarray, what=""):
    """The attention tolerance: max-abs <= 2e-2 and relative L2 <= 5e-3."""
    mx, rl2 = attention_errors(got, ref)
    _record("attn_max_abs", mx)
    _record("attn_rel_l2", rl2)
    assert mx <= 2e-2 and rl2 <= 5e-3, f"{what}: max abs {mx:.3e}, rel L2 {rl2:.3e}"
    return mx, rl2


# Log-sum-exp tolerance, per (row, head).  The tensor cores see the
# normalised (and rotated) query rounded to bf16, qhat_d (1 + e_d) with
# |e_d| <= 2^-8 (standard deviation about 2^-8/sqrt(3) = 2.3e-3), and a
# window token's key, when the kernel rescales or rotates it in bf16, rounded
# the same way.  The log-sum-exp moves by the attention-weighted mean of the
# logit errors: for the query part
#     dLSE = scale * sum_d e_d qhat_d obar_d,   obar = sum_j p_j v_j,
# where p_j are the softmax weights (sink included) and obar is the output
# before its inverse rotation, so |obar| = |o| for the head's output o.  With
# |qhat_d| ~ 1 its standard deviation is about 2.3e-3 * scale * |o|; the key
# part is at most as large again.  The bound is five standard deviations of
# the two together, 5 * sqrt(2) * 2.3e-3 * scale * |o|, plus 1e-4 for the fp32
# accumulation.  A head that attends to one key (|o| ~ sqrt(D)) gets about
# 1.6e-2 at scale 1/sqrt(D); one that spreads over ~1000 keys, about 1e-3.
LSE_SIGMA = 2.3e-3


def lse_tolerance(out_ref, scale):
    """Per-(row, head) LSE bound from the oracle's output [..., H, D]."""
    o = np.linalg.norm(np.asarray(out_ref, np.float64), axis=-1)
    return 5.0 * math.sqrt(2.0) * LSE_SIGMA * scale * o + 1e-4


def assert_lse_close(got, ref, out_ref, what="", scale=None):
    """LSE [..., H] against the oracle's, within lse_tolerance of the oracle's
    output out_ref [..., H, D]; scale is the logit scale (1/sqrt(D) when
    None)."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    if scale is None:
        scale = 1.0 / math.sqrt(np.asarray(out_ref).shape[-1])
    fin = np.isfinite(ref)
    assert np.array_equal(np.isfinite(got), fin), f"{what}: non-finite pattern differs"
    assert np.array_equal(got[~fin], ref[~fin]), f"{what}: infinite values differ"
    if not fin.any():
        return 0.0
    tol = lse_tolerance(out_ref, scale)
    err = np.abs(got - ref)
    _record("lse_abs", float(err[fin].max()))
    _record("lse_over_bound", float((err[fin] / tol[fin]).max()))
    bad = fin & (err > tol)
    assert not bad.any(), (f"{what}: {bad.sum()} LSE values out of tolerance, max error "
                           f"{err[fin].max():.3e}, largest error/bound "
                           f"{(err[fin] / tol[fin]).max():.2f}")
    return float(err[fin].max())
