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
# normalised, rotated query rounded to bf16, qhat_d (1 + e_d) with
# |e_d| <= 2^-8, and every logit of the head shares that rounding.  To first
# order the log-sum-exp moves by the softmax-weighted mean of the logit
# errors,
#     dLSE = scale * sum_d e_d qhat_d obar_d,    obar = sum_j p_j v_j,
# the head's output before its inverse rotation (p_j: the weights, sink
# included), so |dLSE| <= 2^-8 scale sum_d |qhat_d obar_d|
#                       <= 2^-8 scale |qhat| |o|      (Cauchy-Schwarz; the
# rotation keeps the norm, |obar| = |o|).  Window rows that the kernel
# rescales or rotates in bf16 add a key-side rounding of the same order, so
# the bound is doubled; 1e-4 covers the fp32 accumulation.  |qhat| = sqrt(D)
# for a unit gain (qnorm_gain scales it for other gains).  On the 128K decode
# shape the measured errors stay below 0.4 of the query term alone.
def lse_tolerance(out_ref, scale, qnorm_gain=1.0):
    """Per-(row, head) LSE bound from the oracle's output [..., H, D]."""
    o = np.linalg.norm(np.asarray(out_ref, np.float64), axis=-1)
    D = np.asarray(out_ref).shape[-1]
    return 2.0 * 2.0 ** -8 * scale * math.sqrt(D) * qnorm_gain * o + 1e-4


def assert_lse_close(got, ref, out_ref, what="", scale=None, qnorm_gain=1.0):
    """LSE [..., H] against the oracle's, within lse_tolerance of the oracle's
    output out_ref [..., H, D]; scale is the logit scale (1/sqrt(D) when
    None); qnorm_gain the largest query gain (1 without gains)."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    if scale is None:
        scale = 1.0 / math.sqrt(np.asarray(out_ref).shape[-1])
    fin = np.isfinite(ref)
    assert np.array_equal(np.isfinite(got), fin), f"{what}: non-finite pattern differs"
    assert np.array_equal(got[~fin], ref[~fin]), f"{what}: infinite values differ"
    if not fin.any():
        return 0.0
    tol = lse_tolerance(out_ref, scale, qnorm_gain)
    err = np.abs(got - ref)
    _record("lse_abs", float(err[fin].max()))
    _record("lse_over_bound", float((err[fin] / tol[fin]).max()))
    bad = fin & (err > tol)
    assert not bad.any(), (f"{what}: {bad.sum()} LSE values out of tolerance, max error "
                           f"{err[fin].max():.3e}, largest error/bound "
                           f"{(err[fin] / tol[fin]).max():.2f}")
    return float(err[fin].max())
