"""Helpers shared by the GPU parity tests (tensor <-> oracle array conversion,
tolerance checks).  Holds none of the method's arithmetic."""
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


# Log-sum-exp tolerance at the plain logit scale 1/sqrt(D).  The tensor cores
# see the normalised (and rotated) query rounded to bf16, qhat_d (1 + e_d)
# with |e_d| <= 2^-8.  Every key shares that rounding, so the log-sum-exp
# moves by the attention-weighted mean of the logit errors,
#     dLSE = scale * sum_d e_d qhat_d vbar_d,   vbar = sum_j p_j v_j,
# whose standard deviation is about 2^-8/sqrt(3) * |qhat| |vbar| / sqrt(D)
# = 2.3e-3 * |vbar| / sqrt(D) for |qhat| = sqrt(D).  |vbar| <= sqrt(D) (one
# dominant key, the worst case: 2.3e-3), and it is far smaller when the
# attention spreads over many keys.  5e-3 is two standard deviations of that
# worst case; at the test data's near-uniform attention it is a wide margin.
# A larger logit scale (YaRN's gain) scales the bound with it.
LSE_ATOL = 5e-3


def assert_lse_close(got, ref, what="", scale_gain=1.0):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    fin = np.isfinite(ref)
    assert np.array_equal(np.isfinite(got), fin), f"{what}: non-finite pattern differs"
    assert np.array_equal(got[~fin], ref[~fin]), f"{what}: infinite values differ"
    if not fin.any():
        return 0.0
    err = float(np.abs(got[fin] - ref[fin]).max())
    _record("lse_abs", err / scale_gain)
    assert err <= LSE_ATOL * scale_gain, f"{what}: max LSE error {err:.3e}"
    return err
