"""Helpers shared by the GPU parity tests (tensor <-> oracle array conversion,
tolerance checks).  Holds none of the method's arithmetic."""
import numpy as np
import torch


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
    assert mx <= 2e-2 and rl2 <= 5e-3, f"{what}: max abs {mx:.3e}, rel L2 {rl2:.3e}"
    return mx, rl2
