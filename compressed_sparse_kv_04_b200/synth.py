"""Seeded synthetic inputs shared by the tests, the benchmark and the smoke check.

This module only draws random numbers of the right shapes and distributions;
it contains none of the method's arithmetic.  Every tensor comes from a torch
Generator seeded from the workload seed plus a fixed per-tensor offset, so the
same call gives the same bits on any machine (CPU generator) or on any device
of one kind (CUDA generator).

Distributions (the pages fix none; these are this library's choices):
  token KV / indexer streams  N(0, 1)          -> bfloat16
  pooling w_s                 N(0, 0.02)       fp32 [d]
  pooling b_pos               N(0, 0.1)        fp32 [m]
  query                       N(0, 1)          -> bfloat16 [.., H, D]
  indexer query codes         N(0, 64^2) clipped to +-448, cast to E4M3 (torch cast)
  indexer query scales        U(0.5, 1.5) / 64 fp32
  indexer head weights w_h    U(0, 1)          fp32
  sink logits                 N(0, 1)          fp32 [H]
"""
from __future__ import annotations

import torch

# Per-tensor offsets added to the workload seed.
_OFF = dict(kv_tok=1, idx_tok=2, w_s=3, b_pos=4, w_s_idx=5, b_pos_idx=6, q=7, q_idx=8,
            q_scale=9, w=10, sink=11, gamma=12)


def _gen(seed: int, name: str, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed) * 64 + _OFF[name])
    return g


def normal_bf16(shape, seed, name, device="cpu", std=1.0) -> torch.Tensor:
    g = _gen(seed, name, device)
    out = torch.empty(shape, dtype=torch.bfloat16, device=device)
    # Draw in chunks so very large streams do not need an fp32 copy of the whole.
    flat = out.view(-1)
    n = flat.numel()
    step = 1 << 26
    for s in range(0, n, step):
        e = min(n, s + step)
        flat[s:e] = torch.randn(e - s, generator=g, device=device, dtype=torch.float32).mul_(std)
    return out


def normal_f32(shape, seed, name, std, device="cpu") -> torch.Tensor:
    g = _gen(seed, name, device)
    return torch.randn(shape, generator=g, device=device, dtype=torch.float32) * std


def uniform_f32(shape, seed, name, lo, hi, device="cpu") -> torch.Tensor:
    g = _gen(seed, name, device)
    return torch.rand(shape, generator=g, device=device, dtype=torch.float32) * (hi - lo) + lo


def e4m3_codes(shape, seed, name, device="cpu") -> torch.Tensor:
    """Random E4M3 codes (uint8) from a clipped normal through torch's float8 cast."""
    g = _gen(seed, name, device)
    x = torch.randn(shape, generator=g, device=device, dtype=torch.float32).mul_(64.0)
    x.clamp_(-448.0, 448.0)
    return x.to(torch.float8_e4m3fn).view(torch.uint8)


def pool_params(w, device="cpu", indexer=False):
    """(w_s [dim], b_pos [m + overlap]) for the KV stream, or for the indexer stream."""
    dim = w.D_I if indexer else w.d
    ns, nb = ("w_s_idx", "b_pos_idx") if indexer else ("w_s", "b_pos")
    return (normal_f32((dim,), w.seed, ns, 0.02, device),
            normal_f32((w.m + getattr(w, "overlap", 0),), w.seed, nb, 0.1, device))


def token_streams(w, L_cap=None, device="cpu"):
    """(kv_tok [B, L_cap, d] bf16, idx_tok [B, L_cap, D_I] bf16 or None)."""
    L_cap = L_cap or w.L
    kv = normal_bf16((w.B, L_cap, w.d), w.seed, "kv_tok", device)
    idx = normal_bf16((w.B, L_cap, w.D_I), w.seed, "idx_tok", device) if w.csa else None
    return kv, idx


def queries(w, Q=1, device="cpu"):
    """Query-side inputs for Q queries per sequence.

    Returns dict(q [B,Q,H,D] bf16, q_idx [B,Q,H_I,D_I] u8, q_scale [B,Q,H_I],
    w [B,Q,H_I], sink [H]).
    """
    out = dict(q=normal_bf16((w.B, Q, w.H, w.D), w.seed, "q", device),
               sink=normal_f32((w.H,), w.seed, "sink", 1.0, device))
    if w.csa:
        out["q_idx"] = e4m3_codes((w.B, Q, w.H_I, w.D_I), w.seed, "q_idx", device)
        out["q_scale"] = uniform_f32((w.B, Q, w.H_I), w.seed, "q_scale", 0.5 / 64, 1.5 / 64,
                                     device)
        out["w"] = uniform_f32((w.B, Q, w.H_I), w.seed, "w", 0.0, 1.0, device)
    return out


def gains(dim, seed, device="cpu", spread=0.25):
    """Non-unit RMSNorm gains 1 + U(-spread, spread) for tests of the gain path."""
    return uniform_f32((dim,), seed, "gamma", 1.0 - spread, 1.0 + spread, device)
