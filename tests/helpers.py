"""Shared helpers for the parity tests: run the CUDA path through the C ABI
and compare it with the fp64 oracle under one tolerance.

Tolerance (elementwise): |gpu - oracle| <= 1e-2 + 1e-2 * |oracle| for the
output and |gpu_lse - oracle_lse| <= 1e-3 for the log-sum-exp (rows with
no visible key must give exactly 0 and -inf).  Because long-context outputs
are small averages (|O| ~ 0.02-0.05) the absolute term alone would admit
gross errors, so the relative Frobenius error ||gpu - oracle|| / ||oracle||
over everything compared must also stay within 1e-2 (bf16 rounding of P and
of the output contribute about 3e-3).
"""
from __future__ import annotations

import numpy as np
import torch

ATOL, RTOL, LSE_TOL, REL_FRO = 1e-2, 1e-2, 1e-3, 1e-2


def to_device(inp: dict, device="cuda") -> dict:
    d = {"skv": inp["skv"].to(device), "max_skv": inp["max_skv"], "q": inp["q"].to(device)}
    if "cache" in inp:
        cache = inp["cache"].to(device)
        B, S, dk = cache.shape
        d["cache"] = cache
        d["k"] = cache.view(B, 1, S, dk)
        d["v"] = cache.view(B, 1, S, dk)[..., : inp["v"].shape[-1]]
    else:
        d["k"] = inp["k"].to(device)
        d["v"] = inp["v"].to(device)
    return d


def run_gpu(w, dev: dict, causal=None):
    from attention_mqa_gqa_b200 import binding

    out, lse = binding.attention(dev["q"], dev["k"], dev["v"], dev["skv"], dev["max_skv"],
                                 w.scale, w.causal if causal is None else causal)
    torch.cuda.synchronize()
    assert binding.last_device_error() == binding.ATTN_OK
    return out, lse


def oracle_full(w, inp: dict, causal=None):
    from oracle import c_oracle

    return c_oracle.attention_fwd(inp["q"], inp["k"], inp["v"], inp["skv"].tolist(), w.scale,
                                  w.causal if causal is None else causal)


def compare(out_gpu, lse_gpu, ref_o, ref_l, what=""):
    """Assert the tolerance; return (max_abs_err, max_lse_err, rel_frobenius)."""
    o = out_gpu.detach().float().cpu().numpy().astype(np.float64)
    l = lse_gpu.detach().cpu().numpy().astype(np.float64) if lse_gpu is not None else None
    ref_o = np.asarray(ref_o, dtype=np.float64)
    err = np.abs(o - ref_o)
    bound = ATOL + RTOL * np.abs(ref_o)
    bad = err > bound
    assert not np.isnan(o).any(), f"{what}: NaN in output"
    assert not bad.any(), (f"{what}: {bad.sum()} / {bad.size} outputs out of tolerance; "
                           f"max err {err.max():.3e} at {np.unravel_index(err.argmax(), err.shape)}")
    lerr = 0.0
    if l is not None:
        ref_l = np.asarray(ref_l, dtype=np.float64)
        empty = np.isneginf(ref_l)
        assert (np.isneginf(l) == empty).all(), f"{what}: -inf LSE mismatch"
        if (~empty).any():
            lerr = float(np.abs(l[~empty] - ref_l[~empty]).max())
            assert lerr <= LSE_TOL, f"{what}: LSE error {lerr:.3e}"
        assert (o[empty] == 0).all(), f"{what}: rows with no visible key must be 0"
    den = np.linalg.norm(ref_o)
    rel = float(np.linalg.norm(o - ref_o) / den) if den > 0 else 0.0
    assert rel <= REL_FRO, f"{what}: relative Frobenius error {rel:.3e}"
    return float(err.max()), lerr, rel
