"""Comparison rules shared by the GPU parity tests.

Tolerances (bf16 outputs against the fp64 oracle, real rows only):
  max |gpu - oracle| <= 2e-2 and mean |gpu - oracle| <= 2e-3, and the RMS of
  the error <= 1e-2 of the oracle's RMS (a tighter check: with N(0,1) inputs
  the outputs are small, so the absolute bounds alone are weak).
Indices: bit-exact, except that a top-k set may differ from the oracle's only
in KV blocks whose oracle logit lies within 1e-3 of the oracle's k-th largest
logit (a near-tie that fp32 summation order may resolve either way).
"""
from __future__ import annotations

import numpy as np
import torch

MAX_ABS = 2e-2
MEAN_ABS = 2e-3
REL_RMS = 1e-2
TIE_GAP = 1e-3
BLOCK = 64


def to_np(t: torch.Tensor) -> np.ndarray:
    t = t.detach().cpu()
    if t.dtype == torch.bfloat16:
        t = t.float()
    return t.numpy()


def real_rows(sizes) -> np.ndarray:
    return np.concatenate([np.arange(BLOCK * j, BLOCK * j + m) for j, m in enumerate(sizes)])


def error_stats(got, want) -> dict:
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    err = np.abs(got - want)
    rms_w = np.sqrt(np.mean(want ** 2)) if want.size else 0.0
    rms_e = np.sqrt(np.mean(err ** 2)) if err.size else 0.0
    return dict(max_abs=float(err.max(initial=0.0)), mean_abs=float(err.mean()) if err.size else 0.0,
                rel_rms=float(rms_e / rms_w) if rms_w > 0 else float(rms_e))


def assert_outputs_close(got, want, what="output", rel_rms=REL_RMS):
    st = error_stats(got, want)
    assert st["max_abs"] <= MAX_ABS, f"{what}: max abs {st['max_abs']:.3e} > {MAX_ABS}"
    assert st["mean_abs"] <= MEAN_ABS, f"{what}: mean abs {st['mean_abs']:.3e} > {MEAN_ABS}"
    assert st["rel_rms"] <= rel_rms, f"{what}: relative RMS {st['rel_rms']:.3e} > {rel_rms}"
    return st


def check_topk(gpu_idx, gpu_num, scores, topk: int):
    """GPU selection against the oracle's fp64 coarse logits.

    gpu_idx [B,H,nq,stride] int32, gpu_num [B,H,nq]; scores [B,H,nq,nkv] fp64.
    Returns the number of rows whose set differs from the oracle's (each such
    difference being a near-tie)."""
    gpu_idx = np.asarray(gpu_idx)
    gpu_num = np.asarray(gpu_num)
    B, H, nq, nkv = scores.shape
    k = min(topk, nkv)
    assert np.all(gpu_num == k), "q2k_num must equal min(topk, n_kv_blocks)"
    assert np.all(gpu_idx[..., k:] == -1), "entries past q2k_num must be -1"
    sel = gpu_idx[..., :k]
    assert np.all(np.diff(sel, axis=-1) > 0), "each q2k_idx row must be strictly ascending"
    assert sel.min() >= 0 and sel.max() < nkv
    differing = 0
    cols = np.arange(nkv)
    for b in range(B):
        for h in range(H):
            for a in range(nq):
                row = scores[b, h, a]
                order = np.lexsort((cols, -row))
                want = set(order[:k].tolist())
                got = set(sel[b, h, a].tolist())
                if got != want:
                    differing += 1
                    tau = row[order[k - 1]]
                    for j in got ^ want:
                        assert abs(row[j] - tau) < TIE_GAP, (
                            f"(b={b},h={h},a={a}) block {j} logit {row[j]:.6g} vs k-th {tau:.6g}")
    return differing
