"""Shared parity helpers: tolerances and row sampling (test infrastructure).

Tolerances (GPU result vs the fp64 oracle on the same stored inputs):
  * attention output (bf16 / fp16 / fp32 stored): max |err| <= 2e-2 and
    mean |err| <= 2e-3;
  * fp32 lse: |err| <= 1e-3 * max(1, |lse_ref|) (relative error, with the
    reference magnitude floored at 1 so rows whose lse is near 0 are measured
    on the absolute scale).
"""
import numpy as np
import torch

MAX_ABS = 2e-2
MEAN_ABS = 2e-3
LSE_REL = 1e-3


def check_out(got: torch.Tensor, ref: np.ndarray, what: str = "out"):
    g = got.detach().float().cpu().double().numpy().reshape(ref.shape)
    assert np.isfinite(g).all(), f"{what}: non-finite values in the GPU result"
    err = np.abs(g - ref)
    mx, mean = float(err.max(initial=0.0)), float(err.mean()) if err.size else 0.0
    assert mx <= MAX_ABS, f"{what}: max abs err {mx:.3e} > {MAX_ABS}"
    assert mean <= MEAN_ABS, f"{what}: mean abs err {mean:.3e} > {MEAN_ABS}"
    return mx, mean


def check_lse(got: torch.Tensor, ref: np.ndarray, what: str = "lse"):
    g = got.detach().float().cpu().double().numpy().reshape(ref.shape)
    assert np.isfinite(g).all(), f"{what}: non-finite values in the GPU lse"
    rel = np.abs(g - ref) / np.maximum(1.0, np.abs(ref))
    mx = float(rel.max(initial=0.0))
    assert mx <= LSE_REL, f"{what}: lse rel err {mx:.3e} > {LSE_REL}"
    return mx


def sample_rows(seq_len, heads, n, seed=0):
    """Flattened (token*heads + head) rows: every sequence's first and last row, plus random ones."""
    rng = np.random.Generator(np.random.PCG64(seed))
    cu = np.concatenate([[0], np.cumsum(seq_len)])
    total = int(cu[-1])
    rows = set()
    for b in range(len(seq_len)):
        if seq_len[b] == 0:
            continue
        for t in (cu[b], cu[b + 1] - 1, min(cu[b] + 127, cu[b + 1] - 1), min(cu[b] + 128, cu[b + 1] - 1)):
            rows.add(int(t) * heads + int(rng.integers(heads)))
    while len(rows) < n and total > 0:
        rows.add(int(rng.integers(total)) * heads + int(rng.integers(heads)))
    return np.array(sorted(rows), dtype=np.int64)
