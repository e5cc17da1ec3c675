"""Helpers for the GPU parity tests: tolerances and element-wise comparison
with the fp64 oracle."""
from __future__ import annotations

import numpy as np
import torch

# max-abs tolerances on the output: 2e-2 for bf16 inputs, 5e-3 for fp32 inputs
# (TF32 tensor-core products); plus a relative L2 bound that still bites
# where the outputs are small (near-uniform softmax over long rows).
# fp16 (no stated bound): the products are exact and accumulate in fp32; P
# and the output are rounded to fp16 (relative 2^-11 each), so with |v| and
# |out| below ~5 each rounding moves an output by at most ~2.5e-3: 5e-3.
MAX_ABS = {torch.bfloat16: 2e-2, torch.float32: 5e-3, torch.float16: 5e-3}
REL_L2 = 1e-2


def compare(got: torch.Tensor, ref: np.ndarray, dtype: torch.dtype, what: str = ""):
    g = got.detach().float().cpu().numpy().astype(np.float64)
    assert g.shape == ref.shape, f"{what}: shape {g.shape} vs {ref.shape}"
    assert np.all(np.isfinite(g)), f"{what}: non-finite output"
    err = np.abs(g - ref)
    max_abs = float(err.max()) if err.size else 0.0
    den = float(np.linalg.norm(ref))
    rel = float(np.linalg.norm(g - ref) / den) if den > 0 else float(np.linalg.norm(g))
    assert max_abs <= MAX_ABS[dtype], f"{what}: max-abs {max_abs:.3e} > {MAX_ABS[dtype]}"
    if den > 0:
        assert rel <= REL_L2, f"{what}: relative L2 {rel:.3e} > {REL_L2}"
    return max_abs, rel


def sample_rows(n_seq: int, heads, lens, per: int, seed: int = 7):
    """Rows (sequence, head, row) checked on the large workloads: the tile
    edges {0, 1, 127, 128, 129, L-2, L-1} plus `per` random rows, for every
    listed head of every sequence."""
    rng = np.random.default_rng(seed)
    rows = []
    for b in range(n_seq):
        L = int(lens[b])
        if L == 0:
            continue
        fixed = {r for r in (0, 1, 127, 128, 129, L - 2, L - 1) if 0 <= r < L}
        for h in heads:
            pick = set(fixed) | set(rng.integers(0, L, size=per).tolist())
            rows += [(b, h, r) for r in sorted(pick)]
    return np.array(rows, dtype=np.int64)
