"""Helpers shared by the GPU parity tests (comparison only, no method arithmetic)."""

import numpy as np
import torch

BF16_TOL = 2e-2      # max-abs, bf16 inputs with fp32 accumulation
F32_TOL = 1e-4       # max-abs, the fp32 path


def max_abs(gpu, ref):
    g = gpu.detach().float().cpu().numpy().astype(np.float64)
    r = np.asarray(ref, dtype=np.float64)
    assert g.shape == r.shape, (g.shape, r.shape)
    assert np.all(np.isfinite(g)), "non-finite GPU output"
    return float(np.max(np.abs(g - r))) if g.size else 0.0


def sample_rows(B, Tq, Hq, n, seed, tile=128):
    """Flat row indices (b*Hq + hq)*Tq + i: random rows plus tile edges, the
    first and the last position, spread over every batch and head."""
    rng = np.random.default_rng(seed)
    pos = set(rng.integers(0, Tq, size=n).tolist())
    for e in range(0, Tq, tile):
        pos.update({e, max(0, e - 1)})
    pos.update({0, Tq - 1})
    pos = sorted(p for p in pos if 0 <= p < Tq)
    rows = []
    for k, p in enumerate(pos):
        b = k % B
        hq = (k * 7) % Hq
        rows.append((b * Hq + hq) * Tq + p)
        rows.append((((b + 1) % B) * Hq + (hq + Hq // 2 + 1) % Hq) * Tq + p)
    return np.unique(np.array(rows, dtype=np.int64))


def gather_rows(o, rows, Tq, Hq):
    """o [B, Tq, Hq, d] -> [n, d] at flat row indices (b*Hq + hq)*Tq + i."""
    rows = torch.as_tensor(rows)
    i = rows % Tq
    hq = (rows // Tq) % Hq
    b = rows // (Tq * Hq)
    return o[b.to(o.device), i.to(o.device), hq.to(o.device)]


def gather_lse(lse, rows):
    return lse.reshape(-1)[torch.as_tensor(rows).to(lse.device)]
