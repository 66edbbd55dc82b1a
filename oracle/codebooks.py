"""Code tables of the double-quantised NF4 format (oracle; test infrastructure only).

Source for what the tables are: "Soup 层流式 NF4 训练实测：在 4 GB 显存上以位级一致标准完成 8B 模型 LoRA 微调"
(m.mzlw.cn), §2.4 -- the NF4 code table holds 16 fp32 values, the nested
(absmax) code table 256 fp32 values, both constant for every weight, which is
why one resident copy is shared.  The pages print neither table, so the
values follow the published constructions:

* NF4 (QLoRA, Dettmers et al. 2023, §3 "4-bit NormalFloat"): quantiles of
  N(0, 1) taken asymmetrically so that 0 is exact -- 8 positive quantiles at
  probabilities spaced evenly from delta down towards 1/2 (1/2 excluded), 7
  negative ones spaced the same way over 7 steps, plus an exact 0, all divided
  by the largest, so the table runs from exactly -1 to exactly +1.
  delta = ((1 - 1/30) + (1 - 1/32)) / 2.  Computed in float64, rounded once
  to fp32.  The normal quantile function is scipy's ``ndtri`` (a library
  primitive).
* Nested 8-bit table: signed dynamic ("tree") quantisation of Dettmers 2016,
  "8-Bit Approximations for Parallelism in Deep Learning": one sign, a decimal
  exponent level i = 0..6 (scale 10^(i-6)), and at level i the 2^i midpoints
  of an even split of [0.1, 1] into 2^i intervals; plus 0 and 1.  That is
  2 * (1 + 2 + ... + 64) + 2 = 256 values, max magnitude 1.  Computed in
  float64, rounded once to fp32, sorted ascending.

Nearest-entry rule (a reading; the pages do not state one): midpoints
m_j = fp32(exact (c_j + c_{j+1}) / 2); a value u maps to the number of
midpoints strictly below it, so u > m_j selects the upper entry and an exact
tie goes to the lower index.
"""
from __future__ import annotations

import numpy as np
from scipy.special import ndtri

NF4_DELTA = 0.5 * ((1.0 - 1.0 / 30.0) + (1.0 - 1.0 / 32.0))
DECADES = (1e-6, 1e-5, 1e-4, 1e-3, 1e-2, 1e-1, 1.0)


def _even_points(start: float, stop: float, n: int) -> list[float]:
    """start + i * ((stop - start) / n) for i = 0..n-1 (stop itself excluded)."""
    step = (stop - start) / n
    return [start + i * step for i in range(n)]


def nf4_table() -> np.ndarray:
    """16 fp32 NF4 values, ascending, with an exact 0 at index 7."""
    pos = [float(ndtri(p)) for p in _even_points(NF4_DELTA, 0.5, 8)]
    neg = [-float(ndtri(p)) for p in _even_points(NF4_DELTA, 0.5, 7)]
    top = pos[0]
    vals = sorted([v / top for v in pos] + [0.0] + [v / top for v in neg])
    return np.array(vals, dtype=np.float64).astype(np.float32)


def code8_table() -> np.ndarray:
    """256 fp32 values of the signed dynamic tree map, ascending."""
    vals = [0.0, 1.0]
    for i, scale in enumerate(DECADES):
        n = 2 ** i
        step = 0.9 / n
        bounds = [0.1 + j * step for j in range(n + 1)]
        for j in range(n):
            mid = (bounds[j] + bounds[j + 1]) / 2.0
            vals.append(scale * mid)
            vals.append(-scale * mid)
    assert len(vals) == 256
    return np.array(sorted(vals), dtype=np.float64).astype(np.float32)


def midpoints(table: np.ndarray) -> np.ndarray:
    """fp32 midpoints between neighbouring entries (exact mean, one rounding)."""
    t = table.astype(np.float64)
    return ((t[:-1] + t[1:]) / 2.0).astype(np.float32)


def nearest_index(u: np.ndarray, table: np.ndarray) -> np.ndarray:
    """Index of the entry nearest to fp32 ``u`` under the midpoint rule."""
    mids = midpoints(table)
    return np.searchsorted(mids, np.asarray(u, dtype=np.float32), side="left").astype(np.int64)


def zero_index(table: np.ndarray) -> int:
    idx = np.nonzero(table == 0.0)[0]
    assert idx.size == 1
    return int(idx[0])


def fnv1a64(data: bytes) -> int:
    h = 0xCBF29CE484222325
    for b in data:
        h ^= b
        h = (h * 0x100000001B3) & 0xFFFFFFFFFFFFFFFF
    return h


def codebook_hash() -> int:
    """FNV-1a 64 over the little-endian fp32 bytes of the NF4 table, then the 8-bit table."""
    return fnv1a64(nf4_table().astype("<f4").tobytes() + code8_table().astype("<f4").tobytes())
