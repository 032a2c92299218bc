"""Inputs of the indexer FP8 quantiser where rounding decisions are close
(shared by the oracle pins and the GPU parity tests). No method arithmetic:
only a search over bf16 values for rows with a given property."""
from fractions import Fraction

import numpy as np
import torch


def _finite_positive_bf16() -> np.ndarray:
    bits = np.arange(65536, dtype=np.uint32)
    vals = (bits << 16).view(np.float32)
    return vals[np.isfinite(vals) & (vals > 0)]


def _e4m3_midpoints() -> np.ndarray:
    ev = torch.arange(127, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    return np.unique(((ev[:-1] + ev[1:]) / 2).astype(np.float32))


def _to_bf16_bits(x: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.ascontiguousarray(x, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def double_rounding_rows(n_rows: int, seed: int) -> np.ndarray:
    """bf16 rows (as bits) whose row maximum fixes sigma and whose other
    channels x make the binary32 quotient RN(x / sigma) land exactly on an
    E4M3 midpoint while the exact quotient does not: the inputs on which
    rounding the exact quotient and rounding the binary32 quotient differ.
    Found by a vectorised search over every positive bf16 value."""
    mids = _e4m3_midpoints()
    pos = _finite_positive_bf16()
    rng = np.random.default_rng(seed)
    rows = []
    while len(rows) < n_rows:
        amax = np.float32(rng.choice(pos[(pos > 1e-30) & (pos < 1e30)]))
        sg = amax / np.float32(448.0)
        xs = pos[pos < amax]
        q = xs / sg
        hit = xs[np.isin(q, mids)]
        hit = [x for x in hit if Fraction(float(x)) / Fraction(float(sg)) != Fraction(float(x / sg))]
        if not hit:
            continue
        take = np.array(hit[:63], np.float32)
        row = np.zeros(64, np.float32)
        row[0] = amax
        row[1:1 + len(take)] = take * np.where(np.arange(len(take)) % 2 == 0, 1, -1)
        rows.append(row)
    return _to_bf16_bits(np.array(rows))
