"""Seeded synthetic inputs for the CSA2 FP4 sparse-decode workloads.

This module is shared by the CUDA path's tests and benchmark and by the
oracle's tests. It holds none of the method's arithmetic: no quantization,
scoring, selection or attention. It only draws random tensors with the
shapes, value distributions and paging structure of the workloads, on any
torch device, deterministically from a seed.

Distributions (the workloads' recipe):
  * attention query q: N(0,1) rounded to bf16, [B, Sq, 16, 576];
  * global KV latent: N(0,1) with 6 of 576 channels (1%, chosen per KV owner
    from the seed) multiplied by 8, rounded to bf16, [B, T, 576]; the long
    context workload adds a per-channel random walk along position,
    d_t = d_{t-1} + N(0, 1e-3^2);
  * indexer query and keys: integers uniform in [-8, 8] stored as E4M3FN
    bytes ([B, Sq, 4, 64] and [B, T, 64]); per-token indexer scale 1.0;
  * indexer head weights: uniform over {1/4, 1/2, 1, 2}, [B, Sq, 4];
  * SWA rows: N(0,1) bf16, [B, 128 + Sq - 1, 576] per layer;
  * page table: identity, or a random permutation of all physical pages.

Random access: the KV latent and indexer keys of one sequence are drawn in
fixed chunks of CHUNK positions, each from its own generator, so any range
can be regenerated without drawing the whole sequence.
"""
from __future__ import annotations

import dataclasses
import hashlib
from typing import Iterator, Optional, Sequence, Tuple

import torch

HEADS = 16          # attention heads of a query token
DIM = 576           # channels of the global KV latent (keys = values)
IDX_HEADS = 4       # indexer heads
IDX_DIM = 64        # indexer channels
WINDOW = 128        # sliding-window length
PAGE = 64           # tokens per KV page
CHUNK = 16384       # positions per generator chunk
N_OUTLIER = 6       # 1% of 576 channels
OUTLIER_GAIN = 8.0
DRIFT_STD = 1e-3
HEAD_WEIGHTS = (0.25, 0.5, 1.0, 2.0)


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic decode workload.

    modes: per-layer static mode, "F" (Full), "R" (Reindex) or "U" (Reuse).
    seq_lens: optional per-sequence context lengths (ragged batches); when
    absent every sequence has `context` entries. A length counts every cached
    global entry of the sequence, including its Sq newest (query) tokens.
    """
    name: str
    batch: int
    q_tokens: int
    context: int
    top_k: int
    modes: Tuple[str, ...] = ("F",)
    random_pages: bool = False
    drift: bool = False
    seed: int = 0
    seq_lens: Optional[Tuple[int, ...]] = None

    def lens(self) -> Tuple[int, ...]:
        if self.seq_lens is not None:
            assert len(self.seq_lens) == self.batch
            return tuple(self.seq_lens)
        return (self.context,) * self.batch

    @property
    def max_len(self) -> int:
        return max(self.lens())

    @property
    def pages_per_seq(self) -> int:
        return -(-self.max_len // PAGE)

    @property
    def owners(self) -> Tuple[int, ...]:
        return tuple(i for i, m in enumerate(self.modes) if m == "F")


# The five workloads the benchmark and the parity tests run.
WORKLOADS = {
    "full_b1_t4k": Workload("full_b1_t4k", 1, 1, 4096, 512, ("F",), False, False, 0),
    "fru_b8_t16k": Workload("fru_b8_t16k", 8, 1, 16384, 1024, ("F", "R", "U"), False, False, 1),
    "decode_b64_t128k": Workload("decode_b64_t128k", 64, 1, 131072, 2048, ("F",), True, False, 2),
    "verify_b32_sq4_t32k": Workload("verify_b32_sq4_t32k", 32, 4, 32768, 2048,
                                    ("F", "U", "R", "U", "F", "U"), False, False, 3),
    "long_b4_t1m": Workload("long_b4_t1m", 4, 1, 1048576, 2048, ("F",), True, True, 4),
}

# A quarter-batch copy of the 128K decode workload (same per-sequence shape,
# indexer keys still > L2) for profiler captures that must stay small.
PROFILE_WORKLOADS = {
    "decode_b16_t128k": Workload("decode_b16_t128k", 16, 1, 131072, 2048, ("F",), True, False, 2),
}


def _seed(*parts) -> int:
    h = hashlib.sha256(repr(parts).encode()).digest()
    return int.from_bytes(h[:8], "little") & ((1 << 63) - 1)


def generator(device, *parts) -> torch.Generator:
    g = torch.Generator(device=torch.device(device))
    g.manual_seed(_seed(*parts))
    return g


def outlier_channels(wl: Workload, owner: int) -> torch.Tensor:
    """The 6 channels scaled by 8 in the KV latent of one owner (CPU int64)."""
    g = generator("cpu", wl.seed, "outliers", owner)
    return torch.randperm(DIM, generator=g)[:N_OUTLIER]


def _kv_chunk_f32(wl: Workload, owner: int, b: int, c: int, device) -> torch.Tensor:
    g = generator(device, wl.seed, "kv", owner, b, c)
    x = torch.randn(CHUNK, DIM, generator=g, device=device, dtype=torch.float32)
    gain = torch.ones(DIM, device=device)
    gain[outlier_channels(wl, owner).to(device)] = OUTLIER_GAIN
    return x * gain


def _drift_increments(wl: Workload, owner: int, b: int, c: int, device) -> torch.Tensor:
    g = generator(device, wl.seed, "drift", owner, b, c)
    return torch.randn(CHUNK, DIM, generator=g, device=device, dtype=torch.float32) * DRIFT_STD


def kv_chunks(wl: Workload, owner: int, b: int, device, t_end: Optional[int] = None
              ) -> Iterator[Tuple[int, torch.Tensor]]:
    """Yield (t0, bf16 rows [n, 576]) covering positions [0, t_end) in order."""
    t_end = wl.lens()[b] if t_end is None else t_end
    carry = torch.zeros(DIM, device=device, dtype=torch.float32)
    for c in range(-(-t_end // CHUNK)):
        x = _kv_chunk_f32(wl, owner, b, c, device)
        if wl.drift:
            d = torch.cumsum(_drift_increments(wl, owner, b, c, device), dim=0) + carry
            carry = d[-1].clone()
            x = x + d
        t0 = c * CHUNK
        n = min(CHUNK, t_end - t0)
        yield t0, x[:n].to(torch.bfloat16)


def kv_rows(wl: Workload, owner: int, b: int, positions: torch.Tensor, device) -> torch.Tensor:
    """bf16 KV latent rows of sequence b at the given positions, [len, 576]."""
    positions = positions.to("cpu", torch.int64)
    out = torch.empty(len(positions), DIM, dtype=torch.bfloat16, device=device)
    if len(positions) == 0:
        return out
    chunks = torch.unique(positions // CHUNK).tolist()
    carry = torch.zeros(DIM, device=device, dtype=torch.float32)
    last = -1
    for c in chunks:
        if wl.drift:
            for cc in range(last + 1, c):
                carry = carry + _drift_increments(wl, owner, b, cc, device).sum(0)
        x = _kv_chunk_f32(wl, owner, b, c, device)
        if wl.drift:
            d = torch.cumsum(_drift_increments(wl, owner, b, c, device), dim=0) + carry
            carry = d[-1].clone()
            x = x + d
        last = c
        sel = (positions // CHUNK) == c
        local = (positions[sel] - c * CHUNK).to(device)
        out[sel.to(device)] = x[local].to(torch.bfloat16)
    return out


def _small_int_e4m3(shape, g: torch.Generator, device) -> torch.Tensor:
    v = torch.randint(-8, 9, shape, generator=g, device=device, dtype=torch.int32)
    return v.to(torch.float32).to(torch.float8_e4m3fn).view(torch.uint8)


def kidx_chunk(wl: Workload, owner: int, b: int, c: int, device) -> torch.Tensor:
    g = generator(device, wl.seed, "kidx", owner, b, c)
    return _small_int_e4m3((CHUNK, IDX_DIM), g, device)


def kidx_rows(wl: Workload, owner: int, b: int, t0: int, t1: int, device) -> torch.Tensor:
    """Indexer keys (E4M3FN bytes) of sequence b for positions [t0, t1)."""
    parts = []
    for c in range(t0 // CHUNK, -(-t1 // CHUNK)):
        lo = max(t0, c * CHUNK) - c * CHUNK
        hi = min(t1, (c + 1) * CHUNK) - c * CHUNK
        parts.append(kidx_chunk(wl, owner, b, c, device)[lo:hi])
    if not parts:
        return torch.empty(0, IDX_DIM, dtype=torch.uint8, device=device)
    return torch.cat(parts)


def kidx_scale_rows(wl: Workload, owner: int, b: int, t0: int, t1: int, device) -> torch.Tensor:
    """Per-token indexer scale sigma for positions [t0, t1) (1.0 here)."""
    return torch.ones(t1 - t0, dtype=torch.float32, device=device)


def attn_query(wl: Workload, layer: int, device) -> torch.Tensor:
    g = generator(device, wl.seed, "q", layer)
    return torch.randn(wl.batch, wl.q_tokens, HEADS, DIM, generator=g, device=device
                       ).to(torch.bfloat16)


def swa_rows(wl: Workload, layer: int, device) -> torch.Tensor:
    """Per-layer SWA window [B, 128 + Sq - 1, 576]; row r of sequence b holds
    position len_b - (128 + Sq - 1) + r (rows at negative positions unused)."""
    g = generator(device, wl.seed, "swa", layer)
    return torch.randn(wl.batch, WINDOW + wl.q_tokens - 1, DIM, generator=g, device=device
                       ).to(torch.bfloat16)


def idx_query(wl: Workload, layer: int, device) -> torch.Tensor:
    g = generator(device, wl.seed, "qidx", layer)
    return _small_int_e4m3((wl.batch, wl.q_tokens, IDX_HEADS, IDX_DIM), g, device)


def idx_weights(wl: Workload, layer: int, device) -> torch.Tensor:
    g = generator(device, wl.seed, "w", layer)
    pick = torch.randint(0, len(HEAD_WEIGHTS), (wl.batch, wl.q_tokens, IDX_HEADS),
                         generator=g, device=device)
    return torch.tensor(HEAD_WEIGHTS, device=device, dtype=torch.float32)[pick]


def page_table(wl: Workload, device) -> torch.Tensor:
    """int32 [B, pages_per_seq]: physical page of each logical page."""
    n = wl.batch * wl.pages_per_seq
    if wl.random_pages:
        g = generator("cpu", wl.seed, "pages")
        perm = torch.randperm(n, generator=g)
    else:
        perm = torch.arange(n)
    return perm.view(wl.batch, wl.pages_per_seq).to(torch.int32).to(device)


def seq_lens(wl: Workload, device) -> torch.Tensor:
    return torch.tensor(wl.lens(), dtype=torch.int32, device=device)


def small_workload(name: str, batch: int, q_tokens: int, lens: Sequence[int], top_k: int,
                   modes=("F",), random_pages=True, drift=False, seed=123) -> Workload:
    """A ragged workload small enough for the oracle to check every output."""
    return Workload(name, batch, q_tokens, max(lens), top_k, tuple(modes), random_pages,
                    drift, seed, tuple(int(x) for x in lens))
