"""Seeded synthetic inputs for sink attention.

This module only draws random numbers and rounds them to bf16; it holds none
of the attention arithmetic.  The same arrays feed the CUDA path and the fp64
oracle, so both see identical bf16 bits.

Generator: numpy's Philox4x32-10 counter-based bit generator, one independent
stream per tensor (SeedSequence([seed, tensor_id])), standard normal draws in
float32, rounded to bf16 with round-to-nearest-even.

Workloads follow the gpt-oss attention shapes (64 query heads, 8 key/value
heads, head dim 64, scale 1/8) with values ~N(0,1); the long-context case
draws its sinks from N(0, 2^2) so that some heads are sink-dominated.  The
packed-documents case draws document lengths ~U[256, 8192] until the total
reaches 65536 tokens and truncates the last document to hit it exactly.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

_IDS = {"q": 1, "k": 2, "v": 3, "sinks": 4, "dout": 5, "doclens": 6, "rows": 7,
        "dec_q": 11, "dec_k": 12, "dec_v": 13, "dec_sinks": 14}


def _rng(seed: int, name: str) -> np.random.Generator:
    return np.random.Generator(np.random.Philox(np.random.SeedSequence([int(seed), _IDS[name]])))


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bf16 (nearest-even); returns the uint16 bit patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    rounding = ((u >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((u + rounding) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def normal_bf16(seed: int, name: str, shape, std: float = 1.0) -> np.ndarray:
    x = _rng(seed, name).standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        x *= np.float32(std)
    return f32_to_bf16_bits(x)


def uniform_cu_seqlens(batch: int, seqlen: int) -> np.ndarray:
    return (np.arange(batch + 1, dtype=np.int64) * seqlen).astype(np.int32)


def packed_doc_cu_seqlens(seed: int, total: int = 65536, lo: int = 256, hi: int = 8192) -> np.ndarray:
    """Document lengths ~U[lo, hi] (inclusive) until the sum reaches `total`;
    the last document is cut so the lengths add up to `total` exactly."""
    rng = _rng(seed, "doclens")
    lens = []
    acc = 0
    while acc < total:
        n = int(rng.integers(lo, hi, endpoint=True))
        n = min(n, total - acc)
        lens.append(n)
        acc += n
    return np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)


@dataclass
class Workload:
    name: str
    T: int
    Hq: int
    Hkv: int
    D: int
    cu_seqlens: np.ndarray          # int32 [B+1]
    uniform_seqlen: int | None      # S when every document has the same length
    window: int
    scale: float
    sink_std: float = 1.0
    seed: int = 0
    arrays: dict = field(default_factory=dict)

    @property
    def batch(self) -> int:
        return int(self.cu_seqlens.shape[0] - 1)

    @property
    def max_seqlen(self) -> int:
        c = self.cu_seqlens.astype(np.int64)
        return int((c[1:] - c[:-1]).max()) if c.shape[0] > 1 else 0

    def generate(self, with_dout: bool = False) -> dict:
        a = self.arrays
        if "q" not in a:
            a["q"] = normal_bf16(self.seed, "q", (self.T, self.Hq, self.D))
            a["k"] = normal_bf16(self.seed, "k", (self.T, self.Hkv, self.D))
            a["v"] = normal_bf16(self.seed, "v", (self.T, self.Hkv, self.D))
            a["sinks"] = self.sinks_only()
        if with_dout and "dout" not in a:
            a["dout"] = normal_bf16(self.seed, "dout", (self.T, self.Hq, self.D))
        return a

    def sinks_only(self) -> np.ndarray:
        """The workload's sinks (the same draw generate() makes), without
        generating q, k, v."""
        s = _rng(self.seed, "sinks").standard_normal(size=(self.Hq,), dtype=np.float32)
        return (s * np.float32(self.sink_std)).astype(np.float32)

    def sample_rows(self, n: int) -> np.ndarray:
        """Seeded sample of query tokens: for each of the first 8 documents
        five fixed tokens (its first, second and last token, and the tokens
        127 and 128 places after its start, which sit on either side of a
        128-token tile edge), then random tokens up to n; sorted and
        unique."""
        rng = _rng(self.seed, "rows")
        c = self.cu_seqlens.astype(np.int64)
        fixed = set()
        for b in range(min(self.batch, 8)):
            a, e = int(c[b]), int(c[b + 1])
            if e > a:
                fixed.update([a, e - 1, min(a + 1, e - 1), min(a + 127, e - 1), min(a + 128, e - 1)])
        fixed = [t for t in fixed if 0 <= t < self.T]
        rest = rng.integers(0, self.T, size=max(0, n - len(fixed))) if self.T > 0 else []
        return np.unique(np.concatenate([np.array(fixed, np.int64), np.asarray(rest, np.int64)]))


def workload(name: str, seed: int = 0) -> Workload:
    """The named workloads (gpt-oss attention shapes)."""
    scale = 1.0 / 8.0
    base, _, var = name.partition(":")
    window = {"full": 0, "": 0}.get(var, None)
    if window is None:
        window = int(var.lstrip("w"))
    if base == "tiny":
        return Workload(name, 128, 4, 1, 64, uniform_cu_seqlens(1, 128), 128, window, scale, seed=seed)
    if base == "prefill4k":
        return Workload(name, 4 * 4096, 64, 8, 64, uniform_cu_seqlens(4, 4096), 4096, window, scale, seed=seed)
    if base == "varlen64k":
        cu = packed_doc_cu_seqlens(seed)
        return Workload(name, 65536, 64, 8, 64, cu, None, window, scale, seed=seed)
    if base == "long60k":
        return Workload(name, 61440, 64, 8, 64, uniform_cu_seqlens(1, 61440), 61440, window, scale,
                        sink_std=2.0, seed=seed)
    raise KeyError(name)


WORKLOADS = ["tiny:w32", "tiny:full", "prefill4k:w128", "prefill4k:full", "varlen64k:w128",
             "varlen64k:full", "long60k:full", "long60k:w128"]


def decode_inputs(seed: int, cached: list, new_tokens: int, Hq: int, Hkv: int, D: int = 64,
                  sink_std: float = 1.0) -> dict:
    """Seeded inputs of one decode call (gpt-oss head shapes by default).

    Sequence b has `cached[b]` tokens before the call and `new_tokens` new
    ones.  Returns the whole token history of every sequence packed one after
    another -- k, v [T][Hkv][D] bf16 bits with cu [B+1] -- the new tokens'
    queries q_new [B][new_tokens][Hq][D] (bf16 bits) and sinks [Hq] fp32.
    The new tokens of sequence b are history positions cached[b] ..
    cached[b] + new_tokens - 1."""
    lens = [int(c) + int(new_tokens) for c in cached]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    T = int(cu[-1])
    s = _rng(seed, "dec_sinks").standard_normal(size=(Hq,), dtype=np.float32) * np.float32(sink_std)
    return dict(k=normal_bf16(seed, "dec_k", (T, Hkv, D)), v=normal_bf16(seed, "dec_v", (T, Hkv, D)),
                q_new=normal_bf16(seed, "dec_q", (len(cached), new_tokens, Hq, D)),
                sinks=s.astype(np.float32), cu=cu)

