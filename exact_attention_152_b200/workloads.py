"""Named synthetic workloads (shapes, seeds, value distributions).

No attention arithmetic here.  Each workload fixes B, H, Nq, Nk, d, causality,
the seed and the distribution of Q, K and V; the scale is the fp32 value of
1/sqrt(d).  The pages name no dataset or benchmark suite: their workloads are
BF16 multi-head attention forwards on B200 at long sequence lengths, so these
synthetic shapes stand in for them.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

from . import inputs, masks


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    Nq: int
    Nk: int
    d: int
    causal: bool
    seed: int
    q_dist: str = "normal"
    q_mult: float = 1.0
    k_dist: str = "normal"
    v_dist: str = "normal"
    oracle_rows: int | None = None  # sampled rows per head for the oracle; None = all
    Hkv: int | None = None          # key/value heads (grouped-query attention); None = H
    window: tuple | None = None     # key band (left, right), -1 = no bound; replaces causal
    seqlens: tuple | None = None    # packed variable-length batch: one length per sequence
                                    # (queries and keys alike); B = len(seqlens)
    fp8: bool = False               # Q, K, V as E4M3 codes times the descale factors below
    descale: tuple = (1.0, 1.0, 1.0)  # (q, k, v) scale factors of the E4M3 codes
    docs: tuple | None = None       # column-interval document mask: lengths uniform in
                                    # [lo, hi] per batch entry (with causal: block-diagonal causal)

    @property
    def colmask(self) -> bool:
        return self.docs is not None

    def doc_lengths(self, b: int) -> list:
        return masks.document_lengths(self.seed * 1000 + b, self.Nk, *self.docs)

    def colmask_array(self) -> np.ndarray:
        """int32 [B, 1, Nk, 4] column intervals of the document mask."""
        return masks.documents([self.doc_lengths(b) for b in range(self.B)], self.Nk)

    @property
    def packed(self) -> bool:
        return self.seqlens is not None

    @property
    def band(self) -> tuple:
        """(window_left, window_right) of the mask: -1 = no bound."""
        if self.window is not None:
            return tuple(self.window)
        return (-1, 0) if self.causal else (-1, -1)

    @property
    def cu_seqlens(self) -> np.ndarray:
        return np.concatenate([[0], np.cumsum(self.seqlens)]).astype(np.int32)

    @property
    def total(self) -> int:
        return int(sum(self.seqlens))

    @property
    def kv_heads(self) -> int:
        return self.H if self.Hkv is None else self.Hkv

    @property
    def scale(self) -> float:
        return float(np.float32(1.0 / math.sqrt(self.d)))

    @property
    def flops(self) -> float:
        """Algorithmic FLOPs, 4*d per visible (query, key) pair: 4*B*H*Nq*Nk*d
        without a mask, half of that for causal (the usual convention), and the
        exact count of visible pairs for a band or a packed batch."""
        if self.colmask:
            pairs = masks.visible_pairs(self.colmask_array(), self.Nq, self.causal)
            return 4.0 * self.d * self.H * float(pairs.sum())
        if self.window is None and not self.packed:
            f = 4.0 * self.B * self.H * self.Nq * self.Nk * self.d
            return f / 2 if self.causal else f
        lens = self.seqlens if self.packed else [self.Nq] * self.B
        pairs = sum(float(visible_keys(np.arange(n), n, *self.band).sum()) for n in lens)
        return 4.0 * self.d * self.H * pairs

    def shape(self, which: str):
        heads = self.H if which == "q" else self.kv_heads
        if self.packed:
            return (self.total, heads, self.d)
        if which == "q":
            return (self.B, self.H, self.Nq, self.d)
        return (self.B, self.kv_heads, self.Nk, self.d)

    def dist(self, which: str):
        if which == "q":
            return self.q_dist, self.q_mult
        if which == "k":
            return self.k_dist, 1.0
        return self.v_dist, 1.0

    def tensor_bits(self, which: str) -> np.ndarray:
        """BF16 bits (uint16), or E4M3 codes (uint8) for an FP8 workload."""
        dist, mult = self.dist(which)
        if self.fp8:
            return inputs.gen_e4m3(self.seed, which, self.shape(which), dist, mult)
        return inputs.gen_bf16(self.seed, which, self.shape(which), dist, mult)

    def to_f64(self, which: str, bits: np.ndarray) -> np.ndarray:
        """The values the stored bits stand for (E4M3 codes times their descale)."""
        if self.fp8:
            return inputs.e4m3_to_f64(bits) * self.descale["qkv".index(which)]
        return inputs.bf16_bits_to_f64(bits)

    def head_bits(self, which: str, bh: int) -> np.ndarray:
        """BF16 bits of one (b, h) slice, [N, d]; for k/v, bh indexes the B*Hkv
        key/value heads (see kv_head_of)."""
        dist, mult = self.dist(which)
        n = self.Nq if which == "q" else self.Nk
        base = bh * n * self.d
        idx = np.arange(base, base + n * self.d, dtype=np.int64)
        if self.fp8:
            return inputs.e4m3_at(self.seed, which, idx, dist, mult).reshape(n, self.d)
        return inputs.gen_bf16_at(self.seed, which, idx, dist, mult).reshape(n, self.d)

    def q_rows_bits(self, bh: int, rows: np.ndarray) -> np.ndarray:
        dist, mult = self.dist("q")
        base = bh * self.Nq * self.d
        idx = base + rows.astype(np.int64)[:, None] * self.d + np.arange(self.d, dtype=np.int64)[None, :]
        if self.fp8:
            return inputs.e4m3_at(self.seed, "q", idx, dist, mult)
        return inputs.gen_bf16_at(self.seed, "q", idx, dist, mult)

    def kv_head_of(self, bh: int) -> int:
        """Flattened key/value head read by flattened query head bh."""
        b, h = divmod(bh, self.H)
        return b * self.kv_heads + h // (self.H // self.kv_heads)

    def seq_head_bits(self, which: str, s: int, h: int, rows=None) -> np.ndarray:
        """Packed batch: BF16 bits of sequence s, head h (a key/value head for
        k and v), rows `rows` of the sequence (default all) -> [n, d]."""
        dist, mult = self.dist(which)
        heads = self.H if which == "q" else self.kv_heads
        start = int(self.cu_seqlens[s])
        if rows is None:
            rows = np.arange(self.seqlens[s], dtype=np.int64)
        idx = ((start + np.asarray(rows, dtype=np.int64))[:, None] * heads + h) * self.d \
            + np.arange(self.d, dtype=np.int64)[None, :]
        return inputs.gen_bf16_at(self.seed, which, idx, dist, mult)

    def sampled_rows(self, bh: int) -> np.ndarray:
        if self.oracle_rows is None:
            return np.arange(self.Nq, dtype=np.int64)
        return inputs.sample_rows(self.seed, bh, self.Nq, self.oracle_rows)


def visible_keys(rows, nk, window_left, window_right) -> np.ndarray:
    """Number of keys in the band [i - left, i + right] of each query row i,
    clipped to 0 .. nk-1 (-1 = no bound)."""
    rows = np.asarray(rows, dtype=np.int64)
    lo = np.zeros_like(rows) if window_left < 0 else np.maximum(rows - window_left, 0)
    hi = np.full_like(rows, nk - 1) if window_right < 0 else np.minimum(rows + window_right, nk - 1)
    return np.maximum(hi - lo + 1, 0)


def _mixed_lengths(seed, n, lo, hi):
    """n sequence lengths, uniform in [lo, hi], from the counter-based generator."""
    u = inputs.uniform_at(seed, "len", np.arange(n, dtype=np.int64))
    return tuple(int(lo + (hi - lo) * x) for x in u)


WORKLOADS = {
    w.name: w
    for w in [
        Workload("tiny_b1h2n128d64", 1, 2, 128, 128, 64, False, seed=0),
        Workload("mha_b4h16n1k_d128", 4, 16, 1024, 1024, 128, False, seed=1),
        Workload("mha_b2h16n8k_d128", 2, 16, 8192, 8192, 128, False, seed=2, oracle_rows=256),
        Workload("mha_b2h16n8k_d128_causal", 2, 16, 8192, 8192, 128, True, seed=2, oracle_rows=256),
        Workload("wide_logits_b1h32n16k_d128_causal", 1, 32, 16384, 16384, 128, True, seed=3,
                 q_mult=8.0, v_dist="uniform", oracle_rows=256),
        Workload("long_b1h16n128k_d128_causal", 1, 16, 131072, 131072, 128, True, seed=4,
                 oracle_rows=256),
        Workload("gqa_b2h32kv8n8k_d128", 2, 32, 8192, 8192, 128, False, seed=5, oracle_rows=128,
                 Hkv=8),
        Workload("gqa_b2h32kv8n8k_d128_causal", 2, 32, 8192, 8192, 128, True, seed=5,
                 oracle_rows=128, Hkv=8),
        # causal sliding window over the last 4096 keys
        Workload("swa_b1h32n32k_w4k_d128", 1, 32, 32768, 32768, 128, False, seed=6,
                 oracle_rows=128, window=(4095, 0)),
        # E4M3 inputs (the FP8 forward)
        Workload("fp8_b2h16n8k_d128", 2, 16, 8192, 8192, 128, False, seed=8, oracle_rows=128,
                 fp8=True),
        Workload("fp8_b2h16n8k_d128_causal", 2, 16, 8192, 8192, 128, True, seed=8, oracle_rows=128,
                 fp8=True),
        # causal document mask (column intervals): documents of 256 .. 4096 tokens
        Workload("docs_b2h16n8k_d128_causal", 2, 16, 8192, 8192, 128, True, seed=9,
                 oracle_rows=128, docs=(256, 4096)),
        # 16 sequences of mixed length (512 .. 16384 tokens), packed, causal
        Workload("varlen16_h16_d128_causal", 16, 16, 0, 0, 128, True, seed=7, oracle_rows=64,
                 seqlens=_mixed_lengths(7, 16, 512, 16384)),
    ]
}

HEADLINE = "mha_b2h16n8k_d128"
