"""Seeded synthetic inputs for the NVFP4 paged KV path.

This module only draws random numbers and lays out page tables; it holds
none of the path's arithmetic (no quantisation, no attention).  The same
bytes feed the CUDA path and the float64 oracle.

Value recipe (both sides): K, V and q are N(0, 1) drawn as float32 and
rounded to bf16 (round-to-nearest-even, by torch's dtype conversion); four
head_dim channels of K, drawn once per workload and shared by all heads and
tokens, are multiplied by 10 before rounding (outlier channels).  K/V rows
are generated in fixed 4096-row chunks, each from its own counter-seeded
numpy Generator, so any range of positions can be regenerated alone.

Workload shapes follow the serving scenarios the pages describe ("gzenz/ninfer"
README, "Fork changes vs upstream": 3 concurrent agentic sessions of
330k-470k tokens; "knoopx/ninfer" README, "Capabilities and limits": batched
decode, MTP verify with 1-5 drafts, chunked prefill).
"""
from __future__ import annotations

import math
import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field

import numpy as np
import torch

PAGE_TOKENS = 16
CHUNK_ROWS = 4096


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 array -> uint16 array of bf16 bits (round to nearest even)."""
    t = torch.from_numpy(np.ascontiguousarray(x, np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32)


@dataclass
class Workload:
    name: str
    batch: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    T: int                       # new tokens per sequence this step (queries)
    ctx: list                    # tokens cached before the step, per sequence
    mode: str = "decode"         # "decode" (split-K) or "prefill" (chunked)
    shuffled_pages: bool = True
    seed: int = 0
    spare_pages: int = 0
    outliers: np.ndarray = field(default=None, repr=False)

    def __post_init__(self):
        if self.outliers is None:
            rng = np.random.default_rng([self.seed, 3])
            self.outliers = np.sort(rng.choice(self.head_dim, size=4, replace=False))

    # ---- sizes --------------------------------------------------------
    @property
    def group(self) -> int:
        return self.num_q_heads // self.num_kv_heads

    @property
    def kv_lens(self) -> np.ndarray:
        return np.array([c + self.T for c in self.ctx], np.int32)

    @property
    def max_kv_len(self) -> int:
        return int(self.kv_lens.max())

    @property
    def sm_scale(self) -> float:
        return 1.0 / math.sqrt(self.head_dim)

    @property
    def pages_per_seq(self) -> np.ndarray:
        return (self.kv_lens + PAGE_TOKENS - 1) // PAGE_TOKENS

    @property
    def max_pages_per_seq(self) -> int:
        return int(self.pages_per_seq.max())

    @property
    def num_pages(self) -> int:
        return int(self.pages_per_seq.sum()) + self.spare_pages

    def kv_bytes_per_step(self) -> int:
        """NVFP4 KV bytes a full attention step must read: every visible
        cached token, once, for every kv-head, K and V."""
        per_tok = self.num_kv_heads * 2 * (self.head_dim // 2 + self.head_dim // 16)
        return int(self.kv_lens.astype(np.int64).sum()) * per_tok

    # ---- page tables ----------------------------------------------------
    def page_table(self) -> np.ndarray:
        """[batch][max_pages_per_seq] int32; unused entries are -1."""
        n = self.num_pages
        if self.shuffled_pages:
            perm = np.random.default_rng([self.seed, 7]).permutation(n).astype(np.int32)
        else:
            perm = np.arange(n, dtype=np.int32)
        pt = np.full((self.batch, self.max_pages_per_seq), -1, np.int32)
        off = 0
        for b, np_b in enumerate(self.pages_per_seq):
            pt[b, :np_b] = perm[off:off + np_b]
            off += int(np_b)
        return pt

    # ---- values ---------------------------------------------------------
    def _chunk(self, b: int, c: int):
        rng = np.random.default_rng([self.seed, 11, b, c])
        shape = (CHUNK_ROWS, self.num_kv_heads, self.head_dim)
        k = rng.standard_normal(shape, dtype=np.float32)
        k[..., self.outliers] *= 10.0
        v = rng.standard_normal(shape, dtype=np.float32)
        return to_bf16_bits(k), to_bf16_bits(v)

    def kv_rows(self, b: int, start: int, stop: int, threads: int | None = None):
        """bf16 bits of K and V for positions [start, stop) of sequence b,
        each [stop-start][Hkv][D] uint16."""
        n = stop - start
        shape = (n, self.num_kv_heads, self.head_dim)
        k = np.empty(shape, np.uint16)
        v = np.empty(shape, np.uint16)
        if n <= 0:
            return k, v
        c0, c1 = start // CHUNK_ROWS, (stop - 1) // CHUNK_ROWS

        def fill(c):
            kc, vc = self._chunk(b, c)
            lo = max(start, c * CHUNK_ROWS)
            hi = min(stop, (c + 1) * CHUNK_ROWS)
            k[lo - start:hi - start] = kc[lo - c * CHUNK_ROWS:hi - c * CHUNK_ROWS]
            v[lo - start:hi - start] = vc[lo - c * CHUNK_ROWS:hi - c * CHUNK_ROWS]

        nthreads = threads or min(16, os.cpu_count() or 1)
        if c1 == c0 or nthreads == 1:
            for c in range(c0, c1 + 1):
                fill(c)
        else:
            with ThreadPoolExecutor(nthreads) as ex:
                list(ex.map(fill, range(c0, c1 + 1)))
        return k, v

    def new_rows(self):
        """This step's T new rows of every sequence, concatenated
        ([batch*T][Hkv][D] each) with cu_new offsets."""
        ks, vs = [], []
        for b in range(self.batch):
            k, v = self.kv_rows(b, self.ctx[b], self.ctx[b] + self.T)
            ks.append(k)
            vs.append(v)
        cu = np.arange(0, (self.batch + 1) * self.T, self.T, dtype=np.int32)
        return np.concatenate(ks), np.concatenate(vs), cu

    def queries(self) -> np.ndarray:
        """[batch*T][Hq][D] bf16 bits (row b*T + t is query t of sequence b)."""
        out = np.empty((self.batch * self.T, self.num_q_heads, self.head_dim), np.uint16)
        for b in range(self.batch):
            rng = np.random.default_rng([self.seed, 13, b])
            q = rng.standard_normal((self.T, self.num_q_heads, self.head_dim), dtype=np.float32)
            out[b * self.T:(b + 1) * self.T] = to_bf16_bits(q)
        return out

    def query_position(self, b: int, t: int) -> int:
        return int(self.ctx[b]) + t


# --------------------------------------------------------------------------
# the five workloads
# --------------------------------------------------------------------------
def tiny_decode(seed: int = 1001) -> Workload:
    """1 sequence of 4096 tokens, 8 query / 2 KV heads, head_dim 128; all
    4096 rows quantize-appended, then 1 decode query (at position 4095)."""
    return Workload("tiny_decode_4096_h8kv2_d128", 1, 8, 2, 128, 1, [4095],
                    shuffled_pages=False, seed=seed)


def batch2_verify(seed: int = 1002, ctx: int = 32768) -> Workload:
    """2 sequences with 32768 cached tokens, 24/4 heads, head_dim 256,
    shuffled pages, 4 causal query tokens each (3 drafts + 1)."""
    return Workload(f"batch2_mtp4_ctx{ctx}_h24kv4_d256", 2, 24, 4, 256, 4, [ctx, ctx], seed=seed)


def long_context(T: int = 1, seed: int = 1003, ctx=(330000, 420000, 470000)) -> Workload:
    """3 agentic sessions of 330k / 420k / 470k cached tokens, 24/4 heads,
    head_dim 256, random page order; T=1 decode or T=6 MTP verify."""
    name = "long_ctx_" + "_".join(f"{c // 1000}k" for c in ctx) + f"_T{T}_h24kv4_d256"
    return Workload(name, len(ctx), 24, 4, 256, T, list(ctx), seed=seed)


def ragged_batch(seed: int = 1004, batch: int = 64, lo: int = 2048, hi: int = 16384) -> Workload:
    """64 sequences with lengths uniform in [2048, 16384], 24/4 heads,
    head_dim 256, random pages, 1 decode query and 1 appended row each."""
    ctx = np.random.default_rng([seed, 5]).integers(lo, hi + 1, size=batch).tolist()
    return Workload(f"ragged_{batch}x{lo}-{hi}_h24kv4_d256", batch, 24, 4, 256, 1, ctx, seed=seed)


def chunked_prefill(seed: int = 1005, ctx: int = 65536, chunk: int = 2048) -> Workload:
    """1 sequence with 65536 cached tokens plus a new 2048-token chunk
    (quantize-appended first), causal attention of the 2048 chunk queries."""
    return Workload(f"prefill_ctx{ctx}_chunk{chunk}_h24kv4_d256", 1, 24, 4, 256, chunk, [ctx],
                    mode="prefill", seed=seed)


def small(name: str, batch: int, hq: int, hkv: int, d: int, T: int, ctx, mode="decode",
          seed: int = 7, shuffled=True) -> Workload:
    """Small ad-hoc workloads for parity tests."""
    return Workload(name, batch, hq, hkv, d, T, list(ctx), mode=mode, shuffled_pages=shuffled,
                    seed=seed)
