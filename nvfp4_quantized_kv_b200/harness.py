"""Device-side set-up of a synthetic workload and one step of the path.

A step is what one decode (or prefill-chunk) iteration of one attention
layer does: quantise-append this step's new K/V rows into the pool, then
attention of this step's queries against the whole cache (split-K decode +
combine, or chunked prefill).  The cached context before the step is built
once, untimed, by appending the workload's rows chunk by chunk.
"""
from __future__ import annotations

import numpy as np
import torch

from . import (Cache, Seqs, nvkv_append, nvkv_append_k8v4, nvkv_combine, nvkv_decode_attn,
               nvkv_decode_attn_k8v4, nvkv_decode_workspace_bytes, nvkv_prefill_attn,
               nvkv_prefill_attn_k8v4, nvkv_prefill_attn_split, nvkv_prefill_workspace_bytes)

# The calls of each cache format: (append, decode partials, prefill).
_CALLS = {
    "nvfp4": (nvkv_append, nvkv_decode_attn, nvkv_prefill_attn),
    "k8v4": (nvkv_append_k8v4, nvkv_decode_attn_k8v4, nvkv_prefill_attn_k8v4),
}
from .workload import Workload


def _h2d(a: np.ndarray, device, dtype=None) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.view(dtype)
    return t.to(device, non_blocking=False)


def bf16_tensor(bits: np.ndarray, device) -> torch.Tensor:
    return _h2d(bits.view(np.int16), device).view(torch.bfloat16)


class DeviceWorkload:
    def __init__(self, wl: Workload, device="cuda", fill: int | None = 0xA5, num_splits: int = 0,
                 err_word: bool = True, cache_from: "DeviceWorkload | None" = None,
                 kv_format: str = "nvfp4", prefill_splits: "int | None" = None):
        """cache_from: reuse the (already filled) pool of another workload
        with the same cached context -- same seed, lengths, heads and page
        table -- under a different step shape (T=1 decode and T=6 verify).
        kv_format: "nvfp4" (the default) or "k8v4".
        prefill_splits: None runs nvkv_prefill_attn; a count (0: automatic)
        runs nvkv_prefill_attn_split with a workspace (NVFP4 only)."""
        if kv_format not in _CALLS:
            raise ValueError(f"kv_format must be one of {tuple(_CALLS)}")
        self.kv_format = kv_format
        self._append, self._decode, self._prefill = _CALLS[kv_format]
        self.wl = wl
        self.device = torch.device(device)
        self.num_splits = num_splits
        self.page_table_np = wl.page_table()
        if cache_from is not None:
            o = cache_from.wl
            if (o.seed, list(o.ctx), o.num_kv_heads, o.head_dim, o.num_pages) != \
                    (wl.seed, list(wl.ctx), wl.num_kv_heads, wl.head_dim, wl.num_pages) or \
                    not np.array_equal(cache_from.page_table_np, self.page_table_np) or \
                    cache_from.kv_format != kv_format:
                raise ValueError("cache_from: the two workloads do not share a cached context")
            self.cache = cache_from.cache
        else:
            self.cache = Cache.allocate(wl.num_pages, wl.num_kv_heads, wl.head_dim, self.device,
                                        fill, kv_format)
        self.page_table = _h2d(self.page_table_np, self.device)
        self.kv_lens = _h2d(wl.kv_lens, self.device)
        self.err = torch.zeros(1, dtype=torch.int32, device=self.device) if err_word else None
        self.seqs = Seqs(self.page_table, self.kv_lens, wl.max_kv_len, self.err)
        rows = wl.batch * wl.T
        self.out = torch.empty(rows, wl.num_q_heads, wl.head_dim, dtype=torch.bfloat16,
                               device=self.device)
        if wl.mode == "decode":
            nbytes = nvkv_decode_workspace_bytes(wl.batch, wl.T, wl.num_q_heads, wl.num_kv_heads,
                                                 wl.head_dim, num_splits)
            self.workspace = torch.empty(nbytes, dtype=torch.uint8, device=self.device)
        else:
            self.workspace = None
        self.prefill_splits = prefill_splits
        if wl.mode != "decode" and prefill_splits is not None:
            if kv_format != "nvfp4":
                raise ValueError("the key-split prefill takes an NVFP4 cache")
            nbytes = nvkv_prefill_workspace_bytes(rows, wl.num_q_heads, wl.head_dim,
                                                  prefill_splits)
            self.workspace = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=self.device)
        self.k_new = self.v_new = self.cu_new = self.q = None

    # ---- context ---------------------------------------------------------
    def fill_context(self, chunk_rows: int = 65536) -> None:
        """Append positions [0, ctx_b) of every sequence (untimed set-up)."""
        wl = self.wl
        for b in range(wl.batch):
            pt_b = self.page_table[b:b + 1]
            for start in range(0, wl.ctx[b], chunk_rows):
                stop = min(wl.ctx[b], start + chunk_rows)
                k, v = wl.kv_rows(b, start, stop)
                lens = torch.tensor([stop], dtype=torch.int32, device=self.device)
                seqs = Seqs(pt_b, lens, stop, self.err)
                cu = torch.tensor([0, stop - start], dtype=torch.int32, device=self.device)
                self._append(self.cache, seqs, bf16_tensor(k, self.device),
                             bf16_tensor(v, self.device), cu, stop - start, stop - start)
        torch.cuda.synchronize(self.device)

    # ---- step inputs -----------------------------------------------------
    def load_step_inputs(self) -> None:
        k, v, cu = self.wl.new_rows()
        self.k_new_np, self.v_new_np, self.cu_new_np = k, v, cu
        self.q_np = self.wl.queries()
        self.k_new = bf16_tensor(k, self.device)
        self.v_new = bf16_tensor(v, self.device)
        self.cu_new = _h2d(cu, self.device)
        self.q = bf16_tensor(self.q_np, self.device)

    # ---- one step ----------------------------------------------------------
    def append(self, stream=None) -> None:
        wl = self.wl
        self._append(self.cache, self.seqs, self.k_new, self.v_new, self.cu_new, wl.batch * wl.T,
                     wl.T, stream)

    def attend(self, stream=None) -> None:
        wl = self.wl
        if wl.mode == "decode":
            self._decode(self.cache, self.seqs, self.q, wl.T, wl.num_q_heads, wl.sm_scale,
                         self.num_splits, self.workspace, stream)
            nvkv_combine(self.seqs, self.workspace, wl.T, wl.num_q_heads, wl.num_kv_heads,
                         wl.head_dim, self.num_splits, self.out, stream)
        elif self.prefill_splits is not None:
            nvkv_prefill_attn_split(self.cache, self.seqs, self.q, self.cu_new, wl.batch * wl.T,
                                    wl.T, wl.num_q_heads, wl.sm_scale, self.prefill_splits,
                                    self.workspace, self.out, stream)
        else:
            self._prefill(self.cache, self.seqs, self.q, self.cu_new, wl.batch * wl.T, wl.T,
                          wl.num_q_heads, wl.sm_scale, self.out, stream)

    def step(self, stream=None) -> None:
        self.append(stream)
        self.attend(stream)

    def err_bits(self) -> int:
        return int(self.err.item()) if self.err is not None else 0
