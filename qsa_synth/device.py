"""Device-side materialisation of a workload (torch tensors filled by libqsa_synth.so).

Input generation only: every tensor of a ``Config`` is filled on the GPU with the same values the
host generator in ``qsa_synth`` produces, then the host-computed needle rows are copied over.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np
import torch

from . import (TID_IDXK, TID_IDXQ, TID_IDXW, TID_K, TID_Q, TID_V, Config, HostInputs)

_LIB = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libqsa_synth.so")
if not os.path.exists(_LIB):
    raise ImportError(f"{_LIB} is missing: run `python learned_block_sparse_qsa_b200/build.py`")
_lib = ctypes.CDLL(_LIB)
_lib.qsyn_fill_linear.restype = ctypes.c_int
_lib.qsyn_fill_linear.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64, ctypes.c_uint64,
                                  ctypes.c_uint64, ctypes.c_int, ctypes.c_void_p]
_lib.qsyn_fill_paged.restype = ctypes.c_int
_lib.qsyn_fill_paged.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_int,
                                 ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_uint64,
                                 ctypes.c_uint64, ctypes.c_int, ctypes.c_void_p]


def _stream():
    return torch.cuda.current_stream().cuda_stream


def fill_linear(t: torch.Tensor, seed: int, tid: int, dist: int, offset: int = 0):
    assert t.dtype == torch.bfloat16 and t.is_contiguous()
    rc = _lib.qsyn_fill_linear(t.data_ptr(), t.numel(), offset, seed, tid, dist, _stream())
    if rc != 0:
        raise RuntimeError(f"qsyn_fill_linear failed: cuda error {rc}")


def fill_paged(pool: torch.Tensor, owner: torch.Tensor, max_pages: int, seq_stride: int, seed: int,
               tid: int, dist: int):
    assert pool.dtype == torch.bfloat16 and pool.is_contiguous()
    num_pages, page_tokens = pool.shape[0], pool.shape[1]
    row_elems = pool[0, 0].numel()
    rc = _lib.qsyn_fill_paged(pool.data_ptr(), num_pages, page_tokens, row_elems, owner.data_ptr(),
                              max_pages, seq_stride, seed, tid, dist, _stream())
    if rc != 0:
        raise RuntimeError(f"qsyn_fill_paged failed: cuda error {rc}")


def _bits_to_bf16(a: np.ndarray, device) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(device)


class DeviceInputs:
    """All device tensors of one workload.

    q_seq, q_pos   int32 [Nq]           query rows (sequence-major, the last n_new positions)
    page_table     int32 [B, max_pages]
    k_pool, v_pool bf16  [num_pages, 64, Hkv, D]
    kcomp_pool     bf16  [num_pages, 16, Di]   (zeros; the layer's compress step fills it)
    q              bf16  [Nq, Hq, D]
    idx_q          bf16  [Nq, 4, Di];  idx_w bf16 [Nq, 4]
    idx_k          bf16  [B, ctx, Di]          raw indexer keys of every position
    idx_k_new      bf16  [Nq, Di]              raw indexer keys of the step's new tokens
    """

    def __init__(self, cfg: Config, integer: bool = False, device="cuda"):
        self.cfg = cfg
        self.host = HostInputs(cfg, integer)
        h, c, dev = self.host, cfg, torch.device(device)
        d = h.dist
        q_seq, q_pos = h.rows()
        self.q_seq = torch.from_numpy(q_seq).to(dev)
        self.q_pos = torch.from_numpy(q_pos).to(dev)
        self.page_table = torch.from_numpy(h.page_table()).to(dev)
        owner = torch.from_numpy(h.page_owner()).to(dev)
        self.k_pool = torch.empty(c.num_pages, c.page, c.Hkv, c.D, dtype=torch.bfloat16, device=dev)
        self.v_pool = torch.empty_like(self.k_pool)
        fill_paged(self.k_pool, owner, c.max_pages, c.ctx, c.seed, TID_K, d["k"])
        fill_paged(self.v_pool, owner, c.max_pages, c.ctx, c.seed, TID_V, d["v"])
        self.kcomp_pool = torch.zeros(c.num_pages, 16, c.Di, dtype=torch.bfloat16, device=dev)
        self.q = torch.empty(c.num_q, c.Hq, c.D, dtype=torch.bfloat16, device=dev)
        self.idx_q = torch.empty(c.num_q, c.Hi, c.Di, dtype=torch.bfloat16, device=dev)
        self.idx_w = torch.empty(c.num_q, c.Hi, dtype=torch.bfloat16, device=dev)
        self.idx_k = torch.empty(c.batch, c.ctx, c.Di, dtype=torch.bfloat16, device=dev)
        for s in range(c.batch):
            rows = slice(s * c.n_new, (s + 1) * c.n_new)
            base = s * c.ctx + c.ctx_start
            fill_linear(self.q[rows], c.seed, TID_Q, d["q"], base * c.Hq * c.D)
            fill_linear(self.idx_q[rows], c.seed, TID_IDXQ, d["idx_q"], base * c.Hi * c.Di)
            fill_linear(self.idx_w[rows], c.seed, TID_IDXW, d["idx_w"], base * c.Hi)
            fill_linear(self.idx_k[s], c.seed, TID_IDXK, d["idx_k"], s * c.ctx * c.Di)
        nd = h.needles()
        if nd["blocks"]:
            for s in range(c.batch):
                pos = (np.asarray(nd["blocks"][s])[:, None] * c.block + np.arange(c.block)[None, :]).reshape(-1)
                vals = np.repeat(nd["key_rows"][s], c.block, axis=0)
                self.idx_k[s, torch.from_numpy(pos).to(dev)] = _bits_to_bf16(vals, dev)
            if nd["q_rows"]:
                rows = np.array(sorted(nd["q_rows"]), dtype=np.int64)
                vals = np.stack([nd["q_vals"][int(r)] for r in rows])
                self.idx_q[torch.from_numpy(rows).to(dev)] = _bits_to_bf16(vals, dev)
        self.idx_k_new = torch.cat([self.idx_k[s, c.ctx_start:c.ctx] for s in range(c.batch)]).contiguous()
        self.new_seq = self.q_seq
        self.new_pos = self.q_pos

    def prefix_rows(self, s: int):
        """(idx_k rows, new_seq, new_pos) of the blocks before the step's new tokens of sequence s."""
        c = self.cfg
        n = (c.ctx_start // c.block) * c.block
        dev = self.q_seq.device
        seq = torch.full((n,), s, dtype=torch.int32, device=dev)
        pos = torch.arange(n, dtype=torch.int32, device=dev)
        return self.idx_k[s, :n], seq, pos
