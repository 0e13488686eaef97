"""QsaRunner: one QSA layer step = the C-ABI calls in order, with cached workspaces.

The steps, as the article "Qwen's million-token window has a 2,048-token keyhole" describes the
layer (section "A million-token window with a selective view"): compress the new indexer keys
into 4-token micro-blocks, score and select the best blocks plus the tail, then run core
attention over the selected positions only.  Prefill uses the one-CTA-per-row attention; decode
(few rows, section "Three speed claims, three different experiments") uses the split-K form.

PyTorch only allocates the workspaces and the error flag; every step runs in libqsa's kernels.
"""
from __future__ import annotations

import ctypes

import torch

from . import (QSA_OP_DENSE_ATTN_DECODE, QSA_OP_INDEX_SCORE_TOPK, QSA_OP_SPARSE_ATTN_DECODE,
               QsaBatch, QsaConfig, qsa_dense_attn_decode, qsa_dense_attn_prefill,
               qsa_index_compress, qsa_index_score_redo_flags, qsa_index_score_topk,
               qsa_sparse_attn_decode,
               qsa_sparse_attn_prefill, qsa_workspace_size)


def compress_split(carry_pos: int, carry_len: int, pos0: int, n_new: int):
    """How one prefill chunk of a sequence feeds step (a) when chunk boundaries are not multiples
    of the 4-token block (the article's "unfinished block at the sequence tail" carries over).

    carry_pos, carry_len: the carried raw keys cover positions [carry_pos, carry_pos + carry_len)
    of the block that the previous chunk left unfinished (carry_len in 0..3).  The chunk's new
    keys cover [pos0, pos0 + n_new) and must continue the carry.  Returns (start, n_compress,
    next_carry_pos, next_carry_len): the keys [start, start + n_compress) -- carry first, then the
    chunk's -- form whole blocks to compress now, and the rest is carried to the next chunk."""
    if carry_len:
        if carry_pos % 4 or carry_pos + carry_len != pos0:
            raise ValueError("the chunk must continue the carried block")
        start = carry_pos
    else:
        if pos0 % 4:
            raise ValueError("a chunk that starts inside a block needs that block's earlier keys")
        start = pos0
    total = (pos0 + n_new) - start
    n_compress = total // 4 * 4
    return start, n_compress, start + n_compress, total - n_compress


class BlockCarry:
    """Per-sequence raw indexer keys of the unfinished block, carried between prefill chunks so
    that every block is compressed exactly once, when it completes.  Device tensors only; the
    compression itself is qsa_index_compress."""

    def __init__(self):
        self._carry: dict[int, tuple[int, torch.Tensor]] = {}

    def compress_chunk(self, runner: "QsaRunner", b: QsaBatch, seq: int, pos0: int, idx_k_new,
                       kcomp_pool, stream=None):
        """Compress the blocks that the chunk's keys idx_k_new ([n, Di], positions pos0..) complete."""
        cpos, ckeys = self._carry.get(seq, (pos0, idx_k_new[:0]))
        start, n, npos, nlen = compress_split(cpos, ckeys.shape[0], pos0, idx_k_new.shape[0])
        keys = torch.cat([ckeys, idx_k_new]) if ckeys.shape[0] else idx_k_new
        if n:
            dev = keys.device
            seqs = torch.full((n,), seq, dtype=torch.int32, device=dev)
            poss = torch.arange(start, start + n, dtype=torch.int32, device=dev)
            runner.compress(b, keys[:n].contiguous(), seqs, poss, kcomp_pool, stream)
        self._carry[seq] = (npos, keys[n:].clone())
        return n


class QsaRunner:
    def __init__(self, cfg: QsaConfig, device="cuda"):
        self.cfg = cfg
        self.device = torch.device(device)
        self.err = torch.zeros(1, dtype=torch.int32, device=self.device)
        self._ws: dict[int, torch.Tensor] = {}
        self._keep = []

    def batch(self, *, batch: int, num_q: int, max_pages: int, num_pages: int, max_pos: int,
              q_seq: torch.Tensor, q_pos: torch.Tensor, page_table: torch.Tensor) -> QsaBatch:
        self._keep = [q_seq, q_pos, page_table]
        return QsaBatch(batch, num_q, max_pages, num_pages, max_pos, q_seq.data_ptr(),
                        q_pos.data_ptr(), page_table.data_ptr(), self.err.data_ptr())

    def workspace(self, b: QsaBatch, op: int, splits: int = 0):
        n = qsa_workspace_size(self.cfg, b, op, splits)
        buf = self._ws.get(op)
        if n > 0 and (buf is None or buf.numel() < n):
            buf = torch.empty(n, dtype=torch.uint8, device=self.device)
            self._ws[op] = buf
        return (buf if n > 0 else None), n

    def compress(self, b: QsaBatch, idx_k_new, new_seq, new_pos, kcomp_pool, stream=None):
        qsa_index_compress(self.cfg, b, idx_k_new, new_seq, new_pos, int(new_seq.numel()), kcomp_pool,
                           stream)

    def select(self, b: QsaBatch, idx_q, idx_w, kcomp_pool, sel, n_sel, sel_scores=None, stream=None):
        ws, n = self.workspace(b, QSA_OP_INDEX_SCORE_TOPK)
        qsa_index_score_topk(self.cfg, b, idx_q, idx_w, kcomp_pool, sel, n_sel, sel_scores, ws, n,
                             stream)

    def prefill(self, b: QsaBatch, *, q, idx_q, idx_w, kcomp_pool, k_pool, v_pool, out, sel, n_sel,
                idx_k_new=None, new_seq=None, new_pos=None, lse=None, sel_scores=None, stream=None):
        """Whole prefill step: compress (if new keys are given) -> score/select -> attention."""
        with torch.cuda.nvtx.range("qsa.prefill"):
            if idx_k_new is not None:
                self.compress(b, idx_k_new, new_seq, new_pos, kcomp_pool, stream)
            self.select(b, idx_q, idx_w, kcomp_pool, sel, n_sel, sel_scores, stream)
            qsa_sparse_attn_prefill(self.cfg, b, q, k_pool, v_pool, sel, n_sel, out, lse, stream)
        return out

    def decode(self, b: QsaBatch, *, q, idx_q, idx_w, kcomp_pool, k_pool, v_pool, out, sel, n_sel,
               idx_k_new=None, new_seq=None, new_pos=None, lse=None, sel_scores=None, splits=0,
               stream=None):
        """Whole decode step: compress the new block -> score/select -> split-K attention."""
        with torch.cuda.nvtx.range("qsa.decode"):
            if idx_k_new is not None:
                self.compress(b, idx_k_new, new_seq, new_pos, kcomp_pool, stream)
            self.select(b, idx_q, idx_w, kcomp_pool, sel, n_sel, sel_scores, stream)
            ws, n = self.workspace(b, QSA_OP_SPARSE_ATTN_DECODE, splits)
            qsa_sparse_attn_decode(self.cfg, b, q, k_pool, v_pool, sel, n_sel, out, lse, splits,
                                   ws, n, stream)
        return out

    def dense(self, b: QsaBatch, *, q, k_pool, v_pool, out, lse=None, decode=False, splits=0,
              stream=None):
        """Dense paged-GQA baseline on the same pools."""
        if decode:
            ws, n = self.workspace(b, QSA_OP_DENSE_ATTN_DECODE, splits)
            qsa_dense_attn_decode(self.cfg, b, q, k_pool, v_pool, out, lse, splits, ws, n, stream)
        else:
            qsa_dense_attn_prefill(self.cfg, b, q, k_pool, v_pool, out, lse, stream)
        return out

    def redo_flags(self, b: QsaBatch):
        """Host copy (numpy int32 [num_q]) of the last selection's redo flags -- 1 where the exact
        streaming kernel recomputed a row the fast kernel could not settle -- or None when the
        resolved score path keeps none.  Synchronises the device."""
        ws, n = self.workspace(b, QSA_OP_INDEX_SCORE_TOPK)
        if ws is None:
            return None
        p = qsa_index_score_redo_flags(self.cfg, b, ws, n)
        if p is None:
            return None
        off = p - ws.data_ptr()
        return ws[off: off + 4 * b.num_q].view(torch.int32).cpu().numpy()

    def error_bits(self) -> int:
        return int(self.err.item())

    def clear_error(self):
        self.err.zero_()


__all__ = ["QsaRunner", "BlockCarry", "compress_split", "ctypes"]
