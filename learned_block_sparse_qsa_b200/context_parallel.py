"""Context-parallel QSA layer step: one sequence's context split across ranks.

Each rank holds one contiguous range of positions (a shard, whole 64-token pages) of every
sequence: its keys, values and compressed indexer keys, behind a local page table.  One step, as
the C-ABI header describes it (section "Context parallelism" of include/qsa.h):

    1. local positions of the query rows for this shard            (qsa_cp_shard_positions)
    2. the exact best candidates of the shard, in local block ids    (qsa_index_score_topk)
    3. all-gather of every rank's candidate lists                    (collective)
    4. the global selection, and this shard's winners in local ids   (qsa_index_merge_candidates)
    5. attention over this shard's winners: a partial output + lse   (qsa_sparse_attn_*)
    6. all-gather of the partials, merged by log-sum-exp             (collective, then
                                                                      qsa_attn_merge_partials)

The global selection equals the single-GPU one (every global winner is a winner of its own
shard) and the merged output is the layer's output.  The article measures one accelerator; this
is the layer's split for contexts that several must share.

Every step of the path runs in libqsa's kernels; this module sequences them and allocates device
memory.  ``all_gather(t)`` must return a tensor [world, *t.shape] of every rank's ``t`` in rank
order: ``dist_all_gather`` does it with torch.distributed (NCCL over NVLink); a single-process
caller can gather shards it runs itself.  ``ops`` may be replaced (tests run the host logic on CPU
against the oracle); the default is the library.
"""
from __future__ import annotations

import dataclasses

import torch

from . import (QSA_OP_INDEX_SCORE_TOPK, QSA_OP_MERGE_CANDIDATES, QSA_OP_SPARSE_ATTN_DECODE,
               QsaBatch, QsaConfig, qsa_attn_merge_partials, qsa_cp_shard_positions,
               qsa_index_merge_candidates, qsa_index_score_topk, qsa_sparse_attn_decode,
               qsa_sparse_attn_prefill, qsa_workspace_size)


def dist_all_gather(t: torch.Tensor, group=None) -> torch.Tensor:
    """[world, *t.shape]: every rank's tensor, in rank order (torch.distributed; one
    all_gather_into_tensor on NCCL, a list all_gather on other backends)."""
    import torch.distributed as dist

    world = dist.get_world_size(group)
    t = t.contiguous()
    if dist.get_backend(group) == "nccl":
        out = torch.empty((world, *t.shape), dtype=t.dtype, device=t.device)
        dist.all_gather_into_tensor(out, t, group=group)
        return out
    parts = [torch.empty_like(t) for _ in range(world)]
    dist.all_gather(parts, t, group=group)
    return torch.stack(parts)


@dataclasses.dataclass
class Shard:
    """Positions [start, start + length) of every sequence, held by one rank."""

    start: int
    length: int

    @property
    def block_lo(self) -> int:
        return self.start // 4

    @property
    def block_hi(self) -> int:
        return (self.start + self.length) // 4


@dataclasses.dataclass
class Rows:
    """Query rows as one kernel call sees them: positions in some coordinates and the page table
    (device tensors) that maps those coordinates to pages."""

    batch: int
    q_seq: torch.Tensor
    q_pos: torch.Tensor
    page_table: torch.Tensor
    num_pages: int
    max_pos: int


class LibOps:
    """The library's kernels, one method per step (device tensors)."""

    def __init__(self, cfg: QsaConfig, device):
        self.cfg = cfg
        self.device = torch.device(device)
        self.err = torch.zeros(1, dtype=torch.int32, device=self.device)
        self._ws: dict[int, torch.Tensor] = {}

    def _b(self, r: Rows) -> QsaBatch:
        return QsaBatch(r.batch, r.q_pos.numel(), r.page_table.shape[1], r.num_pages, r.max_pos,
                        r.q_seq.data_ptr(), r.q_pos.data_ptr(), r.page_table.data_ptr(),
                        self.err.data_ptr())

    def _workspace(self, b: QsaBatch, op: int, n: int = 0):
        nbytes = qsa_workspace_size(self.cfg, b, op, n)
        buf = self._ws.get(op)
        if nbytes > 0 and (buf is None or buf.numel() < nbytes):
            buf = torch.empty(nbytes, dtype=torch.uint8, device=self.device)
            self._ws[op] = buf
        return (buf if nbytes > 0 else None), nbytes

    def positions(self, q_pos, shard: Shard, pos_sel, pos_attn):
        qsa_cp_shard_positions(q_pos, q_pos.numel(), shard.start, shard.length, pos_sel, pos_attn)

    def select(self, rows: Rows, idx_q, idx_w, kcomp_pool, sel, n_sel, scores):
        b = self._b(rows)
        ws, n = self._workspace(b, QSA_OP_INDEX_SCORE_TOPK)
        qsa_index_score_topk(self.cfg, b, idx_q, idx_w, kcomp_pool, sel, n_sel, scores, ws, n)

    def merge(self, rows: Rows, part_sel, part_scores, part_lo, shard: Shard, sel, n_sel, scores,
              local_sel, local_n):
        b = self._b(rows)
        nparts = part_sel.shape[0]
        ws, n = self._workspace(b, QSA_OP_MERGE_CANDIDATES, nparts)
        qsa_index_merge_candidates(self.cfg, b, nparts, part_sel, part_scores, part_lo,
                                   shard.block_lo, shard.block_hi, sel, n_sel, scores, local_sel,
                                   local_n, ws, n)

    def attend(self, rows: Rows, q, k_pool, v_pool, sel, n_sel, out, lse, decode: bool):
        b = self._b(rows)
        if decode:
            ws, n = self._workspace(b, QSA_OP_SPARSE_ATTN_DECODE, 0)
            qsa_sparse_attn_decode(self.cfg, b, q, k_pool, v_pool, sel, n_sel, out, lse, 0, ws, n)
        else:
            qsa_sparse_attn_prefill(self.cfg, b, q, k_pool, v_pool, sel, n_sel, out, lse)

    def merge_partials(self, part_out, part_lse, out, lse):
        p, nq, hq, d = part_out.shape
        qsa_attn_merge_partials(p, nq, hq, d, part_out, part_lse, out, lse)

    def error_bits(self) -> int:
        return int(self.err.item())


class ContextParallelStep:
    """One rank's side of a context-parallel QSA step (compressed keys of the shard already
    built).  ``shards``: every rank's Shard, in rank order; ``rank``: this rank.  The local page
    table of a shard has length/64 + 1 columns (the last may name any valid page)."""

    def __init__(self, cfg: QsaConfig, shards: list[Shard], rank: int, device="cuda", ops=None):
        for s in shards:
            if s.start % 64 or s.length % 64 or s.length <= 0:
                raise ValueError("shards must be whole 64-token pages")
        self.cfg = cfg
        self.shards = shards
        self.rank = rank
        self.shard = shards[rank]
        self.device = torch.device(device)
        self.ops = ops if ops is not None else LibOps(cfg, device)

    def select_local(self, *, batch: int, q_seq, q_pos, local_page_table, num_pages: int, idx_q,
                     idx_w, kcomp_pool):
        """Steps 1-2: this shard's candidates (sel, scores: [num_q, topk+1], local ids)."""
        nq, k1 = q_pos.numel(), self.cfg.topk_blocks + 1
        dev = self.device
        self._q_seq, self._q_pos = q_seq, q_pos
        self._pos_sel = torch.empty(nq, dtype=torch.int32, device=dev)
        self._pos_attn = torch.empty(nq, dtype=torch.int32, device=dev)
        self.ops.positions(q_pos, self.shard, self._pos_sel, self._pos_attn)
        self._local = (batch, local_page_table, num_pages)
        rows = Rows(batch, q_seq, self._pos_sel, local_page_table, num_pages, self.shard.length)
        sel = torch.empty(nq, k1, dtype=torch.int32, device=dev)
        n_sel = torch.empty(nq, dtype=torch.int32, device=dev)
        scores = torch.empty(nq, k1, dtype=torch.float32, device=dev)
        self.ops.select(rows, idx_q, idx_w, kcomp_pool, sel, n_sel, scores)
        return sel, scores

    def merge_and_attend(self, part_sel, part_scores, *, max_pos: int, q, k_pool, v_pool,
                         decode: bool = False):
        """Steps 4-5 from the gathered lists ([world, num_q, topk+1]): the global selection
        (self.sel, self.n_sel, self.sel_scores) and this shard's partial attention (out bf16
        [num_q, Hq, D], lse [num_q, Hq])."""
        nq, k1 = self._q_pos.numel(), self.cfg.topk_blocks + 1
        dev = self.device
        batch, lpt, num_pages = self._local
        self.sel = torch.empty(nq, k1, dtype=torch.int32, device=dev)
        self.n_sel = torch.empty(nq, dtype=torch.int32, device=dev)
        self.sel_scores = torch.empty(nq, k1, dtype=torch.float32, device=dev)
        local_sel = torch.empty(nq, k1, dtype=torch.int32, device=dev)
        local_n = torch.empty(nq, dtype=torch.int32, device=dev)
        self.ops.merge(Rows(batch, self._q_seq, self._q_pos, lpt, num_pages, max_pos), part_sel,
                       part_scores, [s.block_lo for s in self.shards], self.shard, self.sel,
                       self.n_sel, self.sel_scores, local_sel, local_n)
        out = torch.empty(nq, self.cfg.num_q_heads, self.cfg.head_dim, dtype=torch.bfloat16, device=dev)
        lse = torch.empty(nq, self.cfg.num_q_heads, dtype=torch.float32, device=dev)
        rows = Rows(batch, self._q_seq, self._pos_attn, lpt, num_pages, self.shard.length - 1)
        self.ops.attend(rows, q, k_pool, v_pool, local_sel, local_n, out, lse, decode)
        return out, lse

    def combine(self, part_out, part_lse, out, lse=None):
        """Step 6: the layer's output from every shard's partial ([world, ...])."""
        self.ops.merge_partials(part_out, part_lse, out, lse)
        return out

    def step(self, all_gather, *, batch: int, q_seq, q_pos, max_pos: int, local_page_table,
             num_pages: int, idx_q, idx_w, kcomp_pool, q, k_pool, v_pool, out, lse=None,
             decode: bool = False):
        """The whole step on this rank; ``all_gather`` is called four times, in the same order on
        every rank."""
        sel, scores = self.select_local(batch=batch, q_seq=q_seq, q_pos=q_pos,
                                        local_page_table=local_page_table, num_pages=num_pages,
                                        idx_q=idx_q, idx_w=idx_w, kcomp_pool=kcomp_pool)
        part_sel, part_scores = all_gather(sel), all_gather(scores)
        o, l = self.merge_and_attend(part_sel, part_scores, max_pos=max_pos, q=q, k_pool=k_pool,
                                     v_pool=v_pool, decode=decode)
        part_out, part_lse = all_gather(o), all_gather(l)
        return self.combine(part_out, part_lse, out, lse)


__all__ = ["ContextParallelStep", "Shard", "Rows", "LibOps", "dist_all_gather"]
