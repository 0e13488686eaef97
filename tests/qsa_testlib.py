"""Helpers for the parity tests: run the CUDA path through the C-ABI binding, and compute the
oracle's answer for the same seeded inputs on the host.  The two sides share only the input
generator (qsa_synth); every expected value comes from oracle/."""
from __future__ import annotations

import functools
import math

import numpy as np

from oracle import qsa_oracle as orc
from qsa_synth import CONFIGS, Config, HostInputs

# tolerances (attention allclose form; indexer scores relative to the row's k-th score)
ATTN_ATOL, ATTN_RTOL = 2e-2, 1e-2
SCORE_RTOL = 1e-3


def qsa_config(c: Config, score_path: int = 0, topk: int | None = None):
    from learned_block_sparse_qsa_b200 import QsaConfig

    return QsaConfig.make(c.Hq, c.Hkv, c.D, c.Di, topk=c.topk if topk is None else topk, Hi=c.Hi,
                          block=c.block, page=c.page, score_path=score_path)


class Run:
    """Device inputs + runner + outputs of one workload."""

    def __init__(self, c: Config, integer=False, score_path=0, topk=None, device="cuda"):
        import torch

        from learned_block_sparse_qsa_b200 import QsaRunner
        from qsa_synth.device import DeviceInputs

        self.torch = torch
        self.c = c if topk is None else c.replace(topk=topk)
        self.di = DeviceInputs(self.c, integer, device)
        self.cfg = qsa_config(self.c, score_path)
        self.runner = QsaRunner(self.cfg, device)
        d = self.di
        self.b = self.runner.batch(batch=c.batch, num_q=c.num_q, max_pages=c.max_pages,
                                   num_pages=c.num_pages, max_pos=c.ctx - 1, q_seq=d.q_seq,
                                   q_pos=d.q_pos, page_table=d.page_table)
        k1 = self.c.topk + 1
        self.sel = torch.empty(c.num_q, k1, dtype=torch.int32, device=device)
        self.n_sel = torch.empty(c.num_q, dtype=torch.int32, device=device)
        self.sel_scores = torch.empty(c.num_q, k1, dtype=torch.float32, device=device)
        self.out = torch.empty_like(d.q)
        self.lse = torch.empty(c.num_q, c.Hq, dtype=torch.float32, device=device)
        self.setup_prefix()

    def setup_prefix(self):
        """Compressed keys of every block before the step's new tokens (not part of the step)."""
        from learned_block_sparse_qsa_b200 import QsaBatch

        for s in range(self.c.batch):
            rows, seq, pos = self.di.prefix_rows(s)
            if rows.shape[0]:
                self.runner.compress(self.b, rows, seq, pos, self.di.kcomp_pool)
        self.torch.cuda.synchronize()
        _ = QsaBatch

    def step(self, decode=None, splits=0, compress=True):
        """compress=False skips compressing the step's new tokens (for steps whose new tokens do
        not fill whole blocks; their blocks are never candidates of these rows)."""
        d = self.di
        decode = (self.c.mode == "decode") if decode is None else decode
        kw = dict(q=d.q, idx_q=d.idx_q, idx_w=d.idx_w, kcomp_pool=d.kcomp_pool, k_pool=d.k_pool,
                  v_pool=d.v_pool, out=self.out, sel=self.sel, n_sel=self.n_sel, lse=self.lse,
                  sel_scores=self.sel_scores)
        if compress:
            kw.update(idx_k_new=d.idx_k_new, new_seq=d.new_seq, new_pos=d.new_pos)
        if decode:
            self.runner.decode(self.b, splits=splits, **kw)
        else:
            self.runner.prefill(self.b, **kw)
        self.torch.cuda.synchronize()
        return self

    def redo_flags(self):
        """The score call's redo flags (int32 [num_q], 1 = recomputed by the exact streaming
        kernel) read from the runner's workspace, or None when the path keeps none."""
        return self.runner.redo_flags(self.b)

    def numpy(self):
        t = self.torch
        return dict(sel=self.sel.cpu().numpy(), n_sel=self.n_sel.cpu().numpy(),
                    sel_scores=self.sel_scores.cpu().numpy(),
                    out=self.out.view(t.int16).cpu().numpy().view(np.uint16),
                    lse=self.lse.cpu().numpy())


@functools.lru_cache(maxsize=16)
def host(c: Config, integer: bool) -> HostInputs:
    return HostInputs(c, integer)


@functools.lru_cache(maxsize=8)
def host_kcomp(c: Config, integer: bool, s: int) -> np.ndarray:
    """Oracle compression of every complete block of sequence s (bf16 bits [ctx//4, Di])."""
    h = host(c, integer)
    return orc.compress(h.idx_k(s, 0, c.ctx))


def score_bound(kc_bits, iq_bits, iw_bits, n: int) -> np.ndarray:
    """Absolute error allowance of an fp32 block score: the textbook bound on an fp32 sum of Di
    exact products, Di * 2^-24 * sum|q_i k_i|, summed over heads with their weights, doubled for
    the head sum and weighting.  Needed where a score (or the 512th score) is near zero."""
    k = np.abs(orc.bf16_to_f64(kc_bits[:n]))
    q = np.abs(orc.bf16_to_f64(iq_bits))
    w = np.abs(orc.bf16_to_f64(iw_bits))
    di = k.shape[1] if n else 1
    return 2.0 * di * 2.0 ** -24 * ((k @ q.T) @ w)


def oracle_select_row(c: Config, integer: bool, r: int, topk: int | None = None):
    """(sel, all candidate scores, their fp32 error allowance) of query row r, by the oracle."""
    h = host(c, integer)
    q_seq, q_pos = h.rows()
    s, t = int(q_seq[r]), int(q_pos[r])
    kc = host_kcomp(c, integer, s)
    iq, iw = h.idx_q([r])[0], h.idx_w([r])[0]
    sel, sc = orc.qsa_select(kc, iq, iw, t, c.topk if topk is None else topk)
    return sel, sc, score_bound(kc, iq, iw, t // 4)


def oracle_attend_row(c: Config, integer: bool, r: int, sel: np.ndarray):
    """Oracle attention of row r over the positions of the given selection."""
    h = host(c, integer)
    q_seq, q_pos = h.rows()
    s, t = int(q_seq[r]), int(q_pos[r])
    pos = orc.expand(np.asarray(sel), t)
    k, v = h.kv(s, pos)
    return orc.attend(h.q([r])[0], k, v)


def oracle_dense_row(c: Config, integer: bool, r: int):
    h = host(c, integer)
    q_seq, q_pos = h.rows()
    s, t = int(q_seq[r]), int(q_pos[r])
    k, v = h.kv(s, np.arange(t + 1))
    return orc.dense_causal(h.q([r])[0], k, v, t)


def positive_int_weights(w_bits: np.ndarray) -> np.ndarray:
    """Head weights in {1, 2, 3}, from the generator's integer weights in [-3, 3] (|w| mod 3 + 1),
    as bf16 bits.  Positive weights are what the pages' workloads use; with weights <= 0 a row's
    scores collapse onto a few values and the fast kernel hands the row to the exact one."""
    w = orc.bf16_to_f64(w_bits)
    return orc.f64_to_bf16_bits(np.abs(w) % 3 + 1)


TC_KEEP = 24  # the tensor-core kernel's threshold rank: best sampled scores kept per half-row


def tc_redo_model(scores: np.ndarray, topk: int, nsamp: int, cap: int = 2048, tile: int = 128,
                  sample_every: int = 32, keep: int = TC_KEEP) -> bool:
    """Whether the tensor-core indexer kernel hands a row to the exact streaming kernel, for a row
    whose fp32 candidate scores are known exactly (integer inputs).  A model of the kernel's
    branch, not of the method: each row is split into two column halves of every 128-block tile;
    rows of more than 2 * cap candidates (and more than topk) take as threshold the smaller of the
    two halves' keep-th best score over the sampled tiles (tiles 0, 32, ..., 32 * (nsamp - 1));
    every key at or above it is kept; the row is redone when a half keeps more than cap keys or
    the row keeps fewer than min(topk, candidates)."""
    lim = scores.shape[0]
    if lim == 0:
        return False
    b = np.arange(lim)
    half = (b % tile) // (tile // 2)
    tau = -np.inf
    if lim > topk and lim > 2 * cap:
        sampled = ((b // tile) % sample_every == 0) & ((b // tile) // sample_every < nsamp)
        thr = []
        for hf in (0, 1):
            v = np.sort(scores[sampled & (half == hf)])[::-1]
            thr.append(v[keep - 1] if v.size >= keep else -np.inf)
        tau = min(thr)
    keep = scores >= tau
    n0, n1 = int(np.sum(keep & (half == 0))), int(np.sum(keep & (half == 1)))
    return n0 > cap or n1 > cap or n0 + n1 < min(topk, lim)


def kth_score(scores: np.ndarray, k: int) -> float:
    if scores.size == 0:
        return 0.0
    k = min(k, scores.size)
    return float(np.partition(scores, scores.size - k)[scores.size - k])


def check_selection(gsel_row, gn, gsc_row, ref_sel, ref_scores, t, topk, exact: bool, bound=None):
    """GPU selection of one row against the oracle's.  Exact mode (integer inputs): identical
    blocks and identical fp32 scores.  Otherwise: same count and tail; every selected block's
    score within SCORE_RTOL * max(|s|, |s_k|) + bound_b of the oracle's, s_k the k-th score and
    bound_b the fp32 accumulation allowance of score_bound(); blocks selected by only one side must
    lie within SCORE_RTOL * |s_k| + bound_b of s_k."""
    n = min(topk, t // 4) + 1
    assert gn == n, (gn, n)
    g = np.asarray(gsel_row[:n], dtype=np.int64)
    assert g[-1] == t // 4 and np.all(np.diff(g) > 0), g
    assert np.all(np.asarray(gsel_row[n:]) == -1)
    gs = np.asarray(gsc_row[: n - 1], dtype=np.float64)
    if exact:
        assert np.array_equal(g, ref_sel), (g, ref_sel)
        assert np.array_equal(gs, ref_scores[g[:-1]])
        return 0
    sk = kth_score(ref_scores, topk)
    eb = np.zeros_like(ref_scores) if bound is None else np.asarray(bound, dtype=np.float64)
    gi = g[:-1]
    tol = SCORE_RTOL * np.maximum(np.abs(ref_scores[gi]), abs(sk)) + eb[gi]
    err = np.abs(gs - ref_scores[gi])
    bad = np.nonzero(err > tol)[0]
    assert bad.size == 0, ("score mismatch", [(int(gi[i]), float(gs[i]), float(ref_scores[gi[i]]),
                                               float(tol[i])) for i in bad[:8]], sk)
    a, b = set(gi.tolist()), set(ref_sel[:-1].tolist())
    diff = a ^ b
    for blk in diff:
        assert abs(ref_scores[blk] - sk) <= SCORE_RTOL * abs(sk) + eb[blk] + 1e-7, (blk, ref_scores[blk], sk)
    return len(diff)


def check_attention(gout_row_bits, glse_row, ref_o, ref_lse):
    go = orc.bf16_to_f64(gout_row_bits)
    assert np.allclose(go, ref_o, atol=ATTN_ATOL, rtol=ATTN_RTOL), float(np.max(np.abs(go - ref_o)))
    if glse_row is not None:
        assert np.allclose(glse_row, ref_lse, atol=ATTN_ATOL, rtol=ATTN_RTOL)


def sample_rows(c: Config, n: int) -> list[int]:
    """Evenly spaced query rows including the first and the last."""
    if c.num_q <= n:
        return list(range(c.num_q))
    return sorted(set(np.linspace(0, c.num_q - 1, n).round().astype(int).tolist()))


__all__ = ["CONFIGS", "Run", "positive_int_weights", "tc_redo_model", "host_kcomp", "score_bound", "oracle_select_row", "oracle_attend_row",
           "oracle_dense_row", "check_selection", "check_attention", "sample_rows", "math"]
