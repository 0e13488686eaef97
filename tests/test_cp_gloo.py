"""Host logic of the context-parallel step (learned_block_sparse_qsa_b200.context_parallel) on CPU
with two gloo ranks: shard coordinates, the order and layout of the gathered candidate lists and
partials, the shards' block offsets, and the final log-sum-exp merge.  The kernels are replaced by
stand-ins built on the oracle (CPU tensors, the kernels' documented contracts); the ranks' merged
output and global selection must equal the oracle's single-device layer."""
import math
import multiprocessing as mp
import os
import socket

import numpy as np
import pytest

L, B, HQ, HKV, D, DI, TOPK = 256, 1, 4, 1, 64, 32, 8
ROWS = [3, 50, 100, 127, 128, 131, 200, 254, 255]


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _data():
    import torch

    g = torch.Generator().manual_seed(7)
    bf = lambda *s: torch.randn(*s, generator=g).to(torch.bfloat16)   # noqa: E731
    k, v = bf(L, HKV, D), bf(L, HKV, D)
    idx_k = bf(L, DI)
    idx_q, q = bf(len(ROWS), 4, DI), bf(len(ROWS), HQ, D)
    idx_w = torch.rand(len(ROWS), 4, generator=g).to(torch.bfloat16)
    return k, v, idx_k, idx_q, idx_w, q


def _bits(t):
    import torch

    return t.view(torch.int16).numpy().view(np.uint16)


class OracleOps:
    """CPU stand-ins for the kernels, on this rank's shard only (keys/values of its positions)."""

    def __init__(self, shard_k, shard_v, shard_kc, err):
        self.k, self.v, self.kc, self.err = shard_k, shard_v, shard_kc, err

    def positions(self, q_pos, shard, pos_sel, pos_attn):
        for i, t in enumerate(q_pos.tolist()):
            pos_sel[i] = 0 if t < shard.start else (t - shard.start if t < shard.start + shard.length else shard.length)
            pos_attn[i] = 0 if t < shard.start else min(t - shard.start, shard.length - 1)

    def select(self, rows, idx_q, idx_w, kcomp_pool, sel, n_sel, scores):
        from oracle import qsa_oracle as orc

        for i, t in enumerate(rows.q_pos.tolist()):
            s, sc = orc.qsa_select(self.kc, _bits(idx_q[i]), _bits(idx_w[i]), t, TOPK)
            sel[i] = -1
            scores[i] = float("nan")
            sel[i, :len(s)] = __import__("torch").tensor(s)
            scores[i, :len(s) - 1] = __import__("torch").tensor(sc[s[:-1]])
            scores[i, len(s) - 1] = float("inf")
            n_sel[i] = len(s)

    def merge(self, rows, part_sel, part_scores, part_lo, shard, sel, n_sel, scores, local_sel, local_n):
        import torch

        for i, t in enumerate(rows.q_pos.tolist()):
            blk, sc = [], []
            for p in range(part_sel.shape[0]):
                for b, s in zip(part_sel[p, i].tolist(), part_scores[p, i].tolist()):
                    if b >= 0 and math.isfinite(s):
                        blk.append(b + part_lo[p])
                        sc.append(s)
            blk, sc = np.array(blk, dtype=np.int64), np.array(sc)
            order = np.lexsort((blk, -sc))[: min(TOPK, t // 4)]
            win = np.sort(blk[order])
            full = np.concatenate([win, [t // 4]])
            sel[i] = -1
            sel[i, :len(full)] = torch.tensor(full)
            n_sel[i] = len(full)
            loc = [b - shard.block_lo for b in full if shard.block_lo <= b < shard.block_hi]
            local_sel[i] = -1
            local_sel[i, :len(loc)] = torch.tensor(loc, dtype=torch.int32)
            local_n[i] = len(loc)

    def attend(self, rows, q, k_pool, v_pool, sel, n_sel, out, lse, decode):
        import torch

        from oracle import qsa_oracle as orc

        for i, t in enumerate(rows.q_pos.tolist()):
            n = int(n_sel[i])
            pos = orc.expand(sel[i, :n].numpy(), t) if n else np.zeros(0, dtype=np.int64)
            if pos.size == 0:
                out[i] = 0
                lse[i] = float("-inf")
                continue
            o, l = orc.attend(_bits(q[i]), _bits(self.k[pos]), _bits(self.v[pos]))
            out[i] = torch.tensor(o, dtype=torch.float64).to(torch.bfloat16)
            lse[i] = torch.tensor(l)

    def merge_partials(self, part_out, part_lse, out, lse):
        import torch

        m = part_lse.max(dim=0).values
        w = torch.exp(part_lse - m).nan_to_num(0.0)
        tot = w.sum(0)
        o = (w[..., None] * part_out.float()).sum(0) / tot[..., None]
        out.copy_(o.to(torch.bfloat16))
        if lse is not None:
            lse.copy_(m + torch.log(tot))

    def error_bits(self):
        return 0


def _rank(rank: int, world: int, port: int, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime

    import torch
    import torch.distributed as dist

    from learned_block_sparse_qsa_b200 import QsaConfig
    from learned_block_sparse_qsa_b200.context_parallel import ContextParallelStep, Shard, dist_all_gather
    from oracle import qsa_oracle as orc

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        k, v, idx_k, idx_q, idx_w, qq = _data()
        n = L // world
        shards = [Shard(r * n, n) for r in range(world)]
        sh = shards[rank]
        kc_local = orc.compress(_bits(idx_k[sh.start:sh.start + sh.length]))
        ops = OracleOps(k[sh.start:sh.start + n], v[sh.start:sh.start + n], kc_local, None)
        cfg = QsaConfig.make(HQ, HKV, D, DI, topk=TOPK)
        cp = ContextParallelStep(cfg, shards, rank, device="cpu", ops=ops)
        q_pos = torch.tensor(ROWS, dtype=torch.int32)
        q_seq = torch.zeros(len(ROWS), dtype=torch.int32)
        lpt = torch.zeros(B, n // 64 + 1, dtype=torch.int32)
        out = torch.empty(len(ROWS), HQ, D, dtype=torch.bfloat16)
        lse = torch.empty(len(ROWS), HQ, dtype=torch.float32)
        cp.step(dist_all_gather, batch=B, q_seq=q_seq, q_pos=q_pos, max_pos=L - 1,
                local_page_table=lpt, num_pages=1, idx_q=idx_q, idx_w=idx_w, kcomp_pool=None,
                q=qq, k_pool=None, v_pool=None, out=out, lse=lse)
        q.put((rank, cp.sel.numpy().tolist(), cp.n_sel.numpy().tolist(), out.float().numpy(), lse.numpy()))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_reproduce_the_single_device_layer():
    from oracle import qsa_oracle as orc

    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=180) for _ in procs), key=lambda x: x[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    k, v, idx_k, idx_q, idx_w, qq = _data()
    kc = orc.compress(_bits(idx_k))
    for i, t in enumerate(ROWS):
        o, l, sel = orc.qsa_row(kc, _bits(idx_q[i]), _bits(idx_w[i]), _bits(qq[i]), _bits(k), _bits(v), t, TOPK)
        for _, gsel, gn, gout, glse in res:
            assert gsel[i][: gn[i]] == sel.tolist()
            assert np.allclose(gout[i], o, atol=2e-2, rtol=1e-2)
            assert np.allclose(glse[i], l, atol=1e-4, rtol=1e-4)
