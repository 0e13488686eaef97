"""Seeded synthetic inputs for the QSA layer: the workloads and their host-side generator.

This package is the input generator shared by the CUDA path and the CPU oracle.  It holds
none of the attention method's arithmetic: it only defines the shapes of the workloads, the
counter-based pseudo-random values that fill them, the page tables, and the planted "needle"
blocks.  Every value is addressed by logical coordinates (sequence, position, head, dim), so
the host can regenerate any element of a multi-GiB device tensor without copying it back.

The generator (bit-identical to ``gen_core.h`` on the device):
  key(seed, tid) = SplitMix64 finaliser of ((seed << 20) ^ tid) + gamma
  hash(i)        = SplitMix64 finaliser of key + (i + 1) * gamma
SplitMix64 is the generator of Steele, Lea & Flood (OOPSLA 2014) with the finaliser constants of
Vigna's public-domain ``splitmix64.c``.  The three distributions are described in gen_core.h.

Workload shapes follow the settings the pages give for the QSA layer (Qwen3.8-Flash-Next
article, section "Three speed claims, three different experiments": prefill of the last chunk
at one million tokens with batch 1; decode with batch 4 plus three extra multi-token-prediction
steps), and the needle construction follows the evaluation advice of the same article (section
"What a serious evaluation should preserve": hide evidence at varied positions and check it
survives selection).
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

GAMMA = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)

NORMAL, UNIFORM, INT3 = 0, 1, 2

# tensor ids of the generator streams
TID_Q, TID_K, TID_V, TID_IDXQ, TID_IDXK, TID_IDXW = 1, 2, 3, 4, 5, 6
TID_NEEDLE_DIR, TID_NEEDLE_Z, TID_NEEDLE_PICK, TID_NEEDLE_BLOCK, TID_PAGE_PERM = 7, 8, 9, 10, 11


def _mix(z: np.ndarray) -> np.ndarray:
    z = (z ^ (z >> np.uint64(30))) * _M1
    z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def stream_key(seed: int, tid: int) -> np.uint64:
    with np.errstate(over="ignore"):
        x = np.array([((seed << 20) ^ tid) & 0xFFFFFFFFFFFFFFFF], dtype=np.uint64)
        return _mix(x + GAMMA)[0]


def hashes(seed: int, tid: int, idx) -> np.ndarray:
    """uint64 hash of elements ``idx`` (int array) of stream (seed, tid)."""
    key = stream_key(seed, tid)
    i = np.asarray(idx, dtype=np.uint64)
    with np.errstate(over="ignore"):
        return _mix(key + (i + np.uint64(1)) * GAMMA)


def f32_to_bf16_bits(f: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit pattern, round to nearest even (finite inputs)."""
    u = np.ascontiguousarray(f, dtype=np.float32).view(np.uint32).astype(np.uint64)
    return ((u + np.uint64(0x7FFF) + ((u >> np.uint64(16)) & np.uint64(1))) >> np.uint64(16)).astype(
        np.uint16
    )


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def values_bf16(seed: int, tid: int, idx, dist: int) -> np.ndarray:
    """bf16 bit patterns (uint16) of elements ``idx`` of stream (seed, tid)."""
    h = hashes(seed, tid, idx)
    if dist == NORMAL:
        m = np.uint64(0xFFFF)
        s = (h & m).astype(np.int64) + ((h >> np.uint64(16)) & m).astype(np.int64)
        s += ((h >> np.uint64(32)) & m).astype(np.int64) + ((h >> np.uint64(48)) & m).astype(np.int64)
        f = (s - 131070).astype(np.float32) * np.float32(1.7320508075688772)
        f = f * np.float32(1.52587890625e-05)
        return f32_to_bf16_bits(f)
    if dist == UNIFORM:
        f = (h >> np.uint64(40)).astype(np.float32) * np.float32(5.9604644775390625e-08)
        return f32_to_bf16_bits(f)
    if dist == INT3:
        v = ((h >> np.uint64(32)) % np.uint64(7)).astype(np.int64) - 3
        return f32_to_bf16_bits(v.astype(np.float32))
    raise ValueError(dist)


_HOST_LIB = None


def _host_lib():
    """libqsa_synth.so's host fill (the same values, computed by C++ threads), or None when the
    library has not been built; the numpy path above is then used."""
    global _HOST_LIB
    if _HOST_LIB is None:
        import ctypes
        import os

        path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libqsa_synth.so")
        lib = False
        if os.path.exists(path):
            try:
                lib = ctypes.CDLL(path)
                f = lib.qsyn_fill_rows_host
                f.restype = ctypes.c_int
                f.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64,
                              ctypes.c_uint64, ctypes.c_uint64, ctypes.c_int, ctypes.c_int]
            except (OSError, AttributeError):
                lib = False
        _HOST_LIB = lib
    return _HOST_LIB or None


def rows_bf16(seed: int, tid: int, starts, width: int, dist: int) -> np.ndarray:
    """bf16 bits [len(starts), width]: row r holds elements starts[r] .. starts[r] + width - 1 of
    stream (seed, tid).  Equal to values_bf16 of those indices (checked by tests/test_synth.py)."""
    starts = np.ascontiguousarray(starts, dtype=np.int64).reshape(-1)
    lib = _host_lib()
    if lib is None or starts.size * width < 4096:
        idx = starts[:, None] + np.arange(width, dtype=np.int64)[None, :]
        return values_bf16(seed, tid, idx.reshape(-1), dist).reshape(starts.size, width)
    out = np.empty((starts.size, width), dtype=np.uint16)
    rc = lib.qsyn_fill_rows_host(out.ctypes.data, starts.ctypes.data, starts.size, width, seed, tid,
                                 dist, 0)
    if rc != 0:
        raise RuntimeError("qsyn_fill_rows_host failed")
    return out


def values_f32(seed: int, tid: int, idx, dist: int) -> np.ndarray:
    return bf16_bits_to_f32(values_bf16(seed, tid, idx, dist))


def round_f64_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp64 values (needle construction only) to bf16 bits via fp32."""
    return f32_to_bf16_bits(np.asarray(x, dtype=np.float64).astype(np.float32))


# --------------------------------------------------------------------------------------------
# workloads


@dataclasses.dataclass(frozen=True)
class Config:
    """One QSA-layer workload.  Query rows are sequence-major: row r = s * n_new + i holds
    position ctx - n_new + i of sequence s.  Every sequence holds ``ctx`` tokens in its cache,
    the last ``n_new`` of which are the new tokens of this step."""

    name: str
    mode: str  # "prefill" | "decode"
    batch: int
    ctx: int
    n_new: int
    Hq: int
    Hkv: int
    D: int
    Hi: int
    Di: int
    topk: int = 512
    block: int = 4
    page: int = 64
    needles: int = 0
    shuffle_pages: bool = False
    seed: int = 0x05A0

    @property
    def num_q(self) -> int:
        return self.batch * self.n_new

    @property
    def max_pages(self) -> int:
        return (self.ctx + self.page - 1) // self.page

    @property
    def num_pages(self) -> int:
        return self.batch * self.max_pages

    @property
    def ctx_start(self) -> int:
        return self.ctx - self.n_new

    def replace(self, **kw) -> "Config":
        return dataclasses.replace(self, **kw)


# The five workloads: a small oracle-check layer and the pages' prefill/decode settings at
# 131,072 / 262,144 / 1,048,576 tokens of context.
CONFIGS = {
    "C1": Config("C1_prefill_T4096_4q1kv_d64", "prefill", 1, 4096, 4096, 4, 1, 64, 4, 32,
                 seed=0x05A1),
    "C2": Config("C2_prefill_chunk16384_ctx131072", "prefill", 1, 131072, 16384, 32, 4, 128, 4, 128,
                 needles=64, shuffle_pages=True, seed=0x05A2),
    "C3": Config("C3_decode_b4x4_ctx262144", "decode", 4, 262144, 4, 32, 4, 128, 4, 128,
                 needles=64, shuffle_pages=True, seed=0x05A3),
    "C4": Config("C4_prefill_chunk16384_ctx1048576", "prefill", 1, 1048576, 16384, 32, 4, 128, 4,
                 128, needles=64, shuffle_pages=True, seed=0x05A4),
    "C5": Config("C5_decode_b4x4_ctx1048576", "decode", 4, 1048576, 4, 32, 4, 128, 4, 128,
                 needles=64, shuffle_pages=True, seed=0x05A5),
}


def dists(integer: bool) -> dict:
    """Distribution of each tensor: N(0,1) stand-in with U(0,1) head weights, or all
    integers in [-3, 3] (the pass on which fp32 scores are exact)."""
    if integer:
        return dict(q=INT3, k=INT3, v=INT3, idx_q=INT3, idx_k=INT3, idx_w=INT3)
    return dict(q=NORMAL, k=NORMAL, v=NORMAL, idx_q=NORMAL, idx_k=NORMAL, idx_w=UNIFORM)


class HostInputs:
    """Host-side view of a workload: regenerates any element on demand (numpy)."""

    def __init__(self, cfg: Config, integer: bool = False):
        self.cfg = cfg
        self.integer = integer
        self.dist = dists(integer)
        self._needles = None
        self._page_table = None

    # ---- structure
    def rows(self):
        c = self.cfg
        q_seq = np.repeat(np.arange(c.batch, dtype=np.int32), c.n_new)
        q_pos = np.tile(np.arange(c.ctx_start, c.ctx, dtype=np.int32), c.batch)
        return q_seq, q_pos

    def page_table(self) -> np.ndarray:
        """int32 [batch, max_pages]: identity, or a seeded Fisher-Yates shuffle of the pool."""
        if self._page_table is None:
            c = self.cfg
            n = c.num_pages
            perm = np.arange(n, dtype=np.int64)
            if c.shuffle_pages and n > 1:
                h = hashes(c.seed, TID_PAGE_PERM, np.arange(n, dtype=np.int64))
                for i in range(n - 1, 0, -1):
                    j = int(h[i] % np.uint64(i + 1))
                    perm[i], perm[j] = perm[j], perm[i]
            self._page_table = perm.reshape(c.batch, c.max_pages).astype(np.int32)
        return self._page_table

    def page_owner(self) -> np.ndarray:
        c = self.cfg
        pt = self.page_table().reshape(-1)
        owner = np.full(c.num_pages, -1, dtype=np.int32)
        owner[pt] = np.arange(pt.size, dtype=np.int32)
        return owner

    # ---- needles
    def needles(self):
        """Planted blocks: per sequence, ``needles`` distinct block ids before the new tokens,
        each with a unit direction u_j; the 4 raw indexer keys of the block are sqrt(Di)*u_j.
        Each query row independently (p = 1/4) picks a needle j and gets indexer heads
        sqrt(Di)*(0.8*u_j + 0.6*z_h), z_h a unit vector orthogonal to u_j (cosine 0.8)."""
        if self._needles is not None:
            return self._needles
        c = self.cfg
        out = {"blocks": [], "key_rows": [], "q_rows": {}, "q_vals": {}}
        if c.needles == 0 or self.integer:
            self._needles = out
            return out
        nblk_range = (c.ctx_start // c.block) if c.mode == "prefill" else (c.ctx // c.block - 1)
        nblk_range = max(nblk_range, 1)
        count = min(c.needles, nblk_range)
        sqrt_di = math.sqrt(c.Di)
        dirs = np.zeros((c.batch, count, c.Di), dtype=np.float64)
        for s in range(c.batch):
            picked, i = [], 0
            while len(picked) < count:
                hs = hashes(c.seed, TID_NEEDLE_BLOCK, np.arange(i, i + 4 * count) + s * (1 << 32))
                for hv in hs:
                    b = int(hv % np.uint64(nblk_range))
                    if b not in picked:
                        picked.append(b)
                        if len(picked) == count:
                            break
                i += 4 * count
            out["blocks"].append(np.array(picked, dtype=np.int64))
            idx = (np.arange(count * c.Di, dtype=np.int64) + s * count * c.Di)
            u = values_f32(c.seed, TID_NEEDLE_DIR, idx, NORMAL).astype(np.float64).reshape(count, c.Di)
            u /= np.linalg.norm(u, axis=1, keepdims=True)
            dirs[s] = u
            out["key_rows"].append(round_f64_to_bf16_bits(sqrt_di * u))
        out["dirs"] = dirs
        q_seq, q_pos = self.rows()
        pick = hashes(c.seed, TID_NEEDLE_PICK, np.arange(c.num_q, dtype=np.int64))
        for r in range(c.num_q):
            if int(pick[r] % np.uint64(4)) != 0:
                continue
            s = int(q_seq[r])
            j = int((pick[r] >> np.uint64(8)) % np.uint64(count))
            u = dirs[s, j]
            zidx = (np.arange(c.Hi * c.Di, dtype=np.int64) + r * c.Hi * c.Di)
            z = values_f32(c.seed, TID_NEEDLE_Z, zidx, NORMAL).astype(np.float64).reshape(c.Hi, c.Di)
            z -= (z @ u)[:, None] * u[None, :]
            z /= np.linalg.norm(z, axis=1, keepdims=True)
            qv = sqrt_di * (0.8 * u[None, :] + 0.6 * z)
            out["q_rows"][r] = j
            out["q_vals"][r] = round_f64_to_bf16_bits(qv)
        self._needles = out
        return out

    # ---- tensors (bf16 bit patterns, uint16)
    def _lin(self, tid, dist, starts, width):
        return rows_bf16(self.cfg.seed, tid, starts, width, dist)

    def q(self, rows) -> np.ndarray:
        c = self.cfg
        q_seq, q_pos = self.rows()
        rows = np.asarray(rows, dtype=np.int64)
        starts = ((q_seq[rows].astype(np.int64) * c.ctx + q_pos[rows]) * c.Hq) * c.D
        return self._lin(TID_Q, self.dist["q"], starts, c.Hq * c.D).reshape(len(rows), c.Hq, c.D)

    def idx_q(self, rows) -> np.ndarray:
        c = self.cfg
        q_seq, q_pos = self.rows()
        rows = np.asarray(rows, dtype=np.int64)
        starts = ((q_seq[rows].astype(np.int64) * c.ctx + q_pos[rows]) * c.Hi) * c.Di
        out = self._lin(TID_IDXQ, self.dist["idx_q"], starts, c.Hi * c.Di).reshape(len(rows), c.Hi, c.Di)
        nd = self.needles()
        for i, r in enumerate(rows):
            if int(r) in nd["q_rows"]:
                out[i] = nd["q_vals"][int(r)]
        return out

    def idx_w(self, rows) -> np.ndarray:
        c = self.cfg
        q_seq, q_pos = self.rows()
        rows = np.asarray(rows, dtype=np.int64)
        starts = (q_seq[rows].astype(np.int64) * c.ctx + q_pos[rows]) * c.Hi
        return self._lin(TID_IDXW, self.dist["idx_w"], starts, c.Hi)

    def idx_k(self, s: int, pos0: int, pos1: int) -> np.ndarray:
        """Raw indexer keys of positions [pos0, pos1) of sequence s: bf16 [n, Di]."""
        c = self.cfg
        n = pos1 - pos0
        starts = (s * c.ctx + pos0 + np.arange(n, dtype=np.int64)) * c.Di
        out = rows_bf16(c.seed, TID_IDXK, starts, c.Di, self.dist["idx_k"])
        nd = self.needles()
        if nd["blocks"]:
            for j, blk in enumerate(nd["blocks"][s]):
                for i in range(c.block):
                    p = int(blk) * c.block + i
                    if pos0 <= p < pos1:
                        out[p - pos0] = nd["key_rows"][s][j]
        return out

    def kv(self, s: int, positions) -> tuple[np.ndarray, np.ndarray]:
        """K and V rows of sequence s at the given positions: bf16 [n, Hkv, D] each."""
        c = self.cfg
        positions = np.asarray(positions, dtype=np.int64)
        starts = (s * c.ctx + positions) * (c.Hkv * c.D)
        k = self._lin(TID_K, self.dist["k"], starts, c.Hkv * c.D).reshape(-1, c.Hkv, c.D)
        v = self._lin(TID_V, self.dist["v"], starts, c.Hkv * c.D).reshape(-1, c.Hkv, c.D)
        return k, v
