"""Python binding of libqsa, the B200 (sm_100a) Qwen Sparse Attention layer.

Argument marshalling only: every function here has the name and arguments of the C-ABI entry
point in ``include/qsa.h`` and forwards device pointers (torch tensors or raw integers) to
``libqsa.so``; every step of the layer runs in that library's CUDA kernels.  Importing this
package fails loudly when the library has not been built -- there is no CPU fallback.

    from learned_block_sparse_qsa_b200 import QsaConfig, QsaBatch, qsa_index_score_topk, ...
"""
from __future__ import annotations

import ctypes
import os
from ctypes import c_float, c_int32, c_int64, c_size_t, c_void_p

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libqsa.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python learned_block_sparse_qsa_b200/build.py` "
        "(nvcc, sm_100a). libqsa has no CPU fallback.")
_lib = ctypes.CDLL(LIB_PATH)

QSA_OK, QSA_ERR_INVALID_ARG, QSA_ERR_UNSUPPORTED, QSA_ERR_WORKSPACE, QSA_ERR_CUDA = 0, 1, 2, 3, 4
QSA_OP_INDEX_SCORE_TOPK, QSA_OP_SPARSE_ATTN_DECODE, QSA_OP_DENSE_ATTN_DECODE = 1, 2, 3
QSA_OP_MERGE_CANDIDATES, QSA_OP_DECODE_STEP, QSA_OP_DISTILL_KL = 4, 5, 6
DEVERR = {"SEQ": 1, "POS": 2, "PAGE": 4, "GROUP": 8, "SEL": 16, "TIMEOUT": 32, "INTERNAL": 64}


class QsaConfig(ctypes.Structure):
    _fields_ = [("num_q_heads", c_int32), ("num_kv_heads", c_int32), ("head_dim", c_int32),
                ("idx_heads", c_int32), ("idx_dim", c_int32), ("block_tokens", c_int32),
                ("topk_blocks", c_int32), ("page_tokens", c_int32), ("softmax_scale", c_float),
                ("score_path", c_int32)]

    @classmethod
    def make(cls, Hq, Hkv, D, Di, topk=512, Hi=4, block=4, page=64, scale=0.0, score_path=0):
        return cls(Hq, Hkv, D, Hi, Di, block, topk, page, scale, score_path)


class QsaBatch(ctypes.Structure):
    _fields_ = [("batch", c_int32), ("num_q", c_int32), ("max_pages_per_seq", c_int32),
                ("num_pages", c_int32), ("max_pos", c_int32), ("q_seq", c_void_p),
                ("q_pos", c_void_p), ("page_table", c_void_p), ("err_flag", c_void_p)]


class QsaError(RuntimeError):
    def __init__(self, status: int, where: str):
        msg = _lib.qsa_status_string(status).decode()
        super().__init__(f"{where}: {msg} (status {status})")
        self.status = status


def _p(x):
    """Device (or host) address of a tensor / int / None."""
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(stream):
    if stream is None:
        import torch

        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


_S = ctypes.POINTER(QsaConfig)
_B = ctypes.POINTER(QsaBatch)
_SIGS = {
    "qsa_status_string": (ctypes.c_char_p, [c_int32]),
    "qsa_version": (c_int32, []),
    "qsa_workspace_size": (c_int32, [_S, _B, c_int32, c_int32, ctypes.POINTER(c_size_t)]),
    "qsa_index_compress": (c_int32, [_S, _B, c_void_p, c_void_p, c_void_p, c_int32, c_void_p, c_void_p]),
    "qsa_index_score_topk": (c_int32, [_S, _B, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                       c_void_p, c_void_p, c_size_t, c_void_p]),
    "qsa_index_score_redo_flags": (c_int32, [_S, _B, c_void_p, c_size_t, ctypes.POINTER(c_void_p)]),
    "qsa_index_scores": (c_int32, [_S, _B, c_void_p, c_void_p, c_void_p, c_void_p, c_int64, c_void_p]),
    "qsa_sparse_attn_prefill": (c_int32, [_S, _B, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                          c_void_p, c_void_p, c_void_p]),
    "qsa_sparse_attn_decode": (c_int32, [_S, _B, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                         c_void_p, c_void_p, c_int32, c_void_p, c_size_t, c_void_p]),
    "qsa_sparse_attn_decode_noalloc": (c_int32, [_S, _B, c_void_p, c_void_p, c_void_p, c_void_p,
                                                  c_void_p, c_void_p, c_void_p, c_int32, c_void_p]),
    "qsa_decode_step": (c_int32, [_S, _B, c_void_p, c_void_p, c_void_p, c_int32, c_void_p, c_void_p,
                                  c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                  c_void_p, c_void_p, c_void_p, c_int32, c_void_p, c_size_t,
                                  c_void_p]),
    "qsa_cp_shard_positions": (c_int32, [c_void_p, c_int32, c_int32, c_int32, c_void_p, c_void_p,
                                         c_void_p]),
    "qsa_index_merge_candidates": (c_int32, [_S, _B, c_int32, c_void_p, c_void_p, c_void_p,
                                             c_int32, c_int32, c_void_p, c_void_p, c_void_p,
                                             c_void_p, c_void_p, c_void_p, c_size_t, c_void_p]),
    "qsa_attn_merge_partials": (c_int32, [c_int32, c_int32, c_int32, c_int32, c_void_p, c_void_p,
                                          c_void_p, c_void_p, c_void_p]),
    "qsa_sparse_attn_backward": (c_int32, [_S, _B, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                           c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                           c_void_p, c_void_p]),
    "qsa_index_distill_kl": (c_int32, [_S, _B, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                       c_void_p, c_void_p, c_void_p, c_int64, c_void_p, c_size_t,
                                       c_void_p]),
    "qsa_dense_attn_prefill": (c_int32, [_S, _B, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                         c_void_p]),
    "qsa_dense_attn_decode": (c_int32, [_S, _B, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                        c_int32, c_void_p, c_size_t, c_void_p]),
    "qsa_selftest_wait_timeout": (c_int32, [c_void_p, c_int64, c_void_p]),
}
for _name, (_res, _args) in _SIGS.items():
    _f = getattr(_lib, _name)
    _f.restype = _res
    _f.argtypes = _args


def _check(status: int, where: str):
    if status != QSA_OK:
        raise QsaError(status, where)


def qsa_version() -> int:
    return _lib.qsa_version()


def qsa_status_string(status: int) -> str:
    return _lib.qsa_status_string(status).decode()


def qsa_workspace_size(cfg: QsaConfig, batch: QsaBatch, op: int, num_splits: int = 0) -> int:
    n = c_size_t(0)
    _check(_lib.qsa_workspace_size(ctypes.byref(cfg), ctypes.byref(batch), op, num_splits,
                                   ctypes.byref(n)), "qsa_workspace_size")
    return n.value


def qsa_index_compress(cfg, batch, idx_k, new_seq, new_pos, n_new, kcomp_pool, stream=None):
    _check(_lib.qsa_index_compress(ctypes.byref(cfg), ctypes.byref(batch), _p(idx_k), _p(new_seq),
                                   _p(new_pos), int(n_new), _p(kcomp_pool), _stream(stream)),
           "qsa_index_compress")


def qsa_index_score_topk(cfg, batch, idx_q, idx_w, kcomp_pool, sel, n_sel, sel_scores, workspace,
                         ws_bytes, stream=None):
    _check(_lib.qsa_index_score_topk(ctypes.byref(cfg), ctypes.byref(batch), _p(idx_q), _p(idx_w),
                                     _p(kcomp_pool), _p(sel), _p(n_sel), _p(sel_scores),
                                     _p(workspace), int(ws_bytes), _stream(stream)),
           "qsa_index_score_topk")


def qsa_index_score_redo_flags(cfg, batch, workspace, ws_bytes) -> int | None:
    """Device address of the redo flags (int32 [num_q]) inside the score workspace, or None."""
    out = c_void_p(0)
    _check(_lib.qsa_index_score_redo_flags(ctypes.byref(cfg), ctypes.byref(batch), _p(workspace),
                                           int(ws_bytes), ctypes.byref(out)),
           "qsa_index_score_redo_flags")
    return out.value


def qsa_index_scores(cfg, batch, idx_q, idx_w, kcomp_pool, scores, ld, stream=None):
    _check(_lib.qsa_index_scores(ctypes.byref(cfg), ctypes.byref(batch), _p(idx_q), _p(idx_w),
                                 _p(kcomp_pool), _p(scores), int(ld), _stream(stream)),
           "qsa_index_scores")


def qsa_sparse_attn_prefill(cfg, batch, q, k_pool, v_pool, sel, n_sel, out, lse=None, stream=None):
    _check(_lib.qsa_sparse_attn_prefill(ctypes.byref(cfg), ctypes.byref(batch), _p(q), _p(k_pool),
                                        _p(v_pool), _p(sel), _p(n_sel), _p(out), _p(lse),
                                        _stream(stream)),
           "qsa_sparse_attn_prefill")


def qsa_sparse_attn_decode(cfg, batch, q, k_pool, v_pool, sel, n_sel, out, lse, num_splits,
                           workspace, ws_bytes, stream=None):
    _check(_lib.qsa_sparse_attn_decode(ctypes.byref(cfg), ctypes.byref(batch), _p(q), _p(k_pool),
                                       _p(v_pool), _p(sel), _p(n_sel), _p(out), _p(lse),
                                       int(num_splits), _p(workspace), int(ws_bytes), _stream(stream)),
           "qsa_sparse_attn_decode")


def qsa_sparse_attn_decode_noalloc(cfg, batch, q, k_pool, v_pool, sel, n_sel, out, lse=None,
                                   num_splits=0, stream=None):
    """Split-K decode attention with library-owned scratch (no workspace argument)."""
    _check(_lib.qsa_sparse_attn_decode_noalloc(ctypes.byref(cfg), ctypes.byref(batch), _p(q),
                                               _p(k_pool), _p(v_pool), _p(sel), _p(n_sel), _p(out),
                                               _p(lse), int(num_splits), _stream(stream)),
           "qsa_sparse_attn_decode_noalloc")


def qsa_decode_step(cfg, batch, idx_k_new, new_seq, new_pos, n_new, kcomp_pool, idx_q, idx_w, q,
                    k_pool, v_pool, sel, n_sel, sel_scores, out, lse, num_splits, workspace,
                    ws_bytes, stream=None):
    """The fused one-launch decode step (workspace zero-filled before its first use)."""
    _check(_lib.qsa_decode_step(ctypes.byref(cfg), ctypes.byref(batch), _p(idx_k_new), _p(new_seq),
                                _p(new_pos), int(n_new), _p(kcomp_pool), _p(idx_q), _p(idx_w),
                                _p(q), _p(k_pool), _p(v_pool), _p(sel), _p(n_sel), _p(sel_scores),
                                _p(out), _p(lse), int(num_splits), _p(workspace), int(ws_bytes),
                                _stream(stream)),
           "qsa_decode_step")


def qsa_cp_shard_positions(q_pos, num_q, shard_start, shard_len, pos_sel, pos_attn, stream=None):
    _check(_lib.qsa_cp_shard_positions(_p(q_pos), int(num_q), int(shard_start), int(shard_len),
                                       _p(pos_sel), _p(pos_attn), _stream(stream)),
           "qsa_cp_shard_positions")


def qsa_index_merge_candidates(cfg, batch, nparts, part_sel, part_scores, part_block_lo, block_lo,
                               block_hi, sel, n_sel, sel_scores, local_sel, local_n, workspace,
                               ws_bytes, stream=None):
    """part_block_lo: a host sequence of nparts ints."""
    lo = (c_int32 * int(nparts))(*[int(x) for x in part_block_lo])
    _check(_lib.qsa_index_merge_candidates(ctypes.byref(cfg), ctypes.byref(batch), int(nparts),
                                           _p(part_sel), _p(part_scores), ctypes.cast(lo, c_void_p),
                                           int(block_lo), int(block_hi), _p(sel), _p(n_sel),
                                           _p(sel_scores), _p(local_sel), _p(local_n),
                                           _p(workspace), int(ws_bytes), _stream(stream)),
           "qsa_index_merge_candidates")


def qsa_attn_merge_partials(nparts, num_q, num_q_heads, head_dim, part_out, part_lse, out, lse=None,
                            stream=None):
    _check(_lib.qsa_attn_merge_partials(int(nparts), int(num_q), int(num_q_heads), int(head_dim),
                                        _p(part_out), _p(part_lse), _p(out), _p(lse),
                                        _stream(stream)),
           "qsa_attn_merge_partials")


def qsa_sparse_attn_backward(cfg, batch, q, k_pool, v_pool, sel, n_sel, out, lse, dout, dq,
                             dk_pool, dv_pool, stream=None):
    """Gradients of the sparse attention (dq written; dk_pool, dv_pool accumulated)."""
    _check(_lib.qsa_sparse_attn_backward(ctypes.byref(cfg), ctypes.byref(batch), _p(q), _p(k_pool),
                                         _p(v_pool), _p(sel), _p(n_sel), _p(out), _p(lse),
                                         _p(dout), _p(dq), _p(dk_pool), _p(dv_pool),
                                         _stream(stream)),
           "qsa_sparse_attn_backward")


def qsa_index_distill_kl(cfg, batch, q, k_pool, idx_q, idx_w, kcomp_pool, kl, lse=None,
                         teacher=None, ld=0, workspace=None, ws_bytes=0, stream=None):
    """Per-row KL(block-pooled dense attention || indexer softmax); see include/qsa.h."""
    _check(_lib.qsa_index_distill_kl(ctypes.byref(cfg), ctypes.byref(batch), _p(q), _p(k_pool),
                                     _p(idx_q), _p(idx_w), _p(kcomp_pool), _p(kl), _p(lse),
                                     _p(teacher), int(ld), _p(workspace), int(ws_bytes),
                                     _stream(stream)),
           "qsa_index_distill_kl")


def qsa_dense_attn_prefill(cfg, batch, q, k_pool, v_pool, out, lse=None, stream=None):
    _check(_lib.qsa_dense_attn_prefill(ctypes.byref(cfg), ctypes.byref(batch), _p(q), _p(k_pool),
                                       _p(v_pool), _p(out), _p(lse), _stream(stream)),
           "qsa_dense_attn_prefill")


def qsa_dense_attn_decode(cfg, batch, q, k_pool, v_pool, out, lse, num_splits, workspace, ws_bytes,
                          stream=None):
    _check(_lib.qsa_dense_attn_decode(ctypes.byref(cfg), ctypes.byref(batch), _p(q), _p(k_pool),
                                      _p(v_pool), _p(out), _p(lse), int(num_splits), _p(workspace),
                                      int(ws_bytes), _stream(stream)),
           "qsa_dense_attn_decode")


def qsa_selftest_wait_timeout(err_flag, limit_cycles, stream=None):
    """Launch the bounded-wait self-test (sets QSA_DEVERR_TIMEOUT in err_flag; see include/qsa.h)."""
    _check(_lib.qsa_selftest_wait_timeout(_p(err_flag), int(limit_cycles), _stream(stream)),
           "qsa_selftest_wait_timeout")


from .runner import BlockCarry, QsaRunner, compress_split  # noqa: E402  (step sequencing)

__all__ = [n for n in list(globals()) if n.startswith(("qsa_", "Qsa", "QSA_"))] + [
    "DEVERR", "LIB_PATH", "BlockCarry", "compress_split"]
