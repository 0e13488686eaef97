"""Plain fp64 CPU oracle of the sparse core attention's backward pass -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may import
this module; the product path never calls it and shares no code with it.

Source: the article "Qwen's million-token window has a 2,048-token keyhole" (cronfeed.work),
section "The indexer is trained, not bolted on": after the dense warm-up, QSA selected the blocks
core attention uses and the indexer and the backbone were trained together (sparse training).
Training through the layer needs the gradient of the sparse core attention with respect to its
queries, keys and values, with the selection held fixed (a top-k choice has no gradient).  The
article gives no formula; the gradient below is that of the forward the layer computes (section
"A million-token window with a selective view"), written out from the chain rule:

  forward, one query row and one query head h (key/value head g = h // (Hq/Hkv)):
      z_p = scale * q_h . k_p   over the row's attended positions p,
      a = softmax(z),  o_h = sum_p a_p v_p;
  backward, given the upstream gradient do_h of o_h:
      dv_p += a_p do_h
      da_p  = do_h . v_p
      dz_p  = a_p (da_p - do_h . o_h)
      dq_h  = scale * sum_p dz_p k_p
      dk_p += scale * dz_p q_h
  and dk, dv of a position sum over every head of its group and every row that attends to it.

Pins (tests/test_oracle_backward.py): torch's autograd through its fp64
scaled_dot_product_attention, central finite differences of the forward, and closed forms.
No function here is unpinned.
"""
from __future__ import annotations

import math

import numpy as np

from .qsa_oracle import bf16_to_f64, expand


def attend_backward(q_bits: np.ndarray, k_bits: np.ndarray, v_bits: np.ndarray, do: np.ndarray,
                    scale: float | None = None):
    """Gradients of one row's attention over the given key/value rows.

    q_bits: bf16 [Hq, D]; k_bits, v_bits: bf16 [P, Hkv, D]; do: float [Hq, D] upstream gradient
    of the output.  Returns (dq [Hq, D], dk [P, Hkv, D], dv [P, Hkv, D]) in float64."""
    q = bf16_to_f64(q_bits)
    k = bf16_to_f64(k_bits)
    v = bf16_to_f64(v_bits)
    do = np.asarray(do, dtype=np.float64)
    hq, d = q.shape
    group = hq // k.shape[1]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    for h in range(hq):
        g = h // group
        z = (k[:, g, :] @ q[h]) * scale
        e = np.exp(z - z.max())
        a = e / e.sum()
        o = a @ v[:, g, :]
        dv[:, g, :] += np.outer(a, do[h])
        da = v[:, g, :] @ do[h]
        dz = a * (da - do[h] @ o)
        dq[h] = scale * (dz @ k[:, g, :])
        dk[:, g, :] += scale * np.outer(dz, q[h])
    return dq, dk, dv


def sparse_backward_rows(q_bits: np.ndarray, k_seq_bits: np.ndarray, v_seq_bits: np.ndarray,
                         sels: list, ts: list, do: np.ndarray, scale: float | None = None):
    """Backward of several query rows of one sequence, each attending to the positions of its
    selection (expanded and clipped at its position t).  q_bits: bf16 [R, Hq, D]; k_seq_bits,
    v_seq_bits: bf16 [L, Hkv, D] (the sequence's positions); do: [R, Hq, D].  Returns (dq [R, Hq, D],
    dk [L, Hkv, D], dv [L, Hkv, D]): dk and dv summed over the rows that attend to a position."""
    dq = np.zeros(q_bits.shape, dtype=np.float64)
    dk = np.zeros(k_seq_bits.shape, dtype=np.float64)
    dv = np.zeros(v_seq_bits.shape, dtype=np.float64)
    for r, (sel, t) in enumerate(zip(sels, ts)):
        pos = expand(np.asarray(sel), t)
        gq, gk, gv = attend_backward(q_bits[r], k_seq_bits[pos], v_seq_bits[pos], do[r], scale)
        dq[r] = gq
        np.add.at(dk, pos, gk)
        np.add.at(dv, pos, gv)
    return dq, dk, dv
