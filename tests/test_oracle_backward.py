"""Pins of the backward oracle (oracle/qsa_backward.py) against things other than itself: torch's
autograd through its fp64 scaled_dot_product_attention, central finite differences of the pinned
forward (oracle.qsa_oracle.attend), and closed forms.  The method text is the article "Qwen's
million-token window has a 2,048-token keyhole", section "The indexer is trained, not bolted on"
(sparse training through the layer)."""
import math

import numpy as np
import pytest
import torch

from oracle import qsa_backward as bwd
from oracle import qsa_oracle as orc


def rand_bits(rng, shape, scale=1.0):
    x = (rng.standard_normal(shape) * scale).astype(np.float32)
    return torch.tensor(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


@pytest.mark.parametrize("hq,hkv,d,p", [(4, 1, 16, 9), (8, 2, 32, 37), (6, 3, 8, 5)])
def test_backward_matches_torch_autograd(hq, hkv, d, p):
    rng = np.random.default_rng(20 + p)
    q, k, v = rand_bits(rng, (hq, d)), rand_bits(rng, (p, hkv, d)), rand_bits(rng, (p, hkv, d))
    do = rng.standard_normal((hq, d))
    qt = torch.tensor(orc.bf16_to_f64(q))[None, :, None, :].requires_grad_()
    kt = torch.tensor(orc.bf16_to_f64(k)).permute(1, 0, 2)[None].requires_grad_()   # [1, Hkv, P, D]
    vt = torch.tensor(orc.bf16_to_f64(v)).permute(1, 0, 2)[None].requires_grad_()
    out = torch.nn.functional.scaled_dot_product_attention(
        qt, kt.repeat_interleave(hq // hkv, dim=1), vt.repeat_interleave(hq // hkv, dim=1))
    out.backward(torch.tensor(do)[None, :, None, :])
    dq, dk, dv = bwd.attend_backward(q, k, v, do)
    assert np.allclose(dq, qt.grad[0, :, 0].numpy(), rtol=1e-10, atol=1e-12)
    assert np.allclose(dk, kt.grad[0].permute(1, 0, 2).numpy(), rtol=1e-10, atol=1e-12)
    assert np.allclose(dv, vt.grad[0].permute(1, 0, 2).numpy(), rtol=1e-10, atol=1e-12)


def test_backward_matches_finite_differences_of_the_forward():
    """d/dx of L = sum(do * attend(q, k, v)) by central differences, on inputs perturbed in fp64
    (the forward is evaluated through the pinned oracle with float inputs widened exactly)."""
    rng = np.random.default_rng(21)
    hq, hkv, d, p = 4, 2, 8, 6
    q, k, v = rand_bits(rng, (hq, d)), rand_bits(rng, (p, hkv, d)), rand_bits(rng, (p, hkv, d))
    do = rng.standard_normal((hq, d))
    dq, dk, dv = bwd.attend_backward(q, k, v, do)

    def loss(qf, kf, vf):
        # attend() takes bf16 bits; an fp64 twin of its forward via torch (independent route)
        qt = torch.tensor(qf)[None, :, None, :]
        kt = torch.tensor(kf).permute(1, 0, 2)[None].repeat_interleave(hq // hkv, dim=1)
        vt = torch.tensor(vf).permute(1, 0, 2)[None].repeat_interleave(hq // hkv, dim=1)
        o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt)[0, :, 0].numpy()
        return float(np.sum(do * o))

    base = [orc.bf16_to_f64(x) for x in (q, k, v)]
    h = 1e-6
    for which, grad in ((0, dq), (1, dk), (2, dv)):
        flat = base[which].reshape(-1)
        for i in rng.choice(flat.size, 6, replace=False):
            plus = [b.copy() for b in base]
            minus = [b.copy() for b in base]
            plus[which].reshape(-1)[i] += h
            minus[which].reshape(-1)[i] -= h
            fd = (loss(*plus) - loss(*minus)) / (2 * h)
            assert math.isclose(grad.reshape(-1)[i], fd, rel_tol=1e-5, abs_tol=1e-8)


def test_backward_closed_forms():
    """Constant values: the output no longer depends on the attention weights, so dq = dk = 0
    and each group's dv sums (over positions) to the sum of its heads' upstream gradients; a
    single position gets all of it."""
    rng = np.random.default_rng(22)
    hq, hkv, d, p = 4, 2, 8, 7
    q, k = rand_bits(rng, (hq, d)), rand_bits(rng, (p, hkv, d))
    v = np.repeat(rand_bits(rng, (1, hkv, d)), p, axis=0)
    do = rng.standard_normal((hq, d))
    dq, dk, dv = bwd.attend_backward(q, k, v, do)
    assert np.allclose(dq, 0, atol=1e-12) and np.allclose(dk, 0, atol=1e-12)
    for g in range(hkv):
        assert np.allclose(dv[:, g].sum(0), do[2 * g:2 * g + 2].sum(0), atol=1e-12)
    dq1, dk1, dv1 = bwd.attend_backward(q, k[:1], v[:1], do)
    assert np.allclose(dq1, 0, atol=1e-12) and np.allclose(dk1, 0, atol=1e-12)
    assert np.allclose(dv1[0, 1], do[2] + do[3], atol=1e-12)


def test_rows_accumulate_into_shared_positions():
    """Two rows attending to overlapping selections: dk and dv of a position are the sums of the
    rows' own gradients there; dq is per row."""
    rng = np.random.default_rng(23)
    L, hq, hkv, d = 40, 4, 1, 8
    k, v = rand_bits(rng, (L, hkv, d)), rand_bits(rng, (L, hkv, d))
    q = rand_bits(rng, (2, hq, d))
    do = rng.standard_normal((2, hq, d))
    sels, ts = [np.array([0, 2, 7]), np.array([2, 5, 9])], [30, 39]
    dq, dk, dv = bwd.sparse_backward_rows(q, k, v, sels, ts, do)
    want_k, want_v = np.zeros((L, hkv, d)), np.zeros((L, hkv, d))
    for r in range(2):
        pos = orc.expand(sels[r], ts[r])
        gq, gk, gv = bwd.attend_backward(q[r], k[pos], v[pos], do[r])
        assert np.array_equal(dq[r], gq)
        want_k[pos] += gk
        want_v[pos] += gv
    assert np.allclose(dk, want_k, atol=1e-14) and np.allclose(dv, want_v, atol=1e-14)
    assert np.all(dk[orc.expand(np.array([4, 6]), 39)] == 0)   # positions nobody attends to
