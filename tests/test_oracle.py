"""Pins of the fp64 oracle against things other than itself (CPU only).

Each test ties one oracle step to a hand-worked value, a closed form, an independent brute-force
algorithm, or a library routine (torch's fp64 scaled_dot_product_attention as the textbook
attention, torch's fp32->bf16 cast as the textbook rounding).  The method description they follow
is the article "Qwen's million-token window has a 2,048-token keyhole", section "A million-token
window with a selective view".
"""
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import qsa_oracle as orc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def bits(x):
    """bf16 bit patterns of values that are exactly representable in bf16."""
    t = torch.tensor(np.asarray(x, dtype=np.float32)).to(torch.bfloat16)
    assert torch.equal(t.float(), torch.tensor(np.asarray(x, dtype=np.float32))), "not bf16-exact"
    return t.view(torch.int16).numpy().view(np.uint16)


def rand_bits(rng, shape, scale=1.0):
    x = (rng.standard_normal(shape) * scale).astype(np.float32)
    return torch.tensor(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


# ------------------------------------------------------------------------------- bf16 helpers

def test_bf16_widening_matches_torch():
    rng = np.random.default_rng(1)
    b = rand_bits(rng, 4096, 10.0)
    ref = torch.tensor(b.view(np.int16)).view(torch.bfloat16).double().numpy()
    assert np.array_equal(orc.bf16_to_f64(b), ref)


def test_bf16_rounding_matches_torch_on_fp32_values():
    rng = np.random.default_rng(2)
    x = (rng.standard_normal(100000) * np.exp(rng.uniform(-20, 20, 100000))).astype(np.float32)
    ref = torch.tensor(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(orc.f64_to_bf16_bits(x.astype(np.float64)), ref)


def test_bf16_rounding_ties_to_even():
    # 1 + 2^-8 lies halfway between 1 and 1 + 2^-7: the even neighbour is 1.
    # 1 + 3*2^-8 lies halfway between 1 + 2^-7 and 1 + 2^-6: the even neighbour is 1 + 2^-6.
    got = orc.bf16_to_f64(orc.f64_to_bf16_bits(np.array([1 + 2**-8, 1 + 3 * 2**-8, -(1 + 2**-8)])))
    assert list(got) == [1.0, 1 + 2**-6, -1.0]
    # just above a tie rounds up
    assert orc.bf16_to_f64(orc.f64_to_bf16_bits(np.array([1 + 2**-8 + 2**-30])))[0] == 1 + 2**-7


# ------------------------------------------------------------------------------- compress

def test_compress_golden():
    g = json.load(open(os.path.join(GOLDEN, "qsa_tiny_worked.json")))
    kc = orc.compress(bits(g["kidx_rows_positions_0_to_19"]))
    assert np.array_equal(orc.bf16_to_f64(kc), np.array(g["kcomp"], dtype=np.float64))


def test_compress_equal_rows_is_identity_and_incomplete_block_dropped():
    rng = np.random.default_rng(3)
    row = rand_bits(rng, (3, 16))
    k = np.repeat(row, 4, axis=0)                       # 3 blocks of 4 identical rows
    k = np.concatenate([k, rand_bits(rng, (2, 16))])    # + 2 rows of an unfinished block
    kc = orc.compress(k)
    assert kc.shape == (3, 16)
    assert np.array_equal(kc, row)


def test_compress_mean_rounds_to_nearest_even():
    # column 0: 1,1,1,1+2^-6 -> mean 1 + 2^-8 (tie) -> 1
    # column 1: 1,1,1+2^-6,1+2^-5 -> mean 1 + 3*2^-8 (tie) -> 1 + 2^-6
    # column 2: 2,4,6,8 -> 5 exactly;  column 3: 1,0,0,0 -> 0.25 exactly
    rows = [[1, 1, 2, 1], [1, 1, 4, 0], [1, 1 + 2**-6, 6, 0], [1 + 2**-6, 1 + 2**-5, 8, 0]]
    kc = orc.bf16_to_f64(orc.compress(bits(rows)))[0]
    assert list(kc) == [1.0, 1 + 2**-6, 5.0, 0.25]


def test_compress_is_mean_not_sum_on_random_integers():
    rng = np.random.default_rng(4)
    k = rng.integers(-3, 4, size=(64, 8)).astype(np.float32)
    kc = orc.bf16_to_f64(orc.compress(bits(k)))
    # multiples of 1/4 in [-3, 3] are exact in bf16, so the mean is exact
    assert np.array_equal(kc, k.reshape(16, 4, 8).mean(axis=1))


# ------------------------------------------------------------------------------- scores / select

def test_scores_and_selection_golden():
    g = json.load(open(os.path.join(GOLDEN, "qsa_tiny_worked.json")))
    kc = bits(g["kcomp"])
    t = g["t"]
    s = orc.block_scores(kc, bits(g["idx_q"]), bits(g["idx_w"]), orc.num_candidates(t))
    assert list(s) == g["scores"]
    for k, want in g["sel_by_topk"].items():
        assert list(orc.select_blocks(s, t, topk=int(k))) == want
    sel = orc.select_blocks(s, t, topk=2)
    assert list(orc.expand(sel, t)) == g["positions_topk2"]


def test_scores_closed_forms():
    rng = np.random.default_rng(5)
    kc = rand_bits(rng, (300, 32))
    q = rand_bits(rng, (4, 32))
    # zero head weights -> every score is 0
    assert np.all(orc.block_scores(kc, q, bits([0, 0, 0, 0]), 300) == 0)
    # positive homogeneity in w and in q (scaling by 2 is exact in bf16)
    w = bits([0.5, 1, 0.25, 2])
    s = orc.block_scores(kc, q, w, 300)
    assert np.allclose(orc.block_scores(kc, q, bits([1, 2, 0.5, 4]), 300), 2 * s, rtol=0, atol=1e-9)
    q2 = bits(orc.bf16_to_f64(q) * 2)
    assert np.allclose(orc.block_scores(kc, q2, w, 300), 2 * s, rtol=0, atol=1e-9)
    # negating every query head flips which dot products pass the ReLU: s(q) + s(-q) = sum_h w_h |q_h.k|
    qn = bits(-orc.bf16_to_f64(q))
    qq = orc.bf16_to_f64(q)
    absdot = np.abs(orc.bf16_to_f64(kc) @ qq.T) @ orc.bf16_to_f64(w)
    assert np.allclose(s + orc.block_scores(kc, qn, w, 300), absdot, rtol=1e-12, atol=1e-9)
    # scores never negative with non-negative weights
    assert np.all(s >= 0)


def brute_force_select(scores, t, topk, block=4):
    """Independent selection: repeatedly take the highest remaining score, lowest block on ties."""
    n = t // block
    remaining = list(range(n))
    chosen = []
    for _ in range(min(topk, n)):
        best = remaining[0]
        for b in remaining[1:]:
            if scores[b] > scores[best]:
                best = b
        chosen.append(best)
        remaining.remove(best)
    return sorted(chosen) + [t // block]


@pytest.mark.parametrize("seed", range(6))
def test_select_matches_brute_force_with_ties(seed):
    rng = np.random.default_rng(10 + seed)
    for t in list(range(0, 64)) + [100, 257]:
        n = t // 4
        scores = rng.integers(0, 5, size=n).astype(np.float64)   # many ties
        for topk in (1, 3, 4, 7):
            assert list(orc.select_blocks(scores, t, topk)) == brute_force_select(scores, t, topk)


def test_select_invariants_and_constant_budget():
    rng = np.random.default_rng(7)
    for t in [0, 1, 3, 4, 7, 2047, 2048, 2051, 2052, 2055, 5000, 131071, 1048575]:
        n = t // 4
        s = rng.standard_normal(n)
        sel = orc.select_blocks(s, t)
        assert len(sel) == min(512, n) + 1                     # n_sel
        assert sel[-1] == t // 4                               # tail present, last
        assert np.all(np.diff(sel) > 0)                        # ascending, unique
        pos = orc.expand(sel, t)
        assert pos.max() == t and np.all(pos <= t)             # causal
        assert len(pos) <= 2048 + 4                            # budget constant in t
        if t >= 2052:
            assert len(pos) == 2048 + (t % 4) + 1


def test_select_zero_scores_gives_prefix():
    t = 9001
    sel = orc.select_blocks(np.zeros(t // 4), t)
    assert list(sel) == list(range(512)) + [t // 4]


# ------------------------------------------------------------------------------- attention

def sdpa_ref(q, k, v, mask, scale):
    """torch fp64 scaled_dot_product_attention for one query; q [Hq,D], k/v [P,Hkv,D], mask [P]."""
    hq = q.shape[0]
    kx = torch.tensor(np.repeat(orc.bf16_to_f64(k), hq // k.shape[1], axis=1)).permute(1, 0, 2)
    vx = torch.tensor(np.repeat(orc.bf16_to_f64(v), hq // k.shape[1], axis=1)).permute(1, 0, 2)
    qq = torch.tensor(orc.bf16_to_f64(q))[:, None, :]
    m = torch.tensor(mask)[None, None, :].expand(hq, 1, -1)
    o = torch.nn.functional.scaled_dot_product_attention(qq, kx, vx, attn_mask=m, scale=scale)
    return o[:, 0, :].numpy()


@pytest.mark.parametrize("hq,hkv,d", [(4, 1, 64), (32, 4, 128), (8, 2, 16)])
def test_attend_matches_sdpa(hq, hkv, d):
    rng = np.random.default_rng(hq + d)
    P = 300
    q, k, v = rand_bits(rng, (hq, d)), rand_bits(rng, (P, hkv, d)), rand_bits(rng, (P, hkv, d))
    sub = np.sort(rng.choice(P, size=77, replace=False))
    o, lse = orc.attend(q, k[sub], v[sub])
    mask = np.zeros(P, dtype=bool)
    mask[sub] = True
    ref = sdpa_ref(q, k, v, mask, 1 / math.sqrt(d))
    assert np.allclose(o, ref, rtol=1e-12, atol=1e-12)
    # lse against an independent logsumexp
    qq, kk = orc.bf16_to_f64(q), orc.bf16_to_f64(k[sub])
    z = np.einsum("hd,phd->hp", qq, np.repeat(kk, hq // hkv, axis=1)) / math.sqrt(d)
    assert np.allclose(lse, torch.logsumexp(torch.tensor(z), dim=1).numpy(), rtol=1e-13, atol=1e-12)


def test_dense_matches_sdpa_causal():
    rng = np.random.default_rng(8)
    hq, hkv, d, P = 8, 2, 32, 200
    q, k, v = rand_bits(rng, (hq, d)), rand_bits(rng, (P, hkv, d)), rand_bits(rng, (P, hkv, d))
    for t in [0, 1, 57, 199]:
        o, _ = orc.dense_causal(q, k, v, t)
        mask = np.arange(P) <= t
        assert np.allclose(o, sdpa_ref(q, k, v, mask, 1 / math.sqrt(d)), rtol=1e-12, atol=1e-12)


def test_attend_constant_and_onehot_values():
    rng = np.random.default_rng(9)
    hq, hkv, d, P = 4, 1, 16, 40
    q, k = rand_bits(rng, (hq, d)), rand_bits(rng, (P, hkv, d))
    v = bits(np.full((P, hkv, d), 1.5))
    o, _ = orc.attend(q, k, v)
    assert np.allclose(o, 1.5, rtol=0, atol=1e-14)
    # V = one-hot of position (d >= P): the output row is the probability vector, summing to 1
    d2 = 64
    q2, k2 = rand_bits(rng, (hq, d2)), rand_bits(rng, (P, hkv, d2))
    v2 = np.zeros((P, hkv, d2), dtype=np.float32)
    v2[np.arange(P), 0, np.arange(P)] = 1
    o2, lse2 = orc.attend(q2, k2, bits(v2))
    assert np.allclose(o2.sum(axis=1), 1.0, atol=1e-14)
    logits = np.einsum("hd,pd->hp", orc.bf16_to_f64(q2), orc.bf16_to_f64(k2)[:, 0]) / 8.0
    assert np.allclose(o2[:, :P], np.exp(logits - lse2[:, None]), atol=1e-14)


# ------------------------------------------------------------------------------- whole layer

def small_layer(rng, T, hq=4, hkv=1, d=64, di=32):
    kidx = rand_bits(rng, (T, di))
    q = rand_bits(rng, (T, hq, d))
    k, v = rand_bits(rng, (T, hkv, d)), rand_bits(rng, (T, hkv, d))
    iq = rand_bits(rng, (T, 4, di))
    w = torch.tensor(rng.uniform(0, 1, (T, 4)).astype(np.float32)).to(torch.bfloat16)
    w = w.view(torch.int16).numpy().view(np.uint16)
    return kidx, q, k, v, iq, w


def test_qsa_equals_dense_within_budget():
    """With t <= 2051 every earlier block fits in the budget: QSA is dense causal GQA."""
    rng = np.random.default_rng(11)
    T = 2600
    kidx, q, k, v, iq, w = small_layer(rng, T)
    kc = orc.compress(kidx)
    for t in [0, 1, 2, 3, 4, 5, 100, 1023, 2047, 2048, 2050, 2051]:
        o, lse, sel = orc.qsa_row(kc, iq[t], w[t], q[t], k, v, t)
        od, lsed = orc.dense_causal(q[t], k[: t + 1], v[: t + 1], t)
        assert np.allclose(o, od, rtol=0, atol=1e-12) and np.allclose(lse, lsed, atol=1e-12)
    # beyond the budget the selection is a strict subset and the outputs differ
    t = 2599
    o, _, sel = orc.qsa_row(kc, iq[t], w[t], q[t], k, v, t)
    od, _ = orc.dense_causal(q[t], k[: t + 1], v[: t + 1], t)
    assert len(sel) == 513 and not np.allclose(o, od, atol=1e-6)


def test_qsa_increasing_scores_is_sliding_window():
    """Keys built so that block scores strictly increase with b: the selection is the last 512
    candidate blocks plus the tail, i.e. attention over a window of 2,048 + (t % 4) + 1 tokens."""
    rng = np.random.default_rng(12)
    T, di = 6000, 32
    nb = T // 4
    kc_vals = np.zeros((nb, di))
    kc_vals[:, 0] = np.arange(nb) // 256
    kc_vals[:, 1] = np.arange(nb) % 256
    kidx = bits(np.repeat(kc_vals, 4, axis=0))
    iq = bits(np.tile(np.array([[256, 1] + [0] * (di - 2)], dtype=np.float64), (4, 1)))
    w = bits([1, 1, 1, 1])
    hq, hkv, d = 8, 2, 32
    q = rand_bits(rng, (hq, d))
    k, v = rand_bits(rng, (T, hkv, d)), rand_bits(rng, (T, hkv, d))
    kc = orc.compress(kidx)
    for t in [2052, 3001, 4096, 5999]:
        o, _, sel = orc.qsa_row(kc, iq, w, q, k, v, t)
        lo = 4 * (t // 4 - 512)
        assert list(sel) == list(range(t // 4 - 512, t // 4 + 1))
        mask = (np.arange(T) >= lo) & (np.arange(T) <= t)
        assert np.allclose(o, sdpa_ref(q, k, v, mask, 1 / math.sqrt(d)), rtol=1e-12, atol=1e-12)
