"""Pins of the oracle's KL-alignment loss (index-branch training side), of its
page gather (paged KV cache) and of its packed variable-length forward.

The loss follows snilld.dk "Træning og stabilisering" (the index branch is
trained to match the group-averaged main-branch distribution over the selected
tokens, with gradient detach) under readings R17-R19 of the oracle's header.
None of these checks re-types the oracle's formula: the gradient is pinned by
central finite differences of the loss itself, the value by a closed form on a
two-token row and by the case where the index branch reproduces the teacher
exactly, and the shape of the gradient by the softmax's shift invariance.
"""
import math

import numpy as np
import pytest

from oracle import msa_oracle as O

BK = 128


def _case(seed=0, B=1, Sq=5, Skv=300, Hq=4, Hkv=2, D=8, di=4, K=2, q_pos0=None):
    rng = np.random.default_rng(seed)
    q_pos0 = Skv - Sq if q_pos0 is None else q_pos0
    x = dict(q=rng.standard_normal((B, Sq, Hq, D)), k=rng.standard_normal((B, Skv, Hkv, D)),
             q_idx=rng.standard_normal((B, Sq, Hkv, di)), k_idx=rng.standard_normal((B, Skv, di)))
    q2k = O.select(x["q_idx"], x["k_idx"], q_pos0, BK, K)
    return x, q2k, q_pos0


def _loss(x, q2k, q_pos0):
    return O.index_kl(x["q"], x["k"], x["q_idx"], x["k_idx"], q2k, q_pos0, BK)[0]


def test_gradients_match_central_differences():
    x, q2k, q_pos0 = _case(seed=1, B=2, Sq=3)
    _, dq, dk, _ = O.index_kl(x["q"], x["k"], x["q_idx"], x["k_idx"], q2k, q_pos0, BK)
    eps = 1e-6
    rng = np.random.default_rng(2)
    # every q_idx entry, and k_idx entries of selected and of unselected tokens
    picks = [("q_idx", ix) for ix in np.ndindex(x["q_idx"].shape)]
    for _ in range(40):
        picks.append(("k_idx", (int(rng.integers(2)), int(rng.integers(300)),
                                int(rng.integers(4)))))
    for name, ix in picks:
        y = {n: v.copy() for n, v in x.items()}
        y[name][ix] += eps
        up = _loss(y, q2k, q_pos0)
        y[name][ix] -= 2 * eps
        dn = _loss(y, q2k, q_pos0)
        fd = (up - dn) / (2 * eps)
        an = (dq if name == "q_idx" else dk)[ix]
        assert abs(fd - an) <= 1e-7 + 1e-5 * abs(fd), (name, ix, fd, an)


def test_unselected_tokens_get_no_gradient():
    x, q2k, q_pos0 = _case(seed=3, Sq=3, Skv=700, K=2)  # 6 blocks, 2 kept per row
    _, _, dk, _ = O.index_kl(x["q"], x["k"], x["q_idx"], x["k_idx"], q2k, q_pos0, BK)
    used = set()
    for g in range(q2k.shape[0]):
        for r in range(q2k.shape[1]):
            t = q_pos0 + r
            used.update(O.selected_tokens(q2k[g, r], t, BK).tolist())
    unused = [j for j in range(700) if j not in used]
    assert unused and np.all(dk[0, unused] == 0)


def test_zero_when_index_reproduces_the_teacher():
    # one head per group and index vectors equal to the scaled main ones: the
    # index distribution is the teacher itself
    x, _, q_pos0 = _case(seed=4, Hq=1, Hkv=1, D=8, di=8, K=2)
    scale = 1 / math.sqrt(8)
    x["q_idx"] = scale * x["q"].copy()
    x["k_idx"] = x["k"][:, :, 0, :].copy()
    q2k = O.select(x["q_idx"], x["k_idx"], q_pos0, BK, 2)
    loss, dq, dk, kl = O.index_kl(x["q"], x["k"], x["q_idx"], x["k_idx"], q2k, q_pos0, BK)
    assert abs(loss) < 1e-12 and np.abs(kl).max() < 1e-12
    assert np.abs(dq).max() < 1e-12 and np.abs(dk).max() < 1e-12


def test_two_token_row_closed_form():
    # row at t = 1 sees tokens 0 and 1 of block 0; two query heads in the group
    rng = np.random.default_rng(5)
    D, di = 4, 3
    q = rng.standard_normal((1, 1, 2, D))
    k = rng.standard_normal((1, 2, 1, D))
    q_idx = rng.standard_normal((1, 1, 1, di))
    k_idx = rng.standard_normal((1, 2, di))
    q2k = np.array([[[0]]])
    loss, dq, _, _ = O.index_kl(q, k, q_idx, k_idx, q2k, 1, BK, scale=0.7)
    sig = lambda z: 1 / (1 + math.exp(-z))
    # teacher: mean of the two heads' two-way softmaxes
    pt0 = 0.5 * sum(sig(0.7 * float(q[0, 0, h] @ (k[0, 0, 0] - k[0, 1, 0]))) for h in range(2))
    pi0 = sig(float(q_idx[0, 0, 0] @ (k_idx[0, 0] - k_idx[0, 1])))
    want = pt0 * math.log(pt0 / pi0) + (1 - pt0) * math.log((1 - pt0) / (1 - pi0))
    assert loss == pytest.approx(want, rel=1e-12)
    # d kl / d q_idx = (pi0 - pt0) (k_idx[0] - k_idx[1]) for a two-way softmax
    np.testing.assert_allclose(dq[0, 0, 0], (pi0 - pt0) * (k_idx[0, 0] - k_idx[0, 1]),
                               rtol=1e-12, atol=1e-15)


def test_identical_heads_give_the_single_head_teacher():
    x, q2k, q_pos0 = _case(seed=6, Hq=2, Hkv=1)
    x1 = dict(x, q=x["q"][:, :, :1].copy())
    x2 = dict(x, q=np.repeat(x1["q"], 2, axis=2))
    a = O.index_kl(x1["q"], x["k"], x["q_idx"], x["k_idx"], q2k, q_pos0, BK)
    b = O.index_kl(x2["q"], x["k"], x["q_idx"], x["k_idx"], q2k, q_pos0, BK)
    assert a[0] == pytest.approx(b[0], rel=1e-12)


def test_shift_invariance_of_each_sequence():
    # adding one vector to every index key of a sequence shifts all of a row's
    # scores by the same amount, so the loss cannot change: the gradient with
    # respect to the sequence's index keys sums to zero
    x, q2k, q_pos0 = _case(seed=7, B=2, Sq=4)
    _, _, dk, _ = O.index_kl(x["q"], x["k"], x["q_idx"], x["k_idx"], q2k, q_pos0, BK)
    scale = np.abs(dk).max()
    assert scale > 0
    np.testing.assert_allclose(dk.sum(axis=1), 0, atol=1e-14 * dk.shape[1] + 1e-12 * scale)


def test_gather_pages_inverts_paging():
    # page a contiguous cache by hand (a shuffled pool with unused pages) and
    # gather it back; a two-sequence shared first page too
    rng = np.random.default_rng(8)
    B, L, H, D = 3, 300, 2, 4
    kv = rng.standard_normal((B, L, H, D))
    nblk = -(-L // 128)
    pages = rng.permutation(B * nblk + 5)[: B * nblk].reshape(B, nblk)
    pool = rng.standard_normal((B * nblk + 5, 128, H, D))
    for b in range(B):
        for c in range(nblk):
            n = min(128, L - c * 128)
            pool[pages[b, c], :n] = kv[b, c * 128: c * 128 + n]
    np.testing.assert_array_equal(O.gather_pages(pool, pages, L), kv)
    shared = pages.copy()
    shared[1, 0] = shared[0, 0]
    got = O.gather_pages(pool, shared, L)
    np.testing.assert_array_equal(got[1, :128], kv[0, :128])
    np.testing.assert_array_equal(got[1, 128:], kv[1, 128:])


def _packed(seed, lens_k, lens_q, Hq=4, Hkv=2, D=8, di=4):
    rng = np.random.default_rng(seed)
    tk, tq = sum(lens_k), sum(lens_q)
    x = dict(q=rng.standard_normal((tq, Hq, D)), k=rng.standard_normal((tk, Hkv, D)),
             v=rng.standard_normal((tk, Hkv, D)), q_idx=rng.standard_normal((tq, Hkv, di)),
             k_idx=rng.standard_normal((tk, di)))
    cu_k = np.concatenate([[0], np.cumsum(lens_k)])
    cu_q = np.concatenate([[0], np.cumsum(lens_q)])
    return x, cu_q, cu_k


def test_varlen_with_equal_lengths_is_the_fixed_length_batch():
    x, cu_q, cu_k = _packed(9, [300, 300, 300], [5, 5, 5])
    out, lse, q2k = O.forward_varlen(x["q"], x["k"], x["v"], x["q_idx"], x["k_idx"], cu_q, cu_k,
                                     BK, 2)
    B = 3
    o2, l2, s2 = O.forward(x["q"].reshape(B, 5, 4, 8), x["k"].reshape(B, 300, 2, 8),
                           x["v"].reshape(B, 300, 2, 8), x["q_idx"].reshape(B, 5, 2, 4),
                           x["k_idx"].reshape(B, 300, 4), 295, BK, 2)
    np.testing.assert_array_equal(out, o2.reshape(15, 4, 8))
    np.testing.assert_array_equal(lse, l2.reshape(15, 4))
    np.testing.assert_array_equal(q2k, s2)


def test_varlen_with_a_full_budget_is_dense_causal_attention_per_sequence():
    # top_k * Bk covers every sequence, so each sequence is dense causal GQA over
    # its own keys only (an empty sequence and a decode row included)
    lens_k, lens_q = [300, 1, 129, 70, 0], [7, 1, 2, 70, 0]
    x, cu_q, cu_k = _packed(10, lens_k, lens_q)
    out, lse, _ = O.forward_varlen(x["q"], x["k"], x["v"], x["q_idx"], x["k_idx"], cu_q, cu_k,
                                   BK, 3)
    for b in range(len(lens_k)):
        if lens_q[b] == 0:
            continue
        q0, q1, k0, k1 = cu_q[b], cu_q[b + 1], cu_k[b], cu_k[b + 1]
        do, dl = O.dense_causal_gqa(x["q"][q0:q1][None], x["k"][k0:k1][None],
                                    x["v"][k0:k1][None], lens_k[b] - lens_q[b])
        np.testing.assert_allclose(out[q0:q1], do[0], rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(lse[q0:q1], dl[0], rtol=1e-12, atol=1e-12)
