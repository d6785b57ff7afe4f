"""Pins of the fp64 oracle against what the pages and mathematics fix.

None of these tests compares the oracle with itself: each one checks it against
a hand-worked example, a brute-force enumeration, a closed form, an invariant the
pages state, or a library routine (torch's scaled_dot_product_attention in fp64)
on a special case that reduces to it.  The mutation tests at the end plant
plausible mistakes in copies of the oracle's steps and check that some pin here
catches each of them.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import msa_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand(shape, seed, scale=1.0):
    g = np.random.default_rng(seed)
    return g.standard_normal(shape) * scale


def _ints(shape, seed, lo=-4, hi=5):
    g = np.random.default_rng(seed)
    return g.integers(lo, hi, size=shape).astype(np.float64)


# ---------------------------------------------------------------------------
# Hand-worked golden example
# ---------------------------------------------------------------------------

def _golden():
    with open(os.path.join(GOLDEN, "handworked_selection.json")) as f:
        return json.load(f)


def _golden_inputs(gd):
    k_idx = np.array(gd["k_idx"], dtype=np.float64)[None]            # [1, 20, 2]
    S = k_idx.shape[1]
    qg = np.array(gd["q_idx_groups"], dtype=np.float64)               # [Hkv, di]
    q_idx = np.broadcast_to(qg, (1, S, qg.shape[0], qg.shape[1])).copy()
    return q_idx, k_idx


def test_golden_block_maxima_and_selection():
    gd = _golden()
    q_idx, k_idx = _golden_inputs(gd)
    Bk, k = gd["block_size"], gd["top_k"]
    rows = sorted({r["t"] for r in gd["rows"]})
    bm = O.block_scores(q_idx, k_idx, 0, Bk, rows=rows)
    sel = O.select(q_idx, k_idx, 0, Bk, k, rows=rows)
    for r in gd["rows"]:
        n = len(r["block_max"])
        at = rows.index(r["t"])
        assert bm[r["group"], at, :n].tolist() == r["block_max"], r["why"]
        assert np.all(np.isneginf(bm[r["group"], at, n:]))
        assert sel[r["group"], at].tolist() == r["selection"], r["why"]


def test_golden_token_scores():
    """index_scores_row on the hand-worked keys: the raw dot products of tokens
    0..t, the token at t itself included and t+1 left out, for one group and
    for all groups of a row at once."""
    gd = _golden()
    q_idx, k_idx = _golden_inputs(gd)
    ts = gd["token_scores"]
    t = ts["t"]
    qg = np.array(gd["q_idx_groups"], dtype=np.float64)
    assert O.index_scores_row(qg[1], k_idx[0], t).tolist() == ts["group1"]
    both = O.index_scores_row(qg, k_idx[0], t)
    assert both.shape == (t + 1, 2)
    assert both[:, 0].tolist() == ts["group0"] and both[:, 1].tolist() == ts["group1"]


def test_golden_selection_metrics():
    """The [HF] 验证方法 metrics on a hand-worked 2-group x 3-row example."""
    m = _golden()["selection_metrics"]
    got = O.selection_metrics(np.array(m["a"]), np.array(m["b"]))
    n = m["pairs"]
    assert got["total"] == n
    assert got["divergent"] == m["divergent"]
    assert got["mean_overlap"] == pytest.approx(m["overlap_sum"] / n, abs=1e-15)
    assert got["distinct_a"] == pytest.approx(m["distinct_a_sum"] / n, abs=1e-15)
    assert got["distinct_b"] == pytest.approx(m["distinct_b_sum"] / n, abs=1e-15)
    # swapping the sides swaps only the two distinct counts
    rev = O.selection_metrics(np.array(m["b"]), np.array(m["a"]))
    assert rev["distinct_a"] == got["distinct_b"] and rev["distinct_b"] == got["distinct_a"]
    assert rev["divergent"] == got["divergent"] and rev["mean_overlap"] == got["mean_overlap"]


def test_golden_attention_closed_forms():
    gd = _golden()
    Bk = gd["block_size"]
    a0, a1 = gd["attention"]
    S = 20
    # uniform weights: q = 0
    j = np.arange(S, dtype=np.float64)
    v = np.stack([j, 2 * j], axis=1)
    k = _rand((S, 2), 3)
    o, lse = O.attend_row(np.zeros((1, 2)), k, v, np.array(a0["blocks"]), a0["t"], Bk, 1.0)
    np.testing.assert_allclose(o[0], a0["out"], rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse[0], math.log(a0["lse_exp"]), rtol=0, atol=1e-12)
    # two weight levels
    kk = np.zeros((S, 1))
    kk[16:20, 0] = math.log(2.0)
    o, lse = O.attend_row(np.ones((1, 1)), kk, j[:, None], np.array(a1["blocks"]), a1["t"],
                          Bk, 1.0)
    np.testing.assert_allclose(o[0], a1["out"], rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse[0], math.log(a1["lse_exp"]), rtol=0, atol=1e-12)


# ---------------------------------------------------------------------------
# Index branch: brute force, invariants, exp-free ranking, per-group semantics
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("Bk,S,q_pos0,Sq", [(128, 300, 0, 300), (8, 70, 0, 70), (8, 90, 50, 40)])
def test_block_maxima_brute_force(Bk, S, q_pos0, Sq):
    """Explicit loops over (row, group, block, token) on integer inputs: exact."""
    B, Hkv, di = 2, 2, 3
    q_idx = _ints((B, Sq, Hkv, di), 1)
    k_idx = _ints((B, S, di), 2)
    bm = O.block_scores(q_idx, k_idx, q_pos0, Bk)
    nblk = -(-S // Bk)
    for b in range(B):
        for i in range(Sq):
            t = q_pos0 + i
            for g in range(Hkv):
                for c in range(nblk):
                    best = None
                    for jj in range(c * Bk, min((c + 1) * Bk, S)):
                        if jj > t:
                            continue
                        s = 0.0
                        for d in range(di):
                            s += q_idx[b, i, g, d] * k_idx[b, jj, d]
                        best = s if best is None else max(best, s)
                    want = -np.inf if best is None else best
                    assert bm[g, b * Sq + i, c] == want


def _check_selection_row(sel_row, bmax_row, t, Bk, k):
    c_t = t // Bk
    nvis = c_t + 1
    ksel = min(k, nvis)
    chosen = [int(c) for c in sel_row if c >= 0]
    assert len(chosen) == ksel
    assert list(sel_row[ksel:]) == [-1] * (k - ksel)
    assert chosen == sorted(chosen) and len(set(chosen)) == ksel
    assert c_t in chosen and all(0 <= c <= c_t for c in chosen)
    rest = [c for c in range(c_t) if c not in chosen]
    for a in chosen:
        if a == c_t:
            continue
        for u in rest:
            # every chosen earlier block beats every left-out one; ties go low
            assert (bmax_row[a] > bmax_row[u]) or (bmax_row[a] == bmax_row[u] and a < u)


@pytest.mark.parametrize("k,S,Bk,q_pos0,Sq", [(4, 1100, 128, 0, 1100), (5, 200, 8, 0, 200),
                                               (3, 333, 16, 100, 233)])
def test_selection_invariants_and_topk(k, S, Bk, q_pos0, Sq):
    B, Hkv, di = 1, 3, 8
    q_idx = _rand((B, Sq, Hkv, di), 4)
    k_idx = _rand((B, S, di), 5)
    bm = O.block_scores(q_idx, k_idx, q_pos0, Bk)
    sel = O.select(q_idx, k_idx, q_pos0, Bk, k)
    for r in range(B * Sq):
        t = q_pos0 + r % Sq
        for g in range(Hkv):
            _check_selection_row(sel[g, r], bm[g, r], t, Bk, k)
    # distinct blocks reached per (token, group) = min(k, visible blocks)
    nvis = (q_pos0 + np.arange(Sq)) // Bk + 1
    assert (sel >= 0).sum(axis=2).tolist() == [np.minimum(k, nvis).tolist()] * Hkv


def test_selection_exhaustive_subsets():
    """On rows with few blocks, the choice maximises the sorted score vector
    over every subset of earlier blocks (lexicographic, lower ids on ties)."""
    Bk, k = 4, 4
    S = 28  # 7 blocks
    q_idx = _ints((1, S, 2, 2), 6, -2, 3)   # many ties
    k_idx = _ints((1, S, 2), 7, -2, 3)
    bm = O.block_scores(q_idx, k_idx, 0, Bk)
    sel = O.select(q_idx, k_idx, 0, Bk, k)
    for t in range(S):
        c_t = t // Bk
        ksel = min(k, c_t + 1)
        for g in range(2):
            best_key, best = None, None
            for sub in itertools.combinations(range(c_t), ksel - 1):
                key = (sorted((bm[g, t, c] for c in sub), reverse=True),
                       [-c for c in sorted(sub)])
                if best_key is None or key > best_key:
                    best_key, best = key, sub
            want = sorted(list(best) + [c_t]) + [-1] * (k - ksel)
            assert sel[g, t].tolist() == want


def test_exp_free_ranking_equals_softmax_ranking():
    """Ranking by raw block score equals ranking by softmax probability."""
    Bk, k, S = 16, 6, 400
    q_idx = _rand((1, S, 2, 8), 8)
    k_idx = _rand((1, S, 8), 9)
    bm = O.block_scores(q_idx, k_idx, 0, Bk)
    sel = O.select(q_idx, k_idx, 0, Bk, k)
    for t in range(0, S, 7):
        c_t = t // Bk
        for g in range(2):
            m = bm[g, t, : c_t + 1]
            p = np.exp(m - m.max())
            p = p / p.sum()
            by_p = sorted(range(c_t), key=lambda c: (-p[c], c))[: min(k, c_t + 1) - 1]
            want = sorted(by_p + [c_t])
            assert [c for c in sel[g, t] if c >= 0] == want


def test_scaling_index_query_keeps_selection():
    Bk, k, S = 16, 5, 300
    q_idx = _rand((1, S, 2, 8), 10)
    k_idx = _rand((1, S, 8), 11)
    a = O.select(q_idx, k_idx, 0, Bk, k)
    b = O.select(2.0 * q_idx, k_idx, 0, Bk, k)
    assert np.array_equal(a, b)


def test_per_group_vs_pooled_control():
    """Identical index queries across groups: per-group = pooled.  Different
    index queries: the pooled (bug) selection diverges on most rows."""
    Bk, k, S = 16, 4, 512
    one = _rand((1, S, 1, 8), 12)
    k_idx = _rand((1, S, 8), 13)
    same = np.repeat(one, 4, axis=2)
    per = O.select(same, k_idx, 0, Bk, k)
    pooled = O.pooled_select(same, k_idx, 0, Bk, k)
    for g in range(4):
        assert np.array_equal(per[g], pooled)
    diff = _rand((1, S, 4, 8), 14)
    per = O.select(diff, k_idx, 0, Bk, k)
    pooled = O.pooled_select(diff, k_idx, 0, Bk, k)
    m = O.selection_metrics(per, np.broadcast_to(pooled, per.shape))
    late = S // Bk  # rows with many blocks dominate the count
    assert m["divergent"] > 0.5 * m["total"]
    assert m["mean_overlap"] < k
    # against itself: no divergence, full overlap, k distinct blocks when all visible
    m2 = O.selection_metrics(per[:, -late:], per[:, -late:])
    assert m2["divergent"] == 0 and m2["mean_overlap"] == k and m2["distinct_a"] == k


# ---------------------------------------------------------------------------
# Main branch: special cases that reduce to dense attention (library routine)
# ---------------------------------------------------------------------------

def _sdpa(q, k, v, mask=None, causal=False, scale=None):
    """torch SDPA in fp64 on [B,S,H,D] inputs with GQA heads expanded."""
    G = q.shape[2] // k.shape[2]
    qt = torch.from_numpy(q).permute(0, 2, 1, 3)
    kt = torch.from_numpy(k).repeat_interleave(G, dim=2).permute(0, 2, 1, 3)
    vt = torch.from_numpy(v).repeat_interleave(G, dim=2).permute(0, 2, 1, 3)
    out = torch.nn.functional.scaled_dot_product_attention(
        qt, kt, vt, attn_mask=None if mask is None else torch.from_numpy(mask),
        is_causal=causal, scale=scale)
    return out.permute(0, 2, 1, 3).numpy()


def _mha_inputs(B, S, Hq, Hkv, D, di, seed):
    return (_rand((B, S, Hq, D), seed), _rand((B, S, Hkv, D), seed + 1),
            _rand((B, S, Hkv, D), seed + 2), _rand((B, S, Hkv, di), seed + 3),
            _rand((B, S, di), seed + 4))


@pytest.mark.parametrize("S,Bk,k", [(293, 128, 3), (200, 32, 7)])
def test_full_budget_equals_dense_causal_gqa(S, Bk, k):
    assert k * Bk >= S
    q, kk, v, qi, ki = _mha_inputs(2, S, 8, 2, 16, 4, 20)
    out, lse, _ = O.forward(q, kk, v, qi, ki, 0, Bk, k)
    ref = _sdpa(q, kk, v, causal=True)
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)
    dense, dlse = O.dense_causal_gqa(q, kk, v, 0)
    np.testing.assert_allclose(out, dense, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, dlse, rtol=0, atol=1e-12)


def test_full_budget_with_offset_queries():
    """Chunked prefill (q_pos0 > 0): the queries see the earlier context too."""
    S, Sq, Bk, k = 160, 48, 32, 5
    q, kk, v, qi, ki = _mha_inputs(1, S, 4, 2, 8, 4, 30)
    q, qi = q[:, -Sq:], qi[:, -Sq:]
    p0 = S - Sq
    out, _, _ = O.forward(q, kk, v, qi, ki, p0, Bk, k)
    t = p0 + np.arange(Sq)
    mask = (np.arange(S)[None, :] <= t[:, None])[None, None]
    ref = _sdpa(q, kk, v, mask=np.broadcast_to(mask, (1, 4, Sq, S)).copy())
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)


def test_rows_inside_first_block_are_plain_causal():
    S, Bk = 128, 128
    q, kk, v, qi, ki = _mha_inputs(1, S, 4, 1, 8, 4, 40)
    out, _, _ = O.forward(q, kk, v, qi, ki, 0, Bk, 2)
    np.testing.assert_allclose(out, _sdpa(q, kk, v, causal=True), rtol=0, atol=1e-12)


def test_top1_is_block_local_attention():
    S, Bk = 100, 16
    q, kk, v, qi, ki = _mha_inputs(1, S, 4, 2, 8, 4, 50)
    out, _, sel = O.forward(q, kk, v, qi, ki, 0, Bk, 1)
    pos = np.arange(S)
    mask = (pos[None, :] <= pos[:, None]) & (pos[None, :] // Bk == pos[:, None] // Bk)
    ref = _sdpa(q, kk, v, mask=np.broadcast_to(mask, (1, 4, S, S)).copy())
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)
    assert np.array_equal(sel[..., 0], np.broadcast_to(pos // Bk, (2, S)))


def test_dense_mask_formulation():
    """The fix in "解决步骤": scatter the selection into a block mask per index
    head, expand it to the query heads with repeat_interleave, then run masked
    dense attention.  It must equal the gather-based main branch."""
    B, S, Hq, Hkv, D, di, Bk, k = 2, 150, 8, 2, 16, 4, 16, 3
    q, kk, v, qi, ki = _mha_inputs(B, S, Hq, Hkv, D, di, 60)
    out, _, sel = O.forward(q, kk, v, qi, ki, 0, Bk, k)
    nblk = -(-S // Bk)
    blockmask = np.zeros((B, Hkv, S, nblk), dtype=bool)
    for g in range(Hkv):
        for r in range(B * S):
            b, i = divmod(r, S)
            for c in sel[g, r]:
                if c >= 0:
                    blockmask[b, g, i, c] = True
    tok = np.repeat(blockmask, Bk, axis=3)[..., :S]
    tok &= np.tril(np.ones((S, S), dtype=bool))[None, None]
    mask = torch.from_numpy(tok).repeat_interleave(Hq // Hkv, dim=1).numpy()
    ref = _sdpa(q, kk, v, mask=mask)
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)


def test_row_subset_matches_full_run():
    """Sampled rows (used at full size) give the same values as a full run."""
    q, kk, v, qi, ki = _mha_inputs(2, 90, 4, 2, 8, 4, 70)
    full = O.forward(q, kk, v, qi, ki, 0, 16, 3)
    rows = [0, 17, 89, 90, 133, 179]
    part = O.forward(q, kk, v, qi, ki, 0, 16, 3, rows=rows)
    for n, r in enumerate(rows):
        b, i = divmod(r, 90)
        assert np.array_equal(full[0][b, i], part[0][n])
        assert np.array_equal(full[1][b, i], part[1][n])
        assert np.array_equal(full[2][:, r], part[2][:, n])


# ---------------------------------------------------------------------------
# Planted mistakes: each must be caught by at least one of the pins above
# ---------------------------------------------------------------------------

def _mut_no_local(bm, t, Bk, k):
    c_t = t // Bk
    order = sorted(range(c_t + 1), key=lambda c: (-bm[c], c))[: min(k, c_t + 1)]
    return np.array(sorted(order) + [-1] * (k - len(order)))


def _mut_tie_high(bm, t, Bk, k):
    c_t = t // Bk
    ksel = min(k, c_t + 1)
    order = sorted(range(c_t), key=lambda c: (-bm[c], -c))[: ksel - 1]
    return np.array(sorted(order + [c_t]) + [-1] * (k - ksel))


def _mut_local_outside_k(bm, t, Bk, k):
    c_t = t // Bk
    ksel = min(k + 1, c_t + 1)
    order = sorted(range(c_t), key=lambda c: (-bm[c], c))[: ksel - 1]
    return np.array(sorted(order + [c_t])[:k] + [-1] * (k - min(k, ksel)))


MUTANTS = ["no_local", "tie_high", "local_outside_k", "maxpool_sees_future",
           "gqa_modulo", "missing_causal_in_local", "scale_sqrt_di", "scores_drop_token_t",
           "scores_see_token_t1", "metrics_count_padding", "metrics_overlap_union",
           "metrics_distinct_b_from_a"]


def _run_pins(monkeypatch_ctx):
    """Run a fixed subset of pins; return True if all pass."""
    checks = [test_golden_block_maxima_and_selection, test_golden_attention_closed_forms,
              test_golden_token_scores, test_golden_selection_metrics,
              lambda: test_selection_exhaustive_subsets(),
              lambda: test_full_budget_equals_dense_causal_gqa(200, 32, 7),
              lambda: test_dense_mask_formulation(),
              lambda: test_top1_is_block_local_attention()]
    for c in checks:
        try:
            c()
        except AssertionError:
            return False
    return True


@pytest.mark.parametrize("mutant", MUTANTS)
def test_planted_mistakes_are_caught(mutant, monkeypatch):
    orig_select_row = O.select_row
    orig_bmax_row = O.block_maxima_row
    orig_attend_row = O.attend_row
    orig_attend = O.attend
    orig_metrics = O.selection_metrics
    if mutant == "no_local":
        monkeypatch.setattr(O, "select_row", _mut_no_local)
    elif mutant == "tie_high":
        monkeypatch.setattr(O, "select_row", _mut_tie_high)
    elif mutant == "local_outside_k":
        monkeypatch.setattr(O, "select_row", _mut_local_outside_k)
    elif mutant == "maxpool_sees_future":
        # the local block's score would include tokens after the query
        def bs(q_idx, k_idx, q_pos0, Bk, rows=None):
            qi, ki = O._f64(q_idx), O._f64(k_idx)
            B, Sq, Hkv, _ = qi.shape
            nblk = -(-ki.shape[1] // Bk)
            rl = O._rows(B, Sq, rows)
            out = np.full((Hkv, len(rl), nblk), -np.inf)
            for n, r in enumerate(rl):
                b, i = divmod(r, Sq)
                t = q_pos0 + i
                end = min(ki.shape[1], (t // Bk + 1) * Bk)
                s = ki[b, :end] @ qi[b, i].T
                for g in range(Hkv):
                    m = orig_bmax_row(s[:, g], Bk)
                    out[g, n, : m.shape[0]] = m
            return out
        monkeypatch.setattr(O, "block_scores", bs)
    elif mutant == "gqa_modulo":
        def att(q, k, v, q2k, q_pos0, Bk, scale=None, rows=None):
            qf = O._f64(q)
            B, Sq, Hq, D = qf.shape
            Hkv = k.shape[2]
            scale = 1.0 / math.sqrt(D) if scale is None else scale
            rl = O._rows(B, Sq, rows)
            out = np.full((len(rl), Hq, D), np.nan)
            lse = np.full((len(rl), Hq), np.nan)
            for n, r in enumerate(rl):
                b, i = divmod(r, Sq)
                for h in range(Hq):
                    g = h % Hkv   # wrong: interleaved instead of contiguous groups
                    o, ls = orig_attend_row(qf[b, i, h:h + 1], O._f64(k)[b, :, g],
                                            O._f64(v)[b, :, g], np.asarray(q2k)[g, n],
                                            q_pos0 + i, Bk, scale)
                    out[n, h], lse[n, h] = o[0], ls[0]
            if rows is None:
                return out.reshape(B, Sq, Hq, D), lse.reshape(B, Sq, Hq)
            return out, lse
        monkeypatch.setattr(O, "attend", att)
    elif mutant == "missing_causal_in_local":
        def ar(q_heads, k_seq_g, v_seq_g, blocks, t, Bk, scale):
            return orig_attend_row(q_heads, k_seq_g, v_seq_g, blocks,
                                   min(len(k_seq_g) - 1, (t // Bk + 1) * Bk - 1), Bk, scale)
        monkeypatch.setattr(O, "attend_row", ar)
    elif mutant == "scores_drop_token_t":
        # the slice stops one token short: the query's own token is not scored
        monkeypatch.setattr(O, "index_scores_row",
                            lambda q, k, t: O._f64(k)[:t] @ O._f64(q).T)
    elif mutant == "scores_see_token_t1":
        # the slice reaches one token past the query
        monkeypatch.setattr(O, "index_scores_row",
                            lambda q, k, t: O._f64(k)[: t + 2] @ O._f64(q).T)
    elif mutant.startswith("metrics_"):
        def met(sel_a, sel_b):
            a, b = np.asarray(sel_a), np.asarray(sel_b)
            Hkv, R, _ = a.shape
            d = ov = da = db = 0
            for g in range(Hkv):
                for r in range(R):
                    keep = (lambda x: True) if mutant == "metrics_count_padding" else \
                        (lambda x: x >= 0)
                    sa = set(int(x) for x in a[g, r] if keep(x))
                    sb = set(int(x) for x in b[g, r] if keep(x))
                    d += int(sa != sb)
                    ov += len(sa | sb) if mutant == "metrics_overlap_union" else len(sa & sb)
                    da += len(sa)
                    db += len(sa) if mutant == "metrics_distinct_b_from_a" else len(sb)
            n = Hkv * R
            return {"divergent": d, "total": n, "mean_overlap": ov / n,
                    "distinct_a": da / n, "distinct_b": db / n}
        monkeypatch.setattr(O, "selection_metrics", met)
    elif mutant == "scale_sqrt_di":
        def att(q, k, v, q2k, q_pos0, Bk, scale=None, rows=None):
            return orig_attend(q, k, v, q2k, q_pos0, Bk, 1.0 / math.sqrt(2 * O._f64(q).shape[3]),
                               rows)
        monkeypatch.setattr(O, "attend", att)
    assert not _run_pins(monkeypatch), f"planted mistake '{mutant}' passed every pin"
    assert orig_select_row is not None and orig_metrics is not None
