"""Plain, slow fp64 CPU oracle of the MiniMax Sparse Attention (MSA) forward pass.

TEST INFRASTRUCTURE ONLY.  Only the tests, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import or call
this module.  The product path (the CUDA library and its Python binding) never
does, and this module imports nothing from the product package: the two share
no code.  Inputs are NumPy arrays (or anything ``np.asarray`` accepts) holding
the exact stored values (fp32, or bf16 values widened to fp32); every
computation below runs in float64.

Sources (page title, then section):
  [HF]  "Substantial numerical differences with Minimax MSA attention vs
        Minimax's Reference" (digest of huggingface/transformers issue 46762),
        sections "原因分析" (cause analysis), "解决步骤" (fix steps),
        "验证方法" (verification).
  [ABS] "MiniMax 稀疏注意力" (hyper.ai page of paper 2606.13392), sections
        "摘要" (abstract), "核心贡献" (contributions), "引言" (introduction).
  [DK]  "MiniMax lancerer MSA: blok-sparse attention ..." (snilld.dk), sections
        "Hvad er MSA i praksis", "Teknisk forklaring hvorfor kompleksiteten
        skifter".
  [HU]  "MiniMax új eljárása 28-szorosára csökkenti az AI-figyelem számítási
        igényét" (aiforradalom.online), section "Hogyan működik az indexelő és
        a fő ág?".

Layouts (token-major, as in [HF] "原因分析": the per-head selection is
``[total_qo_len, heads, topk]`` and the kernel list is
``q2k[num_kv_heads, bsz*q_len, topk]``):
  q      [B, Sq, Hq, D]        k, v   [B, Skv, Hkv, D]
  q_idx  [B, Sq, Hkv, di]      k_idx  [B, Skv, di]   (one shared index-key head)
  q2k    [Hkv, B*Sq, top_k]    int, ascending block ids, -1 padded
Query row ``r = b*Sq + i`` sits at absolute position ``t = q_pos0 + i`` and may
see keys ``0..t`` of its own sequence.  Query head ``h`` belongs to GQA group
``g = h // (Hq // Hkv)`` ([HF] "解决步骤": the mask is expanded per index head
with ``repeat_interleave(num_q_heads // H_idx)``, so the heads of one group are
adjacent).

Readings taken where the pages leave a step open (each is also listed in the
design notes of the repository):
  R1  the index score is the raw dot product q_idx . k_idx: no scale, no
      activation ([DK] "Teknisk forklaring": raw scores are ranked).
  R2  a block's score is the max over its causally visible tokens only.
  R3  the forced local block counts inside top_k.
  R4  ties between equal block scores go to the lower block index.
  R5  a row that sees fewer than top_k blocks selects all of them.
  R6  the selected ids are returned in ascending order, -1 padded.
  R7  main-branch scale is 1/sqrt(head_dim) ([DK] "scaled dot-product").
  R17 the index branch's distribution for the KL-alignment loss is the
      softmax of the raw token-level index scores over the same causally
      visible tokens of the selected blocks that the main branch attends.
  R18 the loss is KL(teacher || index) per (query row, group), the teacher
      being the mean over the group's query heads of the main-branch softmax
      over those tokens; the loss is the mean over all (row, group) pairs.
  R19 gradient detach: the teacher and the selection are constants; the
      gradients flow into q_idx and k_idx only.
  R21 in a packed variable-length batch, a sequence's query rows are its last
      tokens (chunked prefill and decode), and sequences are independent.
  R22 NVFP4 index tensors ([HU] "Elérhetőség" lists NVFP4 among the kernel
      precisions and says no more): NVIDIA's NVFP4 format, e2m1 elements (two
      per byte, the even element in the low nibble) with one unsigned e4m3
      (ue4m3) scale per 16 consecutive elements along index_dim, no second
      per-tensor scale (a positive factor changes no selection, R1).  The
      scores are taken over the decoded values.

Additional source for the KL-alignment loss:
  [DK]  section "Træning og stabilisering": Top-k is not differentiable, so an
        extra KL-alignment loss trains the index projections, the index branch
        matching the main branch's attention pattern, whose teacher is the
        group-averaged main distribution over the selected tokens, with
        gradient detach.
  [HU]  section "A betanítás és a kernel-optimalizáció": a KL-divergence loss
        aligns the Index Branch distribution to the Main Branch pattern.
"""
from __future__ import annotations

import math
from typing import Iterable, Optional, Sequence

import numpy as np

NEG_INF = -np.inf


def _np(x) -> np.ndarray:
    """The stored values as a NumPy array (torch tensors are widened to fp32,
    which holds every bf16 value exactly)."""
    if hasattr(x, "detach"):  # a torch tensor given by a test
        x = x.detach().float().cpu().numpy()
    return np.asarray(x)


def _f64(x) -> np.ndarray:
    """Widen an input to float64 without changing its value."""
    return np.asarray(_np(x), dtype=np.float64)


def _take(x, idx: np.ndarray) -> np.ndarray:
    """Rows ``idx`` of x (NumPy array or torch tensor) as float64."""
    if hasattr(x, "detach"):
        import torch  # only when the caller handed in torch tensors
        return _f64(x[torch.from_numpy(np.ascontiguousarray(idx))])
    return _f64(np.asarray(x)[idx])


def _rows(batch: int, q_len: int, rows: Optional[Iterable[int]]) -> list:
    return list(range(batch * q_len)) if rows is None else [int(r) for r in rows]


# ---------------------------------------------------------------------------
# NVFP4 index tensors (reading R22), decoded from the format's definition
# ---------------------------------------------------------------------------

NVFP4_GROUP = 16  # elements per ue4m3 scale


def e2m1_value(code: int) -> float:
    """One 4-bit e2m1 code: bit 3 sign, bits 2-1 exponent (bias 1), bit 0
    mantissa; exponent 0 is subnormal (mantissa x 0.5)."""
    sign = -1.0 if code & 8 else 1.0
    e, m = (code >> 1) & 3, code & 1
    mag = 0.5 * m if e == 0 else 2.0 ** (e - 1) * (1.0 + 0.5 * m)
    return sign * mag


def ue4m3_value(code: int) -> float:
    """One unsigned e4m3 scale byte: bits 6-3 exponent (bias 7), bits 2-0
    mantissa, exponent 0 subnormal (mantissa/8 x 2^-6); 0x7f is NaN and the
    top bit must be clear."""
    if code & 0x80 or code == 0x7F:
        return math.nan
    e, m = (code >> 3) & 15, code & 7
    return (m / 8.0) * 2.0 ** -6 if e == 0 else 2.0 ** (e - 7) * (1.0 + m / 8.0)


def nvfp4_decode(codes, scales) -> np.ndarray:
    """Values of NVFP4 tensors: ``codes`` [..., d/2] bytes (element 2i in the low
    nibble of byte i, 2i+1 in the high nibble), ``scales`` [..., d/16] ue4m3
    bytes.  Returns float64 [..., d]: element j = e2m1(code j) x scale[j // 16]."""
    c = np.asarray(_np(codes)).astype(np.int64)
    sc = np.asarray(_np(scales)).astype(np.int64)
    d = c.shape[-1] * 2
    assert sc.shape[-1] * NVFP4_GROUP == d, "one scale per 16 elements"
    lut_e = np.array([e2m1_value(i) for i in range(16)])
    lut_s = np.array([ue4m3_value(i) for i in range(256)])
    nib = np.empty(c.shape[:-1] + (d,), dtype=np.int64)
    nib[..., 0::2] = c & 15
    nib[..., 1::2] = (c >> 4) & 15
    return lut_e[nib] * np.repeat(lut_s[sc], NVFP4_GROUP, axis=-1)


# ---------------------------------------------------------------------------
# Index branch
# ---------------------------------------------------------------------------

def index_scores_row(q_vecs, k_idx_seq, t: int) -> np.ndarray:
    """Token scores s_j = q_vec . k_idx_seq[j] for every visible key j = 0..t.

    [DK] "Hvad er MSA i praksis" and [HU] "Hogyan működik...": one index-query
    head per GQA group is scored against the single shared index-key head over
    the causally visible key tokens.  Reading R1: the raw dot product.
    ``q_vecs`` is one index query [di] (result [t+1]) or the index queries of
    all groups of a row [Hkv, di] (result [t+1, Hkv], column g = group g).
    """
    return _f64(k_idx_seq)[: t + 1] @ _f64(q_vecs).T


def block_maxima_row(scores: np.ndarray, block_size: int) -> np.ndarray:
    """Max-pool visible token scores into blocks of ``block_size`` tokens.

    [HF] "原因分析": ``scores.amax(dim=-1)`` pools inside each 128-token block.
    Reading R2: only the visible tokens of the last (local) block take part, so
    ``scores`` (length t+1) is cut at t.  Returns the maxima of blocks
    0..floor(t/block_size).
    """
    n = scores.shape[0]
    nvis = (n - 1) // block_size + 1
    out = np.empty(nvis, dtype=np.float64)
    for c in range(nvis):
        out[c] = scores[c * block_size: min((c + 1) * block_size, n)].max()
    return out


def select_row(block_max: np.ndarray, t: int, block_size: int, top_k: int) -> np.ndarray:
    """Exp-free top-k block selection of one (query, GQA group) row.

    [DK] "Hvad er MSA i praksis": each query keeps k blocks per GQA group and the
    query's own block is always among them.  [DK] "Teknisk forklaring": softmax
    keeps the ranking, so raw block scores are ranked (no exponential).
    [HF] "解决步骤": the local-block boost and top-k are applied per index head.
    Readings R3-R6: the local block counts inside k; the other k-1 slots go to
    the highest-scoring earlier blocks, ties to the lower index; a row with fewer
    than k visible blocks takes all of them; ids ascending, -1 padded.
    """
    c_t = t // block_size
    nvis = c_t + 1
    ksel = min(top_k, nvis)
    earlier = sorted(range(c_t), key=lambda c: (-block_max[c], c))
    chosen = sorted([c_t] + earlier[: ksel - 1])
    return np.array(chosen + [-1] * (top_k - ksel), dtype=np.int64)


def block_scores(q_idx, k_idx, q_pos0: int, block_size: int,
                 rows: Optional[Sequence[int]] = None) -> np.ndarray:
    """Block maxima ``bmax[g, n, c]`` of the requested rows (default: all rows).

    Axis 1 follows ``rows`` (for a full run it is the row r = b*Sq + i).  Blocks
    c > floor(t/block_size) are not visible to the row and hold -inf.  Shape
    ``[Hkv, len(rows), nblk]`` with ``nblk = ceil(Skv / block_size)``.
    """
    B, Sq, Hkv, _ = q_idx.shape
    nblk = -(-k_idx.shape[1] // block_size)
    rl = _rows(B, Sq, rows)
    out = np.full((Hkv, len(rl), nblk), NEG_INF)
    kb, kb_of = None, -1
    for n, r in enumerate(rl):
        b, i = divmod(r, Sq)
        t = q_pos0 + i
        if b != kb_of:  # widen one sequence's index keys at a time
            kb, kb_of = _f64(k_idx[b]), b
        s = index_scores_row(q_idx[b, i], kb, t)  # all groups at once: [t+1, Hkv]
        for g in range(Hkv):
            m = block_maxima_row(s[:, g], block_size)
            out[g, n, : m.shape[0]] = m
    return out


def select(q_idx, k_idx, q_pos0: int, block_size: int, top_k: int,
           rows: Optional[Sequence[int]] = None) -> np.ndarray:
    """Per-(query, GQA group) selection ``q2k[Hkv, len(rows), top_k]`` (int64).

    Axis 1 follows ``rows``; for a full run this is the library's
    ``q2k[Hkv, B*Sq, top_k]`` layout.
    """
    B, Sq, Hkv, _ = q_idx.shape
    rl = _rows(B, Sq, rows)
    bm = block_scores(q_idx, k_idx, q_pos0, block_size, rl)
    q2k = np.empty((Hkv, len(rl), top_k), dtype=np.int64)
    for n, r in enumerate(rl):
        t = q_pos0 + r % Sq
        for g in range(Hkv):
            q2k[g, n] = select_row(bm[g, n], t, block_size, top_k)
    return q2k


# ---------------------------------------------------------------------------
# Main branch
# ---------------------------------------------------------------------------

def attend_row(q_heads, k_seq_g, v_seq_g, blocks, t: int, block_size: int,
               scale: float):
    """Exact softmax attention of one query row's heads of one GQA group.

    [DK] "Hvad er MSA i praksis": the main branch gathers the causally visible
    tokens of the selected blocks and runs scaled dot-product softmax over
    exactly those tokens; all query heads of the group share the block set.
    Returns (o [G, D], lse [G]) with lse the natural log of the softmax
    normaliser of the scaled logits.
    """
    keys = []
    for c in blocks:
        if c < 0:
            continue
        lo = c * block_size
        hi = min((c + 1) * block_size, t + 1)
        keys.extend(range(lo, hi))
    J = np.array(sorted(keys), dtype=np.int64)
    K = _take(k_seq_g, J)         # [n, D]
    V = _take(v_seq_g, J)
    z = scale * (_f64(q_heads) @ K.T)  # [G, n]
    m = z.max(axis=1, keepdims=True)
    w = np.exp(z - m)
    l = w.sum(axis=1, keepdims=True)
    o = (w / l) @ V
    lse = (m + np.log(l))[:, 0]
    return o, lse


def attend(q, k, v, q2k, q_pos0: int, block_size: int,
           scale: Optional[float] = None, rows: Optional[Sequence[int]] = None):
    """Main branch over a given selection.

    ``q2k`` is ``[Hkv, len(rows), top_k]`` with axis 1 following ``rows``.
    Returns (out, lse): ``[B, Sq, Hq, D]`` and ``[B, Sq, Hq]`` for a full run,
    ``[len(rows), Hq, D]`` and ``[len(rows), Hq]`` when rows are given.
    ``scale`` defaults to 1/sqrt(D) (reading R7).
    """
    B, Sq, Hq, D = q.shape
    Hkv = k.shape[2]
    G = Hq // Hkv
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    sel = np.asarray(q2k)
    rl = _rows(B, Sq, rows)
    out = np.empty((len(rl), Hq, D))
    lse = np.empty((len(rl), Hq))
    for n, r in enumerate(rl):
        b, i = divmod(r, Sq)
        t = q_pos0 + i
        for g in range(Hkv):
            hs = slice(g * G, (g + 1) * G)
            # only the gathered key rows are widened (inside attend_row)
            o, ls = attend_row(_f64(q[b, i, hs]), k[b, :, g], v[b, :, g], sel[g, n],
                               t, block_size, scale)
            out[n, hs] = o
            lse[n, hs] = ls
    if rows is None:
        return out.reshape(B, Sq, Hq, D), lse.reshape(B, Sq, Hq)
    return out, lse


def forward(q, k, v, q_idx, k_idx, q_pos0: int, block_size: int, top_k: int,
            scale: Optional[float] = None, rows: Optional[Sequence[int]] = None):
    """Index branch then main branch ([ABS] "摘要"; [DK] "Hvad er MSA i praksis").

    Returns (out, lse, q2k).
    """
    q2k = select(q_idx, k_idx, q_pos0, block_size, top_k, rows)
    out, lse = attend(q, k, v, q2k, q_pos0, block_size, scale, rows)
    return out, lse, q2k


# ---------------------------------------------------------------------------
# KL-alignment loss of the index branch (training side)
# ---------------------------------------------------------------------------

def gather_pages(cache, block_table, kv_len: int, page_size: int = 128) -> np.ndarray:
    """The per-sequence layout [B, kv_len, ...] of a paged KV cache.

    A paged cache stores each sequence's tokens in pages of ``page_size`` tokens:
    token j of sequence b is row j % page_size of page block_table[b, j //
    page_size] (a vLLM-style block table).
    This is that definition written out, one token at a time.
    """
    c = np.asarray(cache)
    tab = np.asarray(block_table)
    B = tab.shape[0]
    out = np.empty((B, kv_len) + c.shape[2:], dtype=c.dtype)
    for b in range(B):
        for j in range(kv_len):
            out[b, j] = c[tab[b, j // page_size], j % page_size]
    return out


def selected_tokens(blocks, t: int, block_size: int) -> np.ndarray:
    """The causally visible tokens 0..t of the selected blocks, ascending."""
    keys = []
    for c in blocks:
        if c < 0:
            continue
        keys.extend(range(c * block_size, min((c + 1) * block_size, t + 1)))
    return np.array(sorted(keys), dtype=np.int64)


def index_kl_row(q_heads, k_seq_g, q_idx_vec, k_idx_seq, blocks, t: int, block_size: int,
                 scale: float):
    """KL-alignment term of one (query row, group) and its score gradient.

    [DK] "Træning og stabilisering": the index branch is trained to match the
    main branch; the teacher is the group-averaged main distribution over the
    selected tokens (readings R17-R19).  Over the tokens J of the selected
    blocks (visible ones only):
      index  p_I = softmax_j(q_idx . k_idx[j])                 (raw scores, R1)
      teacher p_T = mean over the group's heads h of softmax_j(scale * q_h . k[j])
      kl = sum_j p_T[j] * (ln p_T[j] - ln p_I[j])
    and d kl / d s_j = p_I[j] - p_T[j].  Returns (kl, J, p_I - p_T).
    """
    J = selected_tokens(blocks, t, block_size)
    s = _take(k_idx_seq, J) @ _f64(q_idx_vec)            # [n]
    lse_i = s.max() + math.log(np.exp(s - s.max()).sum())
    log_pi = s - lse_i
    z = scale * (_f64(q_heads) @ _take(k_seq_g, J).T)    # [G, n]
    a = np.exp(z - z.max(axis=1, keepdims=True))
    a /= a.sum(axis=1, keepdims=True)
    p_t = a.mean(axis=0)
    pos = p_t > 0
    kl = float(np.sum(p_t[pos] * (np.log(p_t[pos]) - log_pi[pos])))
    return kl, J, np.exp(log_pi) - p_t


def index_kl(q, k, q_idx, k_idx, q2k, q_pos0: int, block_size: int,
             scale: Optional[float] = None):
    """Mean KL-alignment loss over all (row, group) pairs and its gradients.

    Returns (loss, dq_idx [B, Sq, Hkv, di], dk_idx [B, Skv, di], kl [Hkv, B*Sq]).
    With N = B*Sq*Hkv pairs, d loss / d s = (p_I - p_T) / N for each pair's
    tokens, so dq_idx[row, g] = sum_j ds_j k_idx[j] and dk_idx[j] collects
    ds_j q_idx[row, g] over every (row, group) whose selection holds token j
    (k_idx is the one index-key head shared by all groups).  q, k and the
    selection q2k are constants (R19).  ``scale`` defaults to 1/sqrt(D) (R7).
    """
    B, Sq, Hq, D = q.shape
    Hkv = k.shape[2]
    G = Hq // Hkv
    di = q_idx.shape[3]
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    sel = np.asarray(q2k)
    N = B * Sq * Hkv
    kl = np.zeros((Hkv, B * Sq))
    dq = np.zeros((B, Sq, Hkv, di))
    dk = np.zeros((B, k_idx.shape[1], di))
    for b in range(B):
        kis = _f64(k_idx[b])
        for i in range(Sq):
            r = b * Sq + i
            t = q_pos0 + i
            for g in range(Hkv):
                qi = _f64(q_idx[b, i, g])
                kl[g, r], J, ds = index_kl_row(q[b, i, g * G:(g + 1) * G], k[b, :, g], qi,
                                               kis, sel[g, r], t, block_size, scale)
                ds = ds / N
                dq[b, i, g] = ds @ kis[J]
                dk[b, J] += np.outer(ds, qi)
    return float(kl.sum() / N), dq, dk, kl


# ---------------------------------------------------------------------------
# Variable-length batches (packed sequences)
# ---------------------------------------------------------------------------

def forward_varlen(q, k, v, q_idx, k_idx, cu_q, cu_k, block_size: int, top_k: int,
                   scale: Optional[float] = None):
    """The forward pass over a packed batch of sequences of different lengths.

    [HF] "原因分析" gives the selection the packed shape [total_qo_len, heads,
    topk]: the query rows of all sequences are concatenated.  Sequence b owns
    query rows cu_q[b] .. cu_q[b+1]-1 and key rows cu_k[b] .. cu_k[b+1]-1 of the
    packed q [total_q, Hq, D], q_idx [total_q, Hkv, di], k, v [total_k, Hkv, D]
    and k_idx [total_k, di].  Reading R21: a sequence's queries are its last
    Sq_b = cu_q[b+1] - cu_q[b] tokens (position L_b - Sq_b + i for its i-th row,
    L_b = cu_k[b+1] - cu_k[b]), as in chunked prefill and decode; sequences never
    see one another.  Returns (out [total_q, Hq, D], lse [total_q, Hq],
    q2k [Hkv, total_q, top_k]).
    """
    cu_q, cu_k = np.asarray(cu_q), np.asarray(cu_k)
    total_q, Hq, D = np.shape(q)
    Hkv = np.shape(k)[1]
    out = np.empty((total_q, Hq, D))
    lse = np.empty((total_q, Hq))
    q2k = np.full((Hkv, total_q, top_k), -1, dtype=np.int64)
    for b in range(len(cu_q) - 1):
        q0, q1, k0, k1 = int(cu_q[b]), int(cu_q[b + 1]), int(cu_k[b]), int(cu_k[b + 1])
        if q1 == q0:
            continue
        one = lambda x, lo, hi: np.asarray(x)[lo:hi][None]  # noqa: E731  (batch of one)
        o, l, sel = forward(one(q, q0, q1), one(k, k0, k1), one(v, k0, k1),
                            one(q_idx, q0, q1), one(k_idx, k0, k1), (k1 - k0) - (q1 - q0),
                            block_size, top_k, scale)
        out[q0:q1], lse[q0:q1], q2k[:, q0:q1] = o[0], l[0], sel
    return out, lse, q2k


# ---------------------------------------------------------------------------
# Independent references used by the pins
# ---------------------------------------------------------------------------

def dense_causal_gqa(q, k, v, q_pos0: int, scale: Optional[float] = None,
                     rows: Optional[Sequence[int]] = None):
    """Dense causal GQA attention written directly from its definition.

    Query head h reads KV head h // (Hq // Hkv) over keys 0..t.  This is what MSA
    must equal when top_k * block_size covers every visible key.
    """
    qf, kf, vf = _f64(q), _f64(k), _f64(v)
    B, Sq, Hq, D = qf.shape
    Hkv = kf.shape[2]
    G = Hq // Hkv
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    out = np.full((B, Sq, Hq, D), np.nan)
    lse = np.full((B, Sq, Hq), np.nan)
    for r in _rows(B, Sq, rows):
        b, i = divmod(r, Sq)
        t = q_pos0 + i
        for h in range(Hq):
            kv = h // G
            z = scale * (kf[b, : t + 1, kv] @ qf[b, i, h])
            m = z.max()
            w = np.exp(z - m)
            out[b, i, h] = (w @ vf[b, : t + 1, kv]) / w.sum()
            lse[b, i, h] = m + math.log(w.sum())
    return out, lse


def pooled_select(q_idx, k_idx, q_pos0: int, block_size: int, top_k: int) -> np.ndarray:
    """The pooled selection that [HF] "原因分析" reports as the bug.

    Block scores are maxed over the index-head axis (``.amax(dim=1)``) so every
    group shares one selection.  Kept only as a negative control for the tests;
    returns ``[B*Sq, top_k]``.
    """
    bm = block_scores(q_idx, k_idx, q_pos0, block_size)
    pooled = bm.max(axis=0)
    Sq = _f64(q_idx).shape[1]
    return np.stack([select_row(pooled[r], q_pos0 + r % Sq, block_size, top_k)
                     for r in range(pooled.shape[0])])


def selection_metrics(sel_a: np.ndarray, sel_b: np.ndarray) -> dict:
    """The three selection metrics of [HF] "验证方法".

    ``sel_a`` and ``sel_b`` are ``[Hkv, R, k]`` (-1 padded).  Returns the number
    of (row, group) selections that differ, the mean per-(row, group) overlap
    and, for each side, the mean number of distinct blocks one (token, group)
    reaches.
    """
    a = np.asarray(sel_a)
    b = np.asarray(sel_b)
    Hkv, R, _ = a.shape
    differ = 0
    overlap = 0
    dist_a = 0
    dist_b = 0
    for g in range(Hkv):
        for r in range(R):
            sa = set(int(x) for x in a[g, r] if x >= 0)
            sb = set(int(x) for x in b[g, r] if x >= 0)
            differ += int(sa != sb)
            overlap += len(sa & sb)
            dist_a += len(sa)
            dist_b += len(sb)
    n = Hkv * R
    return {"divergent": differ, "total": n, "mean_overlap": overlap / n,
            "distinct_a": dist_a / n, "distinct_b": dist_b / n}
