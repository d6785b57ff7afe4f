"""Seeded synthetic inputs for the MSA forward pass.

This module only draws inputs; it holds none of the method's arithmetic and
imports neither the CUDA binding nor the oracle, so both sides (and the bench)
can take their inputs from it.

Recipe (the same for every workload):
  * one ``torch.Generator`` on the target device (the GPU for GPU runs, the CPU
    for CPU-only tests), seeded with ``seed``, draws in this order Q, K, V,
    q_idx and k_idx as standard normals in fp32, row chunk by row chunk (the
    two devices' streams differ; each is fixed by the seed);
  * each tensor is multiplied by 1 (``fp32`` workloads) or by 1/sqrt(d)
    (``bf16`` workloads, d = head_dim for Q/K/V and index_dim for the index
    tensors) and rounded once to the workload's dtype (round to nearest even; q_idx and
    k_idx to fp8 e4m3 instead when index_dtype is "fp8", Q and K when qk_dtype
    is "fp8": the same draws, so an fp8 workload's inputs are its bf16 twin's
    rounded to e4m3);
  * needles: for every sequence b and group g, ``needles`` distinct "past"
    blocks are drawn uniformly (``torch.randperm`` from the same generator, in
    (b, g) order) from blocks ``0 .. upper-1`` where ``upper`` is the block of
    the first query when that is > 0, else the block of the last query.  Every
    token of a drawn block gets ``0.5 * mean_i q_idx[b, i, g, :]`` added to its
    index key, in fp32, before k_idx is rounded to bf16 (the mean is taken over
    the sequence's stored, already rounded q_idx rows).
  * index_dtype "nvfp4": q_idx and k_idx (needles included) are drawn the same
    way in fp32 and then encoded to NVFP4 by quantize_nvfp4 (the needle shift
    uses the mean of the fp32 q_idx draws); the inputs are the codes and the
    scales, and both sides decode them.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, Optional

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    q_len: int
    kv_len: int
    q_pos0: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    index_dim: int
    block_size: int
    top_k: int
    dtype: str          # "f32" or "bf16"
    needles: int        # planted needle blocks per (sequence, group)
    index_dtype: str = ""  # "" (same as dtype), "fp8" (q_idx, k_idx in fp8 e4m3) or
                           # "nvfp4" (e2m1 codes, two per byte, + a ue4m3 scale per 16)
    qk_dtype: str = ""     # "" (same as dtype) or "fp8" (q, k in fp8 e4m3; v stays bf16)

    @property
    def rows(self) -> int:
        return self.batch * self.q_len

    @property
    def nblk(self) -> int:
        return -(-self.kv_len // self.block_size)

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    @property
    def torch_index_dtype(self) -> torch.dtype:
        if self.index_dtype == "nvfp4":
            return torch.uint8
        return torch.float8_e4m3fn if self.index_dtype == "fp8" else self.torch_dtype

    @property
    def torch_qk_dtype(self) -> torch.dtype:
        return torch.float8_e4m3fn if self.qk_dtype == "fp8" else self.torch_dtype

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS: Dict[str, Workload] = {
    "tiny": Workload("tiny", 1, 1024, 1024, 0, 8, 2, 64, 32, 128, 4, "f32", 0),
    "prefill_32k": Workload("prefill_32k", 1, 32768, 32768, 0, 64, 4, 128, 128, 128, 16,
                            "bf16", 8),
    "prefill_128k": Workload("prefill_128k", 1, 131072, 131072, 0, 64, 4, 128, 128, 128,
                             16, "bf16", 32),
    "decode_128k": Workload("decode_128k", 32, 1, 131072, 131071, 64, 4, 128, 128, 128,
                            16, "bf16", 32),
    "chunk_1m": Workload("chunk_1m", 1, 8192, 1048576, 1040384, 64, 4, 128, 128, 128, 16,
                         "bf16", 64),
}

# A packed serving-style batch for the variable-length entry point (prefill_128k
# shapes: 64 query heads, 4 groups, head_dim and index_dim 128, top 16, bf16):
# (query rows, keys) per sequence: two fresh prefills, two prefill chunks at
# 32K and 64K context and sixteen decode rows at 128K (one run of equal lengths).
VARLEN_MIX = ([8192, 16384, 2048] + [1] * 16 + [4096],
              [8192, 16384, 32768] + [131072] * 16 + [65536])

_CHUNK_ELEMS = 1 << 24


def _draw(gen: torch.Generator, shape, scale: float, dtype: torch.dtype) -> torch.Tensor:
    """Standard normals drawn in fp32 row chunk by row chunk, scaled, rounded."""
    out = torch.empty(shape, dtype=dtype, device=gen.device)
    flat = out.view(shape[0], -1)
    per_row = flat.shape[1]
    step = max(1, _CHUNK_ELEMS // max(per_row, 1))
    for r0 in range(0, flat.shape[0], step):
        r1 = min(flat.shape[0], r0 + step)
        x = torch.randn((r1 - r0, per_row), generator=gen, dtype=torch.float32,
                        device=gen.device)
        if scale != 1.0:
            x.mul_(scale)
        flat[r0:r1] = x.to(dtype)
    return out


# NVFP4 encoding of drawn inputs: the sixteen e2m1 magnitudes' grid and the
# 127 finite unsigned e4m3 scale values (codes 0x00 .. 0x7e), ascending.
_E2M1_GRID = (0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0)


def _ue4m3_table() -> list:
    vals = []
    for code in range(127):
        e, m = code >> 3, code & 7
        vals.append(m * 2.0 ** -9 if e == 0 else 2.0 ** (e - 7) * (1 + m / 8))
    return vals


def quantize_nvfp4(x: torch.Tensor):
    """Encodes fp32 values [..., d] (d a multiple of 16) as NVFP4: per group of
    16 the smallest ue4m3 scale s with max|x| / s <= 6, then each x / s to the
    nearest e2m1 value (halfway cases to the smaller magnitude), sign kept.
    Returns (codes uint8 [..., d/2], element 2i in the low nibble; scales
    uint8 [..., d/16])."""
    d = x.shape[-1]
    g = x.float().reshape(*x.shape[:-1], d // 16, 16)
    table = torch.tensor(_ue4m3_table(), dtype=torch.float32, device=x.device)
    target = (g.abs().amax(-1) / 6.0).contiguous()
    sc = torch.searchsorted(table, target).clamp(max=126)
    sval = table[sc].unsqueeze(-1)
    q = torch.where(sval > 0, g / torch.where(sval > 0, sval, torch.ones_like(sval)),
                    torch.zeros_like(g))
    mids = torch.tensor([(a + b) / 2 for a, b in zip(_E2M1_GRID, _E2M1_GRID[1:])],
                        dtype=torch.float32, device=x.device)
    idx = torch.searchsorted(mids, q.abs().contiguous())
    code = (idx | torch.where(q < 0, 8, 0)).to(torch.uint8).reshape(*x.shape[:-1], d)
    packed = code[..., 0::2] | (code[..., 1::2] << 4)
    return packed.contiguous(), sc.to(torch.uint8).contiguous()


def needle_upper(w: Workload) -> int:
    first = w.q_pos0 // w.block_size
    return first if first > 0 else (w.q_pos0 + w.q_len - 1) // w.block_size


def make_inputs(w: Workload, seed: int = 0, device="cpu") -> Dict[str, torch.Tensor]:
    """Inputs of workload ``w`` on ``device``: q, k, v, q_idx, k_idx (+ needle ids)."""
    gen = torch.Generator(device=device).manual_seed(seed)
    dt = w.torch_dtype
    s_main = 1.0 if w.dtype == "f32" else 1.0 / math.sqrt(w.head_dim)
    s_idx = 1.0 if w.dtype == "f32" else 1.0 / math.sqrt(w.index_dim)
    B, Sq, Skv = w.batch, w.q_len, w.kv_len
    nvfp4 = w.index_dtype == "nvfp4"
    q = _draw(gen, (B * Sq, w.num_q_heads, w.head_dim), s_main, w.torch_qk_dtype)
    k = _draw(gen, (B * Skv, w.num_kv_heads, w.head_dim), s_main, w.torch_qk_dtype)
    v = _draw(gen, (B * Skv, w.num_kv_heads, w.head_dim), s_main, dt)
    q_idx = _draw(gen, (B * Sq, w.num_kv_heads, w.index_dim), s_idx,
                  torch.float32 if nvfp4 else w.torch_index_dtype)
    # k_idx stays fp32 until the needles are in, then is rounded once.
    k_idx32 = _draw(gen, (B * Skv, w.index_dim), s_idx, torch.float32)
    needle_ids = torch.full((B, w.num_kv_heads, max(w.needles, 0)), -1, dtype=torch.int64,
                            device=gen.device)
    if w.needles > 0:
        upper = needle_upper(w)
        if upper < w.needles:
            raise ValueError(f"{w.name}: only {upper} past blocks for {w.needles} needles")
        qi = q_idx.view(B, Sq, w.num_kv_heads, w.index_dim)
        kv = k_idx32.view(B, Skv, w.index_dim)
        for b in range(B):
            for g in range(w.num_kv_heads):
                blocks = torch.randperm(upper, generator=gen, device=gen.device)[: w.needles]
                needle_ids[b, g] = blocks
                shift = 0.5 * qi[b, :, g, :].float().mean(dim=0)
                for c in blocks.tolist():
                    lo = c * w.block_size
                    hi = min(lo + w.block_size, Skv)
                    kv[b, lo:hi] += shift
    out = {
        "q": q.view(B, Sq, w.num_q_heads, w.head_dim),
        "k": k.view(B, Skv, w.num_kv_heads, w.head_dim),
        "v": v.view(B, Skv, w.num_kv_heads, w.head_dim),
        "needles": needle_ids,
    }
    if nvfp4:
        qc, qs = quantize_nvfp4(q_idx)
        kc, ks = quantize_nvfp4(k_idx32)
        di = w.index_dim
        out.update(q_idx=qc.view(B, Sq, w.num_kv_heads, di // 2),
                   q_idx_scale=qs.view(B, Sq, w.num_kv_heads, di // 16),
                   k_idx=kc.view(B, Skv, di // 2), k_idx_scale=ks.view(B, Skv, di // 16))
        return out
    out.update(q_idx=q_idx.view(B, Sq, w.num_kv_heads, w.index_dim),
               k_idx=k_idx32.to(w.torch_index_dtype).view(B, Skv, w.index_dim))
    return out


def sample_rows(w: Workload, n: int, seed: int = 0) -> list:
    """``n`` query rows spread evenly over positions, with a seeded jitter.

    Always includes the first and the last row of the batch.
    """
    R = w.rows
    if n >= R:
        return list(range(R))
    gen = torch.Generator().manual_seed(seed + 1)
    base = torch.linspace(0, R - 1, n).long()
    jitter = torch.randint(-3, 4, (n,), generator=gen)
    rows = (base + jitter).clamp(0, R - 1)
    rows[0] = 0
    rows[-1] = R - 1
    return sorted(set(rows.tolist()))


def scaled(w: Workload, name: Optional[str] = None, **kw) -> Workload:
    """A smaller test case with the same structure as ``w``."""
    return w.with_(name=name or (w.name + "_scaled"), **kw)


def make_varlen_inputs(lens_q, lens_k, num_q_heads: int, num_kv_heads: int, head_dim: int,
                       index_dim: int, dtype: str = "bf16", seed: int = 0,
                       device="cpu") -> Dict[str, object]:
    """Packed inputs of a batch of sequences of different lengths: sequence b
    has lens_q[b] query rows (its last tokens) and lens_k[b] keys.  Same draws
    as make_inputs (N(0,1) scaled by 1/sqrt(d) for bf16, order q, k, v, q_idx,
    k_idx, one generator), over the packed rows, without needles; returns q
    [total_q, Hq, D], k, v [total_k, Hkv, D], q_idx [total_q, Hkv, di], k_idx
    [total_k, di] and the prefix sums cu_q, cu_k (Python lists)."""
    if len(lens_q) != len(lens_k) or any(a < 0 or a > b for a, b in zip(lens_q, lens_k)):
        raise ValueError("need 0 <= lens_q[b] <= lens_k[b] for every sequence")
    gen = torch.Generator(device=device).manual_seed(seed)
    dt = torch.float32 if dtype == "f32" else torch.bfloat16
    s_main = 1.0 if dtype == "f32" else 1.0 / math.sqrt(head_dim)
    s_idx = 1.0 if dtype == "f32" else 1.0 / math.sqrt(index_dim)
    tq, tk = sum(lens_q), sum(lens_k)
    cu_q, cu_k = [0], [0]
    for a, b in zip(lens_q, lens_k):
        cu_q.append(cu_q[-1] + a)
        cu_k.append(cu_k[-1] + b)
    return {
        "q": _draw(gen, (tq, num_q_heads, head_dim), s_main, dt),
        "k": _draw(gen, (tk, num_kv_heads, head_dim), s_main, dt),
        "v": _draw(gen, (tk, num_kv_heads, head_dim), s_main, dt),
        "q_idx": _draw(gen, (tq, num_kv_heads, index_dim), s_idx, dt),
        "k_idx": _draw(gen, (tk, index_dim), s_idx, dt),
        "cu_q": cu_q,
        "cu_k": cu_k,
    }
