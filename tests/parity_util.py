"""Comparison helpers for the GPU-vs-oracle parity tests.

Tolerances (written here, derived in the design notes):
  * bf16 problems: attention output max-abs <= 2e-2 and relative Frobenius
    <= 1e-2 (the stated bar for bf16 inputs).
  * fp32 problems: every step runs in fp32 with fp32 partial states, so the
    error is a few fp32 roundings of O(1) values summed over <= 4096 keys:
    max-abs <= 1e-4, relative Frobenius <= 1e-5.
  * block scores: fp32 accumulation of <= 128 exact products against fp64:
    |err| <= 2e-4 + 1e-5 |s|.
  * log-normaliser (lse, an auxiliary output): fp32 problems 1e-4; bf16
    problems sum P in the bf16 the P V product takes, whose per-element
    relative error is below 2^-8, so the normaliser is off by < 2^-8 relative
    and lse (its log) by < 4e-3: atol 5e-3.
  * selections: bit-exact on "decided" rows, where the gap between the last
    kept and the first dropped earlier block exceeds 1e-3 of their magnitude
    (or every visible block is kept); on the other rows the GPU choice must be
    a valid top-k within that 1e-3 band.
"""
import numpy as np
import torch

REL_GAP = 1e-3


def tol(dtype: str):
    return (2e-2, 1e-2) if dtype == "bf16" else (1e-4, 1e-5)


def assert_close_lse(gpu: np.ndarray, ref: np.ndarray, dtype: str):
    if dtype == "bf16":
        np.testing.assert_allclose(gpu, ref, rtol=0, atol=5e-3)
    else:
        np.testing.assert_allclose(gpu, ref, rtol=1e-4, atol=1e-4)


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy()


def rel_fro(a: np.ndarray, b: np.ndarray) -> float:
    return float(np.linalg.norm((a - b).ravel()) / max(np.linalg.norm(b.ravel()), 1e-30))


def assert_close_out(gpu: np.ndarray, ref: np.ndarray, dtype: str, what: str = "out"):
    atol, rfro = tol(dtype)
    assert np.all(np.isfinite(gpu)), f"{what}: non-finite GPU values"
    err = float(np.max(np.abs(gpu - ref))) if gpu.size else 0.0
    fro = rel_fro(gpu, ref) if gpu.size else 0.0
    assert err <= atol and fro <= rfro, f"{what}: max-abs {err:.3g} (<= {atol}), rel-Fro {fro:.3g} (<= {rfro})"
    return err, fro


def check_selection(gpu_q2k: np.ndarray, ora_q2k: np.ndarray, ora_bm: np.ndarray,
                    positions: np.ndarray, Bk: int, k: int):
    """gpu_q2k / ora_q2k: [Hkv, R, k]; ora_bm: [Hkv, R, nblk]; positions: t of each row.

    Returns (decided, agreeing_decided, undecided) counts.
    """
    Hkv, R, _ = ora_q2k.shape
    decided = agree = undecided = 0
    for n in range(R):
        t = int(positions[n])
        c_t = t // Bk
        ksel = min(k, c_t + 1)
        need = ksel - 1
        for g in range(Hkv):
            got = gpu_q2k[g, n]
            chosen = [int(c) for c in got if c >= 0]
            # validity on every row
            assert len(chosen) == ksel, (g, n, got)
            assert list(got[ksel:]) == [-1] * (k - ksel), (g, n, got)
            assert chosen == sorted(set(chosen)) and c_t in chosen, (g, n, got)
            assert all(0 <= c <= c_t for c in chosen), (g, n, got)
            if need == c_t:
                decided += 1
                agree += int(np.array_equal(got, ora_q2k[g, n]))
                assert np.array_equal(got, ora_q2k[g, n]), (g, n, got, ora_q2k[g, n])
                continue
            sc = ora_bm[g, n, :c_t]
            order = np.sort(sc)[::-1]
            a, b = order[need - 1] if need > 0 else np.inf, order[need]
            band = REL_GAP * max(abs(a), abs(b)) if need > 0 else 0.0
            if need == 0 or (a - b) > band:
                decided += 1
                ok = np.array_equal(got, ora_q2k[g, n])
                agree += int(ok)
                assert ok, (g, n, t, got, ora_q2k[g, n])
            else:
                undecided += 1
                earlier = [c for c in chosen if c != c_t]
                rest = [c for c in range(c_t) if c not in earlier]
                assert all(sc[c] >= b - band for c in earlier), (g, n)
                assert all(sc[c] <= a + band for c in rest), (g, n)
    return decided, agree, undecided


def check_selection_properties(q2k: torch.Tensor, q_pos0: int, Sq: int, Bk: int):
    """Properties that hold at any size, checked on the device for every row:
    the local block is present, min(k, visible) distinct ascending visible ids
    and -1 padding after them."""
    Hkv, T, k = q2k.shape
    dev = q2k.device
    r = torch.arange(T, device=dev)
    t = q_pos0 + (r % Sq)
    c_t = (t // Bk).to(torch.int32)
    ksel = torch.clamp(c_t + 1, max=k)
    slot = torch.arange(k, device=dev)
    valid = slot[None, :] < ksel[:, None]                         # [T, k]
    q = q2k.to(torch.int64)
    assert bool(((q >= 0) == valid[None]).all()), "padding / count"
    assert bool((torch.where(valid[None], q, torch.zeros_like(q)) <= c_t[None, :, None].to(torch.int64)).all())
    # ascending among valid, last valid = local block (the largest visible id)
    inc = (q[..., 1:] > q[..., :-1]) | ~valid[None, :, 1:]
    assert bool(inc.all()), "not strictly ascending"
    last = torch.gather(q, 2, (ksel - 1).to(torch.int64)[None, :, None].expand(Hkv, T, 1))[..., 0]
    assert bool((last == c_t[None].to(torch.int64)).all()), "local block missing"
