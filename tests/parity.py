"""Comparison rules between the CUDA path and the CPU oracle.

* Landmarks: bf16 values may differ from the oracle's by one bf16 ulp plus
  the fp32 accumulation error of the d-term projection, bounded here by
  2^-17 * max|L| (the GPU sums in fp32, the oracle in fp64).  So a value next
  to a rounding boundary may land on either side, and a value that cancels to
  nearly zero (whose bf16 ulp is tiny) may differ by the absolute fp32 error.
  fp32 values must be within 1e-5.
* Selection: chunk indices are bit-exact, except where the oracle's scores
  around the cut lie within REL = 1e-3 (relative) of each other.  There, any
  GPU set that differs from the oracle's only among such near-tied chunks is
  accepted.  The router decision is accepted either way when
  |(s_k - s_{k+1}) - tau*|s_k|| <= REL*|s_k|.  GPU scores must match the
  oracle's scores of the same chunks within REL relative to the row's top score.
* Output: max-abs 1e-4 (fp32) / 2e-2 (bf16) against the oracle's output for the
  selection.  For a row whose GPU selection differs (validly) from the
  oracle's, the expectation is the oracle run on that validated selection, with
  the oracle's own fp64 scores.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle

REL = 1e-3
OUT_TOL = {torch.float32: 1e-4, torch.bfloat16: 2e-2}


def bf16_ulp(x: np.ndarray) -> np.ndarray:
    ax = np.abs(x)
    e = np.floor(np.log2(np.where(ax > 0, ax, 1.0)))
    e = np.maximum(e, -126)
    return np.ldexp(1.0, (e - 7).astype(np.int64))


def check_landmarks(L_gpu: torch.Tensor, L_orc: np.ndarray) -> dict:
    g = L_gpu.double().cpu().numpy()
    diff = np.abs(g - L_orc)
    if L_gpu.dtype == torch.bfloat16:
        atol = 2.0 ** -17 * float(np.abs(L_orc).max()) if L_orc.size else 0.0
        bad = diff > bf16_ulp(L_orc) * 1.0000001 + atol
        assert not bad.any(), (f"{bad.sum()} landmark values differ by more than one bf16 ulp + {atol:.2e} "
                               f"(worst: gpu {g[bad][:3]} oracle {L_orc[bad][:3]})")
        return {"flips": int((diff > 0).sum()), "n": diff.size}
    assert diff.max() <= 1e-5, f"fp32 landmark max diff {diff.max()}"
    return {"flips": 0, "n": diff.size, "max_diff": float(diff.max())}


def check_selection(idx, score, keff, orc_sel: dict, ncand: np.ndarray, k: int, tau: float) -> dict:
    """idx/score/keff: GPU outputs flattened to [n, Hkv, kmax] / [n, Hkv].
    orc_sel: oracle select() output with allscores, rows in the same order.
    ncand: [n] candidate counts.  Returns counts and the rows that were accepted
    on a near tie (with the GPU selection validated)."""
    idx = np.asarray(idx)
    score = np.asarray(score, dtype=np.float64)
    keff = np.asarray(keff)
    n, Hkv, kmax = idx.shape
    oidx, okeff, alls = orc_sel["idx"], orc_sel["keff"], orc_sel["allscores"]
    exact = ties = 0
    tie_rows = []
    for r in range(n):
        nc = int(ncand[r])
        for j in range(Hkv):
            ke, oke = int(keff[r, j]), int(okeff[r, j])
            gi = idx[r, j, :ke]
            s_all = alls[r, j, :nc]
            top = float(np.max(np.abs(s_all))) if nc else 1.0
            assert np.all(idx[r, j, ke:] == -1) and np.all(np.isneginf(score[r, j, ke:])), (r, j, "padding")
            if nc:
                assert np.all((gi >= 0) & (gi < nc)), (r, j, "not a candidate", gi, nc)
                assert len(set(gi.tolist())) == ke, (r, j, "duplicate chunk")
                np.testing.assert_allclose(score[r, j, :ke], s_all[gi], rtol=0, atol=REL * max(top, 1e-30),
                                           err_msg=f"row {r} kv {j}: scores")
            if ke == oke and np.array_equal(gi, oidx[r, j, :oke]):
                exact += 1
                continue
            # near-tie acceptance
            order = sorted(range(nc), key=lambda c: (-s_all[c], c))
            srt = s_all[order]
            base = min(k, nc)
            allowed = {oke}
            if tau > 0 and nc > k:
                sk, sk1 = srt[k - 1], srt[k]
                if abs((sk - sk1) - tau * abs(sk)) <= REL * abs(sk):
                    allowed |= {base, min(2 * k, nc)}
            assert ke in allowed, (r, j, "keff", ke, oke, allowed)
            if ke == 0:
                ties += 1
                continue
            s_cut = srt[ke - 1]
            band = REL * max(abs(s_cut), 1e-30)
            gset, oset = set(gi.tolist()), set(order[:ke])
            for c in gset ^ oset:
                assert abs(s_all[c] - s_cut) <= band, (r, j, "set differs outside the tie band", c, s_all[c], s_cut)
            gs = s_all[gi]
            assert np.all(gs[:-1] >= gs[1:] - REL * top), (r, j, "order")
            ties += 1
            tie_rows.append((r, j))
    return {"exact": exact, "ties": ties, "tie_rows": tie_rows}


def selection_mismatch_rate(idx, keff, orc_sel) -> float:
    """Fraction of (row, kv head) selections whose kept SET differs from the
    oracle's (idx/keff: GPU outputs flattened to [n, Hkv, kmax] / [n, Hkv])."""
    idx, keff = np.asarray(idx), np.asarray(keff)
    n, Hkv, _ = idx.shape
    bad = 0
    for r in range(n):
        for j in range(Hkv):
            ke, oke = int(keff[r, j]), int(orc_sel["keff"][r, j])
            if ke != oke or set(idx[r, j, :ke].tolist()) != set(orc_sel["idx"][r, j, :oke].tolist()):
                bad += 1
    return bad / max(1, n * Hkv)


def expected_output(Qr, row_b, K, V, S, orc_sel, idx, keff, tie_rows):
    """Oracle output for the oracle selection, with the validated GPU selection
    substituted in the near-tie rows."""
    sel = {k: np.array(v, copy=True) for k, v in orc_sel.items() if k in ("idx", "score", "keff")}
    alls = orc_sel["allscores"]
    for (r, j) in tie_rows:
        ke = int(keff[r, j])
        sel["keff"][r, j] = ke
        sel["idx"][r, j, :] = -1
        sel["score"][r, j, :] = -np.inf
        sel["idx"][r, j, :ke] = idx[r, j, :ke]
        sel["score"][r, j, :ke] = alls[r, j, idx[r, j, :ke]]
    if K.numel() * K.element_size() > (4 << 30):
        return oracle.attend_gathered(Qr, row_b, K, V, S, sel)
    return oracle.attend(Qr, row_b, K.cpu(), V.cpu(), S, sel)


def check_output(O_gpu_rows: torch.Tensor, O_exp: np.ndarray, dtype) -> float:
    g = O_gpu_rows.double().cpu().numpy()
    err = float(np.max(np.abs(g - O_exp))) if g.size else 0.0
    assert err <= OUT_TOL[dtype], f"output max-abs error {err} > {OUT_TOL[dtype]}"
    return err
