"""CPU oracle for Hierarchical Sparse Attention -- TEST INFRASTRUCTURE ONLY.

A plain, slow, fp64 restatement of the method on the HSA summary page
("Every Token Counts 16m Context": Core Technique and Implementation) and of the
gap router on the value-of-information router page.  The arithmetic lives in
``hsa_oracle.c`` (compiled by ``oracle/build.py``); this wrapper only marshals
arrays.  Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may use it.  It never imports the CUDA library and the library
never imports it.

Parity pins (tests/test_oracle_pins.py): bf16 rounding against torch's
conversion; landmarks against numpy chunk means (W_L = I), a one-hot W_L
(orientation), constant chunks and linearity; selection against exact-integer
brute force with ties, the strict-past candidate rule, the group sum and the
router limits; attention against closed forms (constant-V chunks, V = 1, a
two-chunk sigmoid, a single aligned key), convexity, torch SDPA for single
candidate rows, and the exhaustive limit k >= #candidates; the backward against
central finite differences of the forward above (selection held fixed) and the
closed forms of its sums (sum_u dV_u, the per-chunk sum of dK, sum_i ds_i = 0).
Selection variants (tests/test_oracle_variant_pins.py): the landmark refiner
against torch SDPA, W_v = 0, W_q = 0 and constant chunks; Quest scoring against
its upper-bound property, equality for single-key and constant chunks, the
sign cases, numpy's channel max/min, and brute-force ranking.
"""
from __future__ import annotations

import ctypes

import numpy as np
import torch

from . import build as _build

_F32, _BF16, _F64 = 0, 1, 2
_lib = None


def _bind(lib: ctypes.CDLL) -> ctypes.CDLL:
    """Declare the argument types of the oracle's C entry points on a loaded library."""
    P, I, LL, D = ctypes.c_void_p, ctypes.c_int, ctypes.c_longlong, ctypes.c_double
    lib.hsa_oracle_round.argtypes = [I, P, LL, P]
    lib.hsa_oracle_landmarks.argtypes = [I, I, LL, I, I, I, P, P, P]
    lib.hsa_oracle_select.argtypes = [I, I, I, I, I, LL, I, D, I, LL, P, P, P, P, P, P, P, P]
    lib.hsa_oracle_attend.argtypes = [I, LL, I, I, I, I, I, LL, P, P, P, P, P, P, P, P]
    lib.hsa_oracle_backward.argtypes = [I, I, LL, I, I, I, I, I, LL, P, P, P, P, P, P, P, P, P,
                                        P, P, P, P, P]
    lib.hsa_oracle_landmarks_refined.argtypes = [I, I, LL, I, I, I, P, P, P, P, P, P]
    lib.hsa_oracle_quest_summaries.argtypes = [I, I, LL, I, I, I, P, P]
    lib.hsa_oracle_select_quest.argtypes = [I, I, I, I, I, LL, I, D, I, LL, P, P, P, P, P, P, P, P]
    for f in (lib.hsa_oracle_round, lib.hsa_oracle_landmarks, lib.hsa_oracle_select,
              lib.hsa_oracle_attend, lib.hsa_oracle_backward, lib.hsa_oracle_landmarks_refined,
              lib.hsa_oracle_quest_summaries, lib.hsa_oracle_select_quest):
        f.restype = None
    return lib


def _load():
    global _lib
    if _lib is None:
        _lib = _bind(ctypes.CDLL(_build.build()))
    return _lib


def _buf(x):
    """(dtype code, contiguous numpy array sharing or holding the data)."""
    if isinstance(x, torch.Tensor):
        x = x.detach().cpu().contiguous()
        if x.dtype == torch.bfloat16:
            return _BF16, x.view(torch.int16).numpy()
        if x.dtype == torch.float32:
            return _F32, x.numpy()
        if x.dtype == torch.float64:
            return _F64, x.numpy()
        raise TypeError(f"unsupported dtype {x.dtype}")
    x = np.ascontiguousarray(x)
    if x.dtype == np.float32:
        return _F32, x
    if x.dtype == np.float64:
        return _F64, x
    raise TypeError(f"unsupported dtype {x.dtype}")


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def round_to(dtype: str, x) -> np.ndarray:
    """Round doubles to the storage dtype ("f32" or "bf16"), ties to even; result as float64."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    y = np.empty_like(x)
    _load().hsa_oracle_round({"f32": _F32, "bf16": _BF16}[dtype], _ptr(x), x.size, _ptr(y))
    return y


def landmarks(K, W_L, S: int) -> np.ndarray:
    """fp64 landmarks [B,Hkv,C,d] = mean over each complete chunk's keys, times W_L."""
    dk, Ka = _buf(K)
    dw, Wa = _buf(W_L)
    if dw != dk:
        raise TypeError("K and W_L must share a dtype")
    B, T, Hkv, d = Ka.shape
    C = T // S
    L = np.zeros((B, Hkv, C, d), dtype=np.float64)
    _load().hsa_oracle_landmarks(dk, B, T, Hkv, d, S, _ptr(Ka), _ptr(Wa), _ptr(L))
    return L


def landmarks_stored(K, W_L, S: int, dtype: str) -> np.ndarray:
    """Landmarks as the library stores them: fp64 result rounded once to dtype."""
    return round_to(dtype, landmarks(K, W_L, S))


def landmarks_stored_sliced(K, W_L, S: int, dtype: str, chunks_per_slice: int = 8192) -> np.ndarray:
    """:func:`landmarks_stored` for caches too long for one host copy: K (any
    device) is brought to the host a slice of whole chunks at a time."""
    B, T, Hkv, d = K.shape
    C = T // S
    L = np.empty((B, Hkv, C, d), dtype=np.float64)
    W = W_L.cpu() if isinstance(W_L, torch.Tensor) else W_L
    for b in range(B):
        for c0 in range(0, C, chunks_per_slice):
            c1 = min(C, c0 + chunks_per_slice)
            Ks = K[b:b + 1, c0 * S:c1 * S].cpu()
            L[b:b + 1, :, c0:c1] = landmarks_stored(Ks, W, S, dtype)
    return L


def landmarks_refined(K, W_L, W_q, W_k, W_v, S: int) -> np.ndarray:
    """fp64 refined landmarks [B,Hkv,C,d]: the pooled landmark mean(K) W_L plus
    one head of cross-attention from it (query L0 W_q) to the chunk's keys
    (keys K W_k, values K W_v, scale 1/sqrt(d))."""
    dk, Ka = _buf(K)
    ws = [_buf(w) for w in (W_L, W_q, W_k, W_v)]
    if any(dw != dk for dw, _ in ws):
        raise TypeError("K and the weights must share a dtype")
    B, T, Hkv, d = Ka.shape
    C = T // S
    L = np.zeros((B, Hkv, C, d), dtype=np.float64)
    _load().hsa_oracle_landmarks_refined(dk, B, T, Hkv, d, S, _ptr(Ka), *(_ptr(a) for _, a in ws), _ptr(L))
    return L


def landmarks_refined_stored(K, W_L, W_q, W_k, W_v, S: int, dtype: str) -> np.ndarray:
    """Refined landmarks as the library stores them: rounded once to dtype."""
    return round_to(dtype, landmarks_refined(K, W_L, W_q, W_k, W_v, S))


def quest_summaries(K, S: int) -> np.ndarray:
    """Quest chunk summaries [B,Hkv,C,2d] (fp64 holding stored values): the
    channel-wise max of each complete chunk's keys, then the channel-wise min."""
    dk, Ka = _buf(K)
    B, T, Hkv, d = Ka.shape
    C = T // S
    Lq = np.zeros((B, Hkv, C, 2 * d), dtype=np.float64)
    _load().hsa_oracle_quest_summaries(dk, B, T, Hkv, d, S, _ptr(Ka), _ptr(Lq))
    return Lq


def select_quest(Qr, row_b, row_p, Lq: np.ndarray, S: int, k: int, tau: float, H: int,
                 want_all: bool = False) -> dict:
    """Top-k selection by Quest's criticality bound for query rows Qr [n,H,d]
    against chunk summaries Lq [B,Hkv,C,2d]; same outputs as :func:`select`."""
    dq, Qa = _buf(Qr)
    Lq = np.ascontiguousarray(Lq, dtype=np.float64)
    n, Hq, d = Qa.shape
    assert Hq == H
    B, Hkv, C, d2 = Lq.shape
    assert d2 == 2 * d and H % Hkv == 0
    kmax = 2 * k if tau > 0 else k
    rb = np.ascontiguousarray(row_b, dtype=np.int32)
    rp = np.ascontiguousarray(row_p, dtype=np.int64)
    idx = np.empty((n, Hkv, kmax), dtype=np.int32)
    score = np.empty((n, Hkv, kmax), dtype=np.float64)
    keff = np.empty((n, Hkv), dtype=np.int32)
    alls = np.empty((n, Hkv, C), dtype=np.float64) if want_all else None
    _load().hsa_oracle_select_quest(dq, H, Hkv, d, S, C, k, float(tau), kmax, n, _ptr(rb), _ptr(rp),
                                    _ptr(Qa), _ptr(Lq), _ptr(idx), _ptr(score), _ptr(keff),
                                    _ptr(alls) if alls is not None else None)
    out = {"idx": idx, "score": score, "keff": keff}
    if want_all:
        out["allscores"] = alls
    return out


def select(Qr, row_b, row_p, L: np.ndarray, S: int, k: int, tau: float, H: int,
           want_all: bool = False) -> dict:
    """Top-k selection for query rows Qr [n,H,d] at batches row_b and absolute
    positions row_p against landmarks L [B,Hkv,C,d] (fp64 storage values)."""
    dq, Qa = _buf(Qr)
    L = np.ascontiguousarray(L, dtype=np.float64)
    n, Hq, d = Qa.shape
    assert Hq == H
    B, Hkv, C, dl = L.shape
    assert dl == d and H % Hkv == 0
    kmax = 2 * k if tau > 0 else k
    rb = np.ascontiguousarray(row_b, dtype=np.int32)
    rp = np.ascontiguousarray(row_p, dtype=np.int64)
    idx = np.empty((n, Hkv, kmax), dtype=np.int32)
    score = np.empty((n, Hkv, kmax), dtype=np.float64)
    keff = np.empty((n, Hkv), dtype=np.int32)
    alls = np.empty((n, Hkv, C), dtype=np.float64) if want_all else None
    _load().hsa_oracle_select(dq, H, Hkv, d, S, C, k, float(tau), kmax, n, _ptr(rb), _ptr(rp),
                              _ptr(Qa), _ptr(L), _ptr(idx), _ptr(score), _ptr(keff),
                              _ptr(alls) if alls is not None else None)
    out = {"idx": idx, "score": score, "keff": keff}
    if want_all:
        out["allscores"] = alls
    return out


def attend(Qr, row_b, K, V, S: int, sel: dict) -> np.ndarray:
    """Chunk attention + fusion for rows Qr [n,H,d] given a selection dict
    (idx, score, keff) whose chunk indices refer to K, V [B,Tkv,Hkv,d]."""
    dq, Qa = _buf(Qr)
    dk, Ka = _buf(K)
    dv, Va = _buf(V)
    if not (dq == dk == dv):
        raise TypeError("Q, K, V must share a dtype")
    n, H, d = Qa.shape
    B, Tkv, Hkv, _ = Ka.shape
    idx = np.ascontiguousarray(sel["idx"], dtype=np.int32)
    score = np.ascontiguousarray(sel["score"], dtype=np.float64)
    keff = np.ascontiguousarray(sel["keff"], dtype=np.int32)
    kmax = idx.shape[-1]
    rb = np.ascontiguousarray(row_b, dtype=np.int32)
    O = np.zeros((n, H, d), dtype=np.float64)
    _load().hsa_oracle_attend(dq, Tkv, H, Hkv, d, S, kmax, n, _ptr(rb), _ptr(Qa), _ptr(Ka),
                              _ptr(Va), _ptr(idx), _ptr(score), _ptr(keff), _ptr(O))
    return O


def attend_gathered(Qr, row_b, K, V, S: int, sel: dict) -> np.ndarray:
    """Same as :func:`attend`, but copies only the chunks the selection names
    out of K and V first (torch tensors on any device), so that very long
    caches never need a full host copy."""
    idx = np.asarray(sel["idx"])
    keff = np.asarray(sel["keff"])
    row_b = np.asarray(row_b, dtype=np.int64)
    used = sorted({(int(row_b[r]), int(c)) for r in range(idx.shape[0])
                   for j in range(idx.shape[1]) for c in idx[r, j, :keff[r, j]]})
    remap = {bc: i for i, bc in enumerate(used)}
    Hkv, d = K.shape[2], K.shape[3]
    Kc = torch.empty(1, max(1, len(used)) * S, Hkv, d, dtype=K.dtype)
    Vc = torch.empty_like(Kc)
    for i, (b, c) in enumerate(used):
        Kc[0, i * S:(i + 1) * S] = K[b, c * S:(c + 1) * S].cpu()
        Vc[0, i * S:(i + 1) * S] = V[b, c * S:(c + 1) * S].cpu()
    idx2 = np.full_like(idx, -1)
    for r in range(idx.shape[0]):
        for j in range(idx.shape[1]):
            for i in range(keff[r, j]):
                idx2[r, j, i] = remap[(int(row_b[r]), int(idx[r, j, i]))]
    sel2 = dict(sel, idx=idx2)
    return attend(Qr, np.zeros_like(row_b, dtype=np.int32), Kc, Vc, S, sel2)


def forward_rows(Q, K, V, W_L, S: int, k: int, tau: float, q_pos0: int, rows_b, rows_t,
                 L: np.ndarray | None = None, want_all: bool = False) -> dict:
    """Whole method for the query rows (rows_b[i], rows_t[i]) of Q [B,Tq,H,d]:
    landmarks (unless given, as storage values), selection, attention and
    fusion.  Returns L, the selection and O [n,H,d] (all fp64)."""
    dtype = "bf16" if Q.dtype == torch.bfloat16 else "f32"
    if L is None:
        L = landmarks_stored(K, W_L, S, dtype)
    rows_b = np.asarray(rows_b, dtype=np.int64)
    rows_t = np.asarray(rows_t, dtype=np.int64)
    Qr = Q[torch.as_tensor(rows_b), torch.as_tensor(rows_t)].cpu()
    sel = select(Qr, rows_b, rows_t + q_pos0, L, S, k, tau, Q.shape[2], want_all=want_all)
    if K.numel() * K.element_size() > (4 << 30):
        O = attend_gathered(Qr, rows_b, K, V, S, sel)
    else:
        O = attend(Qr, rows_b, K.cpu(), V.cpu(), S, sel)
    return {"L": L, "sel": sel, "O": O}


def backward(Qr, row_b, K, V, W_L, L, S: int, sel: dict, dO) -> dict:
    """Gradients of the method for rows Qr [n,H,d] (batches row_b) with the
    selection ``sel`` (idx, keff; chunk indices into K, V [B,Tkv,Hkv,d]) held
    fixed.  L [B,Hkv,C,d] holds the landmarks the scores are taken from; dO
    [n,H,d] is the output gradient.  Returns fp64 dQ [n,H,d], dK, dV
    [B,Tkv,Hkv,d], dW [d,d] and dL [B,Hkv,C,d]."""
    dq, Qa = _buf(Qr)
    dk, Ka = _buf(K)
    dv, Va = _buf(V)
    dw, Wa = _buf(W_L)
    if not (dq == dk == dv == dw):
        raise TypeError("Q, K, V, W_L must share a dtype")
    n, H, d = Qa.shape
    B, Tkv, Hkv, _ = Ka.shape
    L = np.ascontiguousarray(L, dtype=np.float64)
    if L.shape != (B, Hkv, Tkv // S, d):
        raise ValueError(f"L has shape {L.shape}, expected {(B, Hkv, Tkv // S, d)}")
    idx = np.ascontiguousarray(sel["idx"], dtype=np.int32)
    keff = np.ascontiguousarray(sel["keff"], dtype=np.int32)
    kmax = idx.shape[-1]
    rb = np.ascontiguousarray(row_b, dtype=np.int32)
    g = np.ascontiguousarray(dO.detach().cpu().double().numpy() if isinstance(dO, torch.Tensor) else dO,
                             dtype=np.float64)
    out = {"dQ": np.empty((n, H, d)), "dK": np.empty((B, Tkv, Hkv, d)), "dV": np.empty((B, Tkv, Hkv, d)),
           "dW": np.empty((d, d)), "dL": np.empty((B, Hkv, L.shape[2], d))}
    _load().hsa_oracle_backward(dq, B, Tkv, H, Hkv, d, S, kmax, n, _ptr(rb), _ptr(Qa), _ptr(Ka), _ptr(Va),
                                _ptr(Wa), _ptr(L), _ptr(idx), _ptr(keff), _ptr(g), _ptr(out["dQ"]),
                                _ptr(out["dK"]), _ptr(out["dV"]), _ptr(out["dW"]), _ptr(out["dL"]))
    return out


__all__ = ["round_to", "landmarks", "landmarks_stored", "landmarks_stored_sliced", "select", "attend",
           "attend_gathered", "forward_rows", "backward"]
