"""Pins of the oracle's backward (oracle.backward) to things other than itself.

The backward differentiates the method with the chunk selection held fixed
(HSA summary page, Implementation: the retrieval scores weight the chunk
outputs, so they carry a gradient; which chunks are kept is a discrete choice).
It is checked against:
  * central finite differences of the oracle's forward (landmarks, scores of
    the fixed slots, chunk attention and fusion), every element of Q, K, V and
    W_L, with and without the gap router;
  * torch autograd of scaled_dot_product_attention where every row keeps one
    chunk (its fusion weight is then 1, so the score path carries nothing);
  * closed forms of sums: sum_u dV_u equals the summed output gradients of the
    rows that keep any chunk, the per-chunk sum of dK equals the landmark
    gradient times W_L^T (the attention part of a chunk's key gradients sums
    to zero), the landmark gradients of a (batch, kv head) sum to zero (the
    fusion softmax's score gradients sum to zero per row), and tokens of the
    trailing partial chunk get no gradient.
"""
import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle


def _problem(seed, B=2, C=5, S=4, tail=3, H=4, Hkv=2, d=4):
    rng = np.random.default_rng(seed)
    T = C * S + tail
    Q = torch.tensor(rng.standard_normal((B, T, H, d)))
    K = torch.tensor(rng.standard_normal((B, T, Hkv, d)))
    V = torch.tensor(rng.standard_normal((B, T, Hkv, d)))
    W = torch.tensor(rng.standard_normal((d, d)) / d ** 0.5)
    dO = rng.standard_normal((B * T, H, d))
    return Q, K, V, W, dO, S


def _rows(Q):
    B, T = Q.shape[:2]
    rb = np.repeat(np.arange(B), T)
    rp = np.tile(np.arange(T), B)
    return Q.reshape(B * T, *Q.shape[2:]), rb, rp


def _loss(Q, K, V, W, S, sel_fixed, dO):
    """<dO, O> for the fixed slots: landmarks and scores recomputed from the inputs."""
    Qr, rb, rp = _rows(Q)
    L = oracle.landmarks(K, W, S)
    allsc = oracle.select(Qr, rb, rp, L, S, 1, 0.0, Q.shape[2], want_all=True)["allscores"]
    idx, keff = sel_fixed["idx"], sel_fixed["keff"]
    score = np.full(idx.shape, -np.inf)
    n, Hkv, km = idx.shape
    for r in range(n):
        for j in range(Hkv):
            for i in range(keff[r, j]):
                score[r, j, i] = allsc[r, j, idx[r, j, i]]
    O = oracle.attend(Qr, rb, K, V, S, {"idx": idx, "score": score, "keff": keff})
    return float(np.sum(O * dO))


def _grads(Q, K, V, W, S, k, tau, dO):
    Qr, rb, rp = _rows(Q)
    L = oracle.landmarks(K, W, S)
    sel = oracle.select(Qr, rb, rp, L, S, k, tau, Q.shape[2])
    return sel, oracle.backward(Qr, rb, K, V, W, L, S, sel, dO)


@pytest.mark.parametrize("k,tau,seed", [(2, 0.0, 1), (2, 0.9, 2), (3, 0.0, 3)])
def test_backward_matches_central_finite_differences(k, tau, seed):
    Q, K, V, W, dO, S = _problem(seed)
    sel, g = _grads(Q, K, V, W, S, k, tau, dO)
    if tau > 0:
        assert (sel["keff"] > k).any(), "the router case must double some rows"
    eps = 1e-6
    for name, X, G in (("Q", Q, g["dQ"].reshape(Q.shape)), ("K", K, g["dK"]), ("V", V, g["dV"]),
                       ("W", W, g["dW"])):
        flat = X.view(-1)
        num = np.empty(flat.numel())
        for i in range(flat.numel()):
            x0 = float(flat[i])
            flat[i] = x0 + eps
            lp = _loss(Q, K, V, W, S, sel, dO)
            flat[i] = x0 - eps
            lm = _loss(Q, K, V, W, S, sel, dO)
            flat[i] = x0
            num[i] = (lp - lm) / (2 * eps)
        err = np.max(np.abs(num - G.reshape(-1)))
        assert err < 1e-7 * max(1.0, np.max(np.abs(num))), f"d{name}: max error {err:.3g}"


def test_single_slot_rows_match_sdpa_autograd():
    """k = 1: each row keeps one chunk with weight 1, so the gradients are those
    of plain softmax attention over that chunk's keys (torch autograd of SDPA)."""
    Q, K, V, W, dO, S = _problem(11, B=2, C=6, S=4, tail=2, H=4, Hkv=2, d=8)
    sel, g = _grads(Q, K, V, W, S, 1, 0.0, dO)
    B, T, H, d = Q.shape
    Hkv, G = K.shape[2], H // K.shape[2]
    Qa, Ka, Va = (x.clone().requires_grad_(True) for x in (Q, K, V))
    loss = torch.zeros((), dtype=torch.float64)
    dOt = torch.tensor(dO).reshape(B, T, H, d)
    for b in range(B):
        for t in range(T):
            r = b * T + t
            for j in range(Hkv):
                if sel["keff"][r, j] == 0:
                    continue
                c = int(sel["idx"][r, j, 0])
                q = Qa[b, t, j * G:(j + 1) * G].unsqueeze(1)                 # [G, 1, d]
                kk = Ka[b, c * S:(c + 1) * S, j].unsqueeze(0).expand(G, S, d)
                vv = Va[b, c * S:(c + 1) * S, j].unsqueeze(0).expand(G, S, d)
                o = F.scaled_dot_product_attention(q, kk, vv)[:, 0]         # [G, d]
                loss = loss + (o * dOt[b, t, j * G:(j + 1) * G]).sum()
    loss.backward()
    assert np.allclose(g["dQ"].reshape(Q.shape), Qa.grad.numpy(), atol=1e-12)
    assert np.allclose(g["dK"], Ka.grad.numpy(), atol=1e-12)   # the landmark share is 0: w = 1
    assert np.allclose(g["dV"], Va.grad.numpy(), atol=1e-12)
    assert np.max(np.abs(g["dW"])) < 1e-13 and np.max(np.abs(g["dL"])) < 1e-13


@pytest.mark.parametrize("tau", [0.0, 0.5])
def test_gradient_sums_closed_forms(tau):
    Q, K, V, W, dO, S = _problem(21, B=2, C=7, S=8, tail=5, H=8, Hkv=2, d=8)
    sel, g = _grads(Q, K, V, W, S, 3, tau, dO)
    B, T, H, d = Q.shape
    Hkv, G = K.shape[2], H // K.shape[2]
    C = T // S
    dOr = dO.reshape(B, T, H, d)
    ke = sel["keff"].reshape(B, T, Hkv)
    for b in range(B):
        for j in range(Hkv):
            # the kept chunks' softmax weights sum to 1 and each in-chunk softmax sums to 1
            expect = sum(dOr[b, t, j * G:(j + 1) * G].sum(0) for t in range(T) if ke[b, t, j] > 0)
            assert np.allclose(g["dV"][b, :, j].sum(0), expect, atol=1e-12)
            # the fusion softmax's score gradients sum to zero in every row
            assert np.allclose(g["dL"][b, j].sum(0), 0.0, atol=1e-12)
            for c in range(C):
                # shifting a chunk's keys by one vector leaves its in-chunk softmax alone,
                # so only the landmark path remains in their summed gradient
                kc = g["dK"][b, c * S:(c + 1) * S, j].sum(0)
                assert np.allclose(kc, g["dL"][b, j, c] @ W.numpy().T, atol=1e-12)
    assert np.all(g["dK"][:, C * S:] == 0) and np.all(g["dV"][:, C * S:] == 0)
    # rows with no candidate have no gradient
    none = sel["keff"].reshape(B, T, Hkv) == 0
    dQ = g["dQ"].reshape(B, T, Hkv, G, d)
    assert none.any() and np.all(dQ[none] == 0)
