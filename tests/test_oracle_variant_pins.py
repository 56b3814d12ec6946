"""Pins of the oracle's selection variants against things other than itself.

Landmark refiner (HSA summary page, Implementation: a cross-attention layer
refines the mean-pooled landmark; reading: the pooled landmark L0 = mean(K) W_L
queries the chunk's own keys, L = L0 + softmax(L0 W_q (K W_k)^T / sqrt(d)) K W_v):
  * torch's scaled_dot_product_attention (float64) on the same projections;
  * W_v = 0 leaves the pinned plain landmark unchanged;
  * W_q = 0 makes the attention uniform: L = mean(K) (W_L + W_v) (numpy);
  * constant chunks: L = k (W_L + W_v) whatever W_q and W_k;
  * a chunk with one dominant key: L = L0 + K_u* W_v.
Quest scoring (value-of-information router page, abstract: block scoring such
as Quest under the router; reading: per-channel max/min of the chunk's keys,
score = sum_h sum_e max(q_h[e] Mx[e], q_h[e] Mn[e])):
  * the summaries against numpy's channel max and min;
  * the score bounds every key's group logit from above (Quest's property);
  * equality for single-key chunks (S = 1) and constant chunks;
  * all-positive and all-negative queries reduce to q . Mx and q . Mn;
  * ranking, ties and the router against a Python brute-force sort.
"""
import math

import numpy as np
import pytest
import torch

import oracle


def _rand(shape, seed, scale=1.0, dtype=torch.float32):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(*shape, generator=g) * scale).to(dtype)


def _weights(d, seed, dtype=torch.float32, zero=()):
    names = ("W_L", "W_q", "W_k", "W_v")
    out = {}
    for i, n in enumerate(names):
        w = _rand((d, d), seed + i, 1.0 / math.sqrt(d), dtype)
        out[n] = torch.zeros_like(w) if n in zero else w
    return out


def _chunk_keys(K, S):
    """K [B,T,Hkv,d] -> [B,Hkv,C,S,d] float64 of the complete chunks."""
    B, T, Hkv, d = K.shape
    C = T // S
    return K[:, :C * S].double().reshape(B, C, S, Hkv, d).permute(0, 3, 1, 2, 4).numpy()


# ---------------------------------------------------------------------------- refiner

@pytest.mark.parametrize("dtype,d,S", [(torch.float32, 16, 8), (torch.bfloat16, 32, 16), (torch.float32, 8, 32)])
def test_refiner_matches_sdpa(dtype, d, S):
    B, Hkv, T = 2, 3, 5 * S + 3
    K = _rand((B, T, Hkv, d), 1, 1.5, dtype)
    W = _weights(d, 10, dtype)
    # larger W_q so the attention is far from uniform
    W["W_q"] = (W["W_q"].float() * 6.0).to(dtype)
    L = oracle.landmarks_refined(K, W["W_L"], W["W_q"], W["W_k"], W["W_v"], S)
    L0 = oracle.landmarks(K, W["W_L"], S)
    Kc = torch.from_numpy(_chunk_keys(K, S))                    # [B,Hkv,C,S,d]
    Wd = {n: w.double() for n, w in W.items()}
    q = torch.from_numpy(L0) @ Wd["W_q"]                         # [B,Hkv,C,d]
    kk, vv = Kc @ Wd["W_k"], Kc @ Wd["W_v"]
    att = torch.nn.functional.scaled_dot_product_attention(q.unsqueeze(-2), kk, vv).squeeze(-2)
    ref = L0 + att.numpy()
    assert np.abs(L - ref).max() <= 1e-10 * np.abs(ref).max()
    # and the attention is peaked enough that a softmax mistake would show
    p = torch.softmax((q.unsqueeze(-2) @ kk.transpose(-1, -2)).squeeze(-2) / math.sqrt(d), -1)
    assert float(p.max()) > 0.5


def test_refiner_without_value_path_is_the_plain_landmark():
    d, S = 16, 8
    K = _rand((1, 6 * S, 2, d), 2)
    W = _weights(d, 20, zero=("W_v",))
    L = oracle.landmarks_refined(K, W["W_L"], W["W_q"], W["W_k"], W["W_v"], S)
    assert np.array_equal(L, oracle.landmarks(K, W["W_L"], S))


def test_refiner_with_zero_query_projection_is_uniform_attention():
    d, S = 16, 8
    K = _rand((2, 7 * S + 5, 2, d), 3)
    W = _weights(d, 30, zero=("W_q",))
    L = oracle.landmarks_refined(K, W["W_L"], W["W_q"], W["W_k"], W["W_v"], S)
    mean = _chunk_keys(K, S).mean(axis=3)                        # numpy chunk means [B,Hkv,C,d]
    ref = mean @ (W["W_L"].double().numpy() + W["W_v"].double().numpy())
    assert np.abs(L - ref).max() <= 1e-12 * max(1.0, np.abs(ref).max())


def test_refiner_constant_chunks():
    d, S, C = 8, 16, 5
    base = _rand((1, C, 1, 2, d), 4)                             # one key per (chunk, kv head)
    K = base.expand(1, C, S, 2, d).reshape(1, C * S, 2, d).contiguous()
    W = _weights(d, 40)
    W["W_k"] = W["W_k"] * 50.0                                   # any attention pattern: all keys are equal
    L = oracle.landmarks_refined(K, W["W_L"], W["W_q"], W["W_k"], W["W_v"], S)
    k = base[0, :, 0].double().numpy().transpose(1, 0, 2)        # [Hkv,C,d]
    ref = k @ (W["W_L"].double().numpy() + W["W_v"].double().numpy())
    assert np.abs(L[0] - ref).max() <= 1e-12 * max(1.0, np.abs(ref).max())


def test_refiner_one_dominant_key():
    d, S = 8, 8
    e1, e2 = np.eye(d)[0], np.eye(d)[1]
    keys = np.tile(e1, (S, 1))
    ustar = 5
    keys[ustar] = e1 + 5.0 * e2                                  # the key most aligned with the pooled landmark
    K = torch.from_numpy(keys).float().view(1, S, 1, d)
    eye = torch.eye(d)
    beta = 400.0 * math.sqrt(d)
    L = oracle.landmarks_refined(K, eye, eye, eye * beta, eye, S)
    L0 = keys.mean(0)
    ref = L0 + keys[ustar]                                       # softmax is one-hot at u*
    assert np.abs(L[0, 0, 0] - ref).max() <= 1e-12


# ---------------------------------------------------------------------------- Quest

def test_quest_summaries_are_channel_max_and_min():
    # shifted key sets make every channel's max negative or its min positive too
    for dtype, shift in ((torch.float32, 0.0), (torch.bfloat16, 0.0), (torch.float32, 20.0), (torch.float32, -20.0)):
        K = (_rand((2, 9 * 16 + 7, 3, 32), 5, 2.0) + shift).to(dtype)
        Lq = oracle.quest_summaries(K, 16)
        Kc = _chunk_keys(K, 16)
        assert np.array_equal(Lq[..., :32], Kc.max(axis=3))
        assert np.array_equal(Lq[..., 32:], Kc.min(axis=3))


def _all_rows(B, T):
    return np.repeat(np.arange(B), T), np.tile(np.arange(T), B)


def _group_logits(Q, K, S):
    """max over each chunk's keys of the group-summed logit, and the sum over heads of
    each head's own max: [B*T, Hkv, C] each (float64)."""
    B, T, H, d = Q.shape
    Hkv = K.shape[2]
    G = H // Hkv
    Kc = _chunk_keys(K, S)                                       # [B,Hkv,C,S,d]
    Qd = Q.double().numpy().reshape(B, T, Hkv, G, d)
    per = np.einsum("btjgd,bjcsd->btjcgs", Qd, Kc)               # [B,T,Hkv,C,G,S]
    joint = per.sum(4).max(-1)
    sep = per.max(-1).sum(-1)
    C = Kc.shape[2]
    return joint.reshape(B * T, Hkv, C), sep.reshape(B * T, Hkv, C)


def test_quest_score_bounds_every_key():
    B, T, H, Hkv, d, S = 2, 6 * 16 + 5, 6, 2, 16, 16
    Q = _rand((B, T, H, d), 6)
    K = _rand((B, T, Hkv, d), 7)
    Lq = oracle.quest_summaries(K, S)
    rb, rt = _all_rows(B, T)
    sel = oracle.select_quest(Q.reshape(B * T, H, d), rb, rt, Lq, S, 3, 0.0, H, want_all=True)
    joint, sep = _group_logits(Q, K, S)
    s = sel["allscores"]
    live = np.isfinite(s)
    assert live.sum() > 0
    assert (s[live] >= sep[live] - 1e-9).all()
    assert (sep[live] >= joint[live] - 1e-9).all()
    assert (s[live] > joint[live] + 1e-3).mean() > 0.5          # not an equality on random data


@pytest.mark.parametrize("mode", ["single_key", "constant"])
def test_quest_score_is_exact_when_the_chunk_has_one_key_value(mode):
    B, H, Hkv, d = 1, 8, 2, 16
    if mode == "single_key":
        S, T = 1, 40
        K = _rand((B, T, Hkv, d), 8)
    else:
        S, C = 8, 6
        base = _rand((B, C, 1, Hkv, d), 9)
        K = base.expand(B, C, S, Hkv, d).reshape(B, C * S, Hkv, d).contiguous()
        T = C * S
    Q = _rand((B, T, H, d), 10)
    Lq = oracle.quest_summaries(K, S)
    rb, rt = _all_rows(B, T)
    sel = oracle.select_quest(Q.reshape(B * T, H, d), rb, rt, Lq, S, 2, 0.0, H, want_all=True)
    joint, _ = _group_logits(Q, K, S)
    live = np.isfinite(sel["allscores"])
    assert np.abs(sel["allscores"][live] - joint[live]).max() <= 1e-12


@pytest.mark.parametrize("sign", [1.0, -1.0])
def test_quest_sign_cases(sign):
    B, T, H, Hkv, d, S = 1, 5 * 8, 4, 2, 16, 8
    Q = (_rand((B, T, H, d), 11).abs() * sign)
    K = _rand((B, T, Hkv, d), 12)
    Lq = oracle.quest_summaries(K, S)
    rb, rt = _all_rows(B, T)
    sel = oracle.select_quest(Q.reshape(B * T, H, d), rb, rt, Lq, S, 2, 0.0, H, want_all=True)
    Kc = _chunk_keys(K, S)
    M = Kc.max(axis=3) if sign > 0 else Kc.min(axis=3)          # [B,Hkv,C,d]
    qbar = Q.double().numpy().reshape(B, T, Hkv, H // Hkv, d).sum(3)
    ref = np.einsum("btjd,bjcd->btjc", qbar, M).reshape(B * T, Hkv, -1)
    live = np.isfinite(sel["allscores"])
    assert np.abs(sel["allscores"][live] - ref[live]).max() <= 1e-12


@pytest.mark.parametrize("tau", [0.0, 0.25])
def test_quest_ranking_matches_brute_force(tau):
    """Integer-valued inputs give exact scores with many ties; the ranking, the
    tie rule (lower chunk first), keff and the router rule follow a plain sort."""
    B, T, H, Hkv, d, S, k = 2, 12 * 4 + 3, 4, 2, 8, 4, 3
    g = torch.Generator().manual_seed(13)
    Q = torch.randint(-2, 3, (B, T, H, d), generator=g).float()
    K = torch.randint(-1, 2, (B, T, Hkv, d), generator=g).float()
    Lq = oracle.quest_summaries(K, S)
    rb, rt = _all_rows(B, T)
    sel = oracle.select_quest(Q.reshape(B * T, H, d), rb, rt, Lq, S, k, tau, H, want_all=True)
    kmax = 2 * k if tau > 0 else k
    ties = 0
    for r in range(B * T):
        nc = min(rt[r] // S, T // S)
        for j in range(Hkv):
            s = sel["allscores"][r, j, :nc]
            order = sorted(range(nc), key=lambda c: (-s[c], c))
            ke = min(k, nc)
            if tau > 0 and nc > k and (s[order[k - 1]] - s[order[k]]) < tau * abs(s[order[k - 1]]):
                ke = min(2 * k, nc)
            ties += len(set(s.tolist())) < nc
            assert sel["keff"][r, j] == ke
            assert list(sel["idx"][r, j, :ke]) == order[:ke]
            assert all(x == -1 for x in sel["idx"][r, j, ke:kmax])
    assert ties > 10
