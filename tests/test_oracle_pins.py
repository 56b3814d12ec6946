"""Pins for the CPU oracle: each test ties one part of it to something other
than itself (brute force, a closed form, an invariant, a library routine), so
that a dropped term, a wrong sign or index or a transposed operand fails.

Method reference: HSA summary page ("Every Token Counts 16m Context"),
Core Technique and Implementation; gap router: value-of-information router page.
"""
import math
from fractions import Fraction

import numpy as np
import pytest
import scipy.special
import torch
import torch.nn.functional as F

import oracle


def _gen(seed):
    return torch.Generator().manual_seed(seed)


def _full(Q, K, V, W, S, k, tau=0.0, q_pos0=0):
    """Run the oracle on every query row of an fp64 problem."""
    B, Tq, H, d = Q.shape
    L = oracle.landmarks(K, W, S)
    rows_b = np.repeat(np.arange(B), Tq)
    rows_t = np.tile(np.arange(Tq), B)
    Qr = Q.reshape(B * Tq, H, d)
    sel = oracle.select(Qr, rows_b, rows_t + q_pos0, L, S, k, tau, H, want_all=True)
    O = oracle.attend(Qr, rows_b, K, V, S, sel)
    return L, sel, O.reshape(B, Tq, H, d)


# ----------------------------------------------------------------------------- rounding

def test_round_bf16_matches_torch_conversion():
    g = _gen(1)
    x = torch.randn(200000, generator=g) * torch.exp(torch.randn(200000, generator=g) * 12)
    x = torch.cat([x, torch.tensor([3.4e38, -3.4e38, 1e-40, -2e-39, 0.0])]).float()
    ours = oracle.round_to("bf16", x.double().numpy())
    ref = x.to(torch.bfloat16).double().numpy()
    assert np.array_equal(ours, ref)


def test_round_bf16_ties_to_even():
    r = oracle.round_to("bf16", np.array([1 + 2**-8, 1 + 3 * 2**-8, -(1 + 2**-8), 1 + 2**-8 + 2**-30]))
    assert list(r) == [1.0, 1 + 2**-6, -1.0, 1 + 2**-7]


def test_round_f32_is_single_rounding():
    x = np.array([1 + 2**-24, 1 + 3 * 2**-24, math.pi, 1e-45])
    np.testing.assert_array_equal(oracle.round_to("f32", x), x.astype(np.float32).astype(np.float64))


# ----------------------------------------------------------------------------- landmarks

def test_landmarks_identity_projection_is_chunk_mean():
    B, T, Hkv, d, S = 2, 300, 3, 8, 64          # 4 complete chunks and a 44-token tail
    K = torch.randn(B, T, Hkv, d, dtype=torch.float64, generator=_gen(2))
    L = oracle.landmarks(K, torch.eye(d, dtype=torch.float64), S)
    C = T // S
    ref = K[:, :C * S].numpy().reshape(B, C, S, Hkv, d).mean(axis=2).transpose(0, 2, 1, 3)
    assert L.shape == (B, Hkv, C, d)
    np.testing.assert_allclose(L, ref, rtol=0, atol=1e-14)


def test_landmarks_projection_orientation():
    """W_L[e_in][e_out]: a single one at (3, 5) moves input dim 3 to output dim 5."""
    B, T, Hkv, d, S = 1, 256, 2, 8, 64
    K = torch.randn(B, T, Hkv, d, dtype=torch.float64, generator=_gen(3))
    W = torch.zeros(d, d, dtype=torch.float64)
    W[3, 5] = 1.0
    L = oracle.landmarks(K, W, S)
    mean = K.numpy().reshape(B, 4, S, Hkv, d).mean(axis=2).transpose(0, 2, 1, 3)
    np.testing.assert_allclose(L[..., 5], mean[..., 3], rtol=0, atol=1e-14)
    assert np.all(np.delete(L, 5, axis=-1) == 0.0)


def test_landmarks_constant_chunk_equals_row_times_W():
    B, Hkv, d, S, C = 1, 2, 16, 64, 3
    kv = torch.randn(B, C, Hkv, d, dtype=torch.float64, generator=_gen(4))
    K = kv.repeat_interleave(S, dim=1)                         # every key of chunk c equals kv[c]
    W = torch.randn(d, d, dtype=torch.float64, generator=_gen(5))
    L = oracle.landmarks(K, W, S)
    ref = np.einsum("bcje,ef->bjcf", kv.numpy(), W.numpy())
    np.testing.assert_allclose(L, ref, rtol=1e-13, atol=1e-13)


def test_landmarks_linear_and_tail_ignored():
    B, T, Hkv, d, S = 1, 64 * 5 + 17, 2, 8, 64
    g = _gen(6)
    K1 = torch.randn(B, T, Hkv, d, dtype=torch.float64, generator=g)
    K2 = torch.randn(B, T, Hkv, d, dtype=torch.float64, generator=g)
    W = torch.randn(d, d, dtype=torch.float64, generator=g)
    L12 = oracle.landmarks(2.0 * K1 - 3.0 * K2, W, S)
    np.testing.assert_allclose(L12, 2.0 * oracle.landmarks(K1, W, S) - 3.0 * oracle.landmarks(K2, W, S),
                               rtol=1e-12, atol=1e-12)
    K3 = K1.clone()
    K3[:, 5 * S:] = 1e6                                          # the partial chunk has no landmark
    np.testing.assert_array_equal(oracle.landmarks(K3, W, S), oracle.landmarks(K1, W, S))


def test_landmarks_sliced_equals_whole():
    B, T, Hkv, d, S = 2, 64 * 9, 2, 8, 64
    K = torch.randn(B, T, Hkv, d, generator=_gen(7)).to(torch.bfloat16)
    W = (torch.randn(d, d, generator=_gen(8)) / math.sqrt(d)).to(torch.bfloat16)
    np.testing.assert_array_equal(oracle.landmarks_stored_sliced(K, W, S, "bf16", chunks_per_slice=4),
                                  oracle.landmarks_stored(K, W, S, "bf16"))


# ----------------------------------------------------------------------------- selection

@pytest.mark.parametrize("tau", [0.0, 0.25])
def test_select_matches_exact_integer_brute_force(tau):
    """Small-integer Q and L give many exact score ties; ranking must be
    (score desc, chunk asc), candidates the complete chunks strictly before
    the query's chunk, and the router rule applied on exact rationals."""
    rng = np.random.default_rng(9)
    B, T, H, Hkv, d, S, k = 2, 4 * 20 + 3, 4, 2, 3, 4, 3
    C = T // S
    G = H // Hkv
    Q = rng.integers(-2, 3, size=(B, T, H, d)).astype(np.float64)
    L = rng.integers(-2, 3, size=(B, Hkv, C, d)).astype(np.float64)
    rows_b = np.repeat(np.arange(B), T)
    rows_t = np.tile(np.arange(T), B)
    sel = oracle.select(Q.reshape(B * T, H, d), rows_b, rows_t, L, S, k, tau, H)
    kmax = 2 * k if tau > 0 else k
    tau_q = Fraction(tau)
    n_doubled = 0
    for r in range(B * T):
        b, t = int(rows_b[r]), int(rows_t[r])
        ncand = min(t // S, C)
        for j in range(Hkv):
            s = [sum(int(Q[b, t, h, e]) * int(L[b, j, c, e]) for h in range(j * G, (j + 1) * G)
                     for e in range(d)) for c in range(ncand)]
            order = sorted(range(ncand), key=lambda c: (-s[c], c))
            ke = min(k, ncand)
            if tau > 0 and ncand > k and (s[order[k - 1]] - s[order[k]]) < tau_q * abs(s[order[k - 1]]):
                ke = min(2 * k, ncand)
                n_doubled += 1
            assert sel["keff"][r, j] == ke
            assert list(sel["idx"][r, j, :ke]) == order[:ke]
            assert list(sel["score"][r, j, :ke]) == [float(s[c]) for c in order[:ke]]
            assert all(sel["idx"][r, j, ke:kmax] == -1)
            assert all(np.isneginf(sel["score"][r, j, ke:kmax]))
    if tau > 0:
        assert n_doubled > 0


def test_select_group_sum_decides():
    """Two query heads of one kv head disagree; the group sum picks the chunk."""
    L = np.array([[[[1.0, 0.0], [0.0, 1.0]]]])                  # B1 Hkv1 C2 d2
    for q1, want in (([0.0, 2.0], 0), ([0.0, 4.0], 1)):
        Q = np.array([[[3.0, 0.0], q1]])                        # n1 H2 d2: head0 likes chunk 0
        sel = oracle.select(Q, [0], [2 * 4], L, 4, 1, 0.0, 2)
        assert sel["idx"][0, 0, 0] == want
        assert sel["score"][0, 0, 0] == max(3.0, q1[1])


def test_router_threshold_hand_cases():
    """Scores (10, 9.9, ...) give a normalised gap 0.01 < 0.02: k doubles.
    Scores (10, 9.7, ...) give 0.03: it does not.  s_k = 0 never routes."""
    for s2, want in ((9.9, 2), (9.7, 1)):
        L = np.array([[[[10.0], [s2], [5.0], [4.0]]]])
        sel = oracle.select(np.array([[[1.0]]]), [0], [4 * 4], L, 4, 1, 0.02, 1)
        assert sel["keff"][0, 0] == want
        assert sel["idx"][0, 0, 0] == 0
    L = np.array([[[[0.0], [0.0], [-1.0]]]])
    assert oracle.select(np.array([[[1.0]]]), [0], [12], L, 4, 1, 0.02, 1)["keff"][0, 0] == 1


def test_router_limits_and_scale_invariance():
    B, T, H, Hkv, d, S, k = 1, 64 * 12, 4, 2, 16, 64, 3
    g = _gen(10)
    Q = torch.randn(B, T, H, d, dtype=torch.float64, generator=g)
    L = torch.randn(B, Hkv, T // S, d, dtype=torch.float64, generator=g).numpy()
    rb, rt = np.zeros(T, dtype=np.int64), np.arange(T)
    Qr = Q.reshape(T, H, d)
    base = oracle.select(Qr, rb, rt, L, S, k, 0.0, H)
    lo = oracle.select(Qr, rb, rt, L, S, k, 1e-12, H)
    hi = oracle.select(Qr, rb, rt, L, S, k, 1e12, H)
    ncand = np.minimum(rt // S, T // S)[:, None]
    np.testing.assert_array_equal(lo["keff"], base["keff"])
    want = np.broadcast_to(np.where(ncand > k, np.minimum(2 * k, ncand), ncand), hi["keff"].shape)
    np.testing.assert_array_equal(hi["keff"], want)
    np.testing.assert_array_equal(hi["idx"][..., :k], base["idx"])
    scaled = oracle.select(Qr * 2.0, rb, rt, L, S, k, 0.0, H)
    np.testing.assert_array_equal(scaled["idx"], base["idx"])


def test_decode_position_sees_all_complete_chunks():
    B, T, H, Hkv, d, S, k = 1, 64 * 6 + 9, 2, 1, 8, 64, 16
    g = _gen(11)
    K = torch.randn(B, T, Hkv, d, dtype=torch.float64, generator=g)
    Q = torch.randn(B, 1, H, d, dtype=torch.float64, generator=g)
    L = oracle.landmarks(K, torch.eye(d, dtype=torch.float64), S)
    sel = oracle.select(Q.reshape(1, H, d), [0], [T], L, S, k, 0.0, H)
    assert sel["keff"][0, 0] == 6
    assert sorted(sel["idx"][0, 0, :6]) == list(range(6))


# ----------------------------------------------------------------------------- attention

def _problem(seed, B=1, T=64 * 6 + 11, H=4, Hkv=2, d=16, S=64, dtype=torch.float64):
    g = _gen(seed)
    Q = torch.randn(B, T, H, d, dtype=dtype, generator=g)
    K = torch.randn(B, T, Hkv, d, dtype=dtype, generator=g)
    V = torch.randn(B, T, Hkv, d, dtype=dtype, generator=g)
    W = torch.randn(d, d, dtype=dtype, generator=g) / math.sqrt(d)
    return Q, K, V, W


def test_constant_value_chunks_closed_form():
    """With every value row of chunk c equal to v_c, each chunk output is v_c
    and O = sum_i softmax(score)_i v_{c_i}."""
    Q, K, _, W = _problem(12)
    B, T, H, d = Q.shape
    Hkv, S, k = K.shape[2], 64, 3
    vc = torch.randn(B, T // S + 1, Hkv, d, dtype=torch.float64, generator=_gen(13))
    V = vc.repeat_interleave(S, dim=1)[:, :T].contiguous()
    _, sel, O = _full(Q, K, V, W, S, k)
    G = H // Hkv
    for t in range(T):
        for j in range(Hkv):
            ke = sel["keff"][t, j]
            if ke == 0:
                assert np.all(O[0, t, j * G:(j + 1) * G] == 0.0)
                continue
            w = scipy.special.softmax(sel["score"][t, j, :ke])
            want = (w[:, None] * vc[0, sel["idx"][t, j, :ke], j].numpy()).sum(0)
            for h in range(j * G, (j + 1) * G):
                np.testing.assert_allclose(O[0, t, h], want, rtol=1e-12, atol=1e-12)


def test_unit_values_give_unit_output_and_zero_without_candidates():
    Q, K, V, W = _problem(14)
    V = torch.ones_like(V)
    _, sel, O = _full(Q, K, V, W, 64, 4)
    has = np.repeat(sel["keff"] > 0, Q.shape[2] // K.shape[2], axis=1)   # [T, H]
    np.testing.assert_allclose(O[0][has], 1.0, rtol=0, atol=1e-14)
    assert np.all(O[0][~has] == 0.0)
    assert np.all(~has[:64]) and np.all(has[64:])


def test_output_is_convex_combination_of_kept_values():
    Q, K, V, W = _problem(15)
    S = 64
    _, sel, O = _full(Q, K, V, W, S, 2)
    H, Hkv = Q.shape[2], K.shape[2]
    G = H // Hkv
    Vn = V[0].numpy()
    for t in range(S, Q.shape[1]):
        for j in range(Hkv):
            rows = np.concatenate([Vn[c * S:(c + 1) * S, j] for c in sel["idx"][t, j, :sel["keff"][t, j]]])
            lo, hi = rows.min(0), rows.max(0)
            for h in range(j * G, (j + 1) * G):
                assert np.all(O[0, t, h] >= lo - 1e-12) and np.all(O[0, t, h] <= hi + 1e-12)


def test_exhaustive_limit_equals_all_chunk_attention():
    """k >= #candidates keeps every candidate; compare with a loop over all
    candidate chunks that never sorts."""
    Q, K, V, W = _problem(16)
    B, T, H, d = Q.shape
    Hkv, S = K.shape[2], 64
    L, sel, O = _full(Q, K, V, W, S, k=T // S)
    G = H // Hkv
    Qn, Kn, Vn = Q[0].numpy(), K[0].numpy(), V[0].numpy()
    for t in range(0, T, 7):
        ncand = t // S
        for h in range(H):
            j = h // G
            if ncand == 0:
                assert np.all(O[0, t, h] == 0)
                continue
            s = np.array([sum(Qn[t, hh] @ L[0, j, c] for hh in range(j * G, (j + 1) * G))
                          for c in range(ncand)])
            w = scipy.special.softmax(s)
            acc = np.zeros(d)
            for c in range(ncand):
                Kc, Vc = Kn[c * S:(c + 1) * S, j], Vn[c * S:(c + 1) * S, j]
                acc += w[c] * (scipy.special.softmax(Kc @ Qn[t, h] / math.sqrt(d)) @ Vc)
            np.testing.assert_allclose(O[0, t, h], acc, rtol=1e-11, atol=1e-12)


def test_single_candidate_rows_match_sdpa():
    """Queries in chunk 1 have exactly one candidate (chunk 0): plain scaled
    dot-product attention over chunk 0 (torch SDPA in float64)."""
    Q, K, V, W = _problem(17)
    H, Hkv, d, S = Q.shape[2], K.shape[2], Q.shape[3], 64
    _, sel, O = _full(Q, K, V, W, S, 3)
    G = H // Hkv
    for h in range(H):
        j = h // G
        q = Q[0, S:2 * S, h].reshape(1, 1, S, d)
        kk = K[0, :S, j].reshape(1, 1, S, d)
        vv = V[0, :S, j].reshape(1, 1, S, d)
        ref = F.scaled_dot_product_attention(q, kk, vv)[0, 0].numpy()
        np.testing.assert_allclose(O[0, S:2 * S, h], ref, rtol=1e-12, atol=1e-13)
    assert np.all(sel["keff"][S:2 * S] == 1)


def test_attention_scale_closed_form_single_aligned_key():
    """Chunk 0 holds one key a*e0 and zeros; V has 1 at that key's row, dim 0.
    q = e0 at a chunk-1 position: O[0] = e^{a/sqrt(d)} / (e^{a/sqrt(d)} + S - 1)."""
    S, d, a = 64, 16, 3.0
    T = 2 * S
    Q = torch.zeros(1, T, 1, d, dtype=torch.float64)
    Q[0, :, 0, 0] = 1.0
    K = torch.zeros(1, T, 1, d, dtype=torch.float64)
    K[0, 0, 0, 0] = a
    V = torch.zeros(1, T, 1, d, dtype=torch.float64)
    V[0, 0, 0, 0] = 1.0
    _, _, O = _full(Q, K, V, torch.eye(d, dtype=torch.float64), S, 1)
    want = math.exp(a / math.sqrt(d)) / (math.exp(a / math.sqrt(d)) + S - 1)
    np.testing.assert_allclose(O[0, S:, 0, 0], want, rtol=1e-14)
    assert np.all(O[0, S:, 0, 1:] == 0)


def test_two_chunk_fusion_is_sigmoid_of_score_gap():
    """Chunk 0 keys all (1,0) and values 0; chunk 1 keys all (0,1) and values 1.
    With W_L = I the landmarks are (1,0) and (0,1), so q = (x, y) scores them
    x and y, and O = softmax weight of chunk 1 = 1 / (1 + e^{x - y})."""
    S, d, x, y = 4, 2, 0.7, -0.4
    T = 3 * S
    K = torch.zeros(1, T, 1, d, dtype=torch.float64)
    K[0, :S, 0, 0] = 1.0
    K[0, S:2 * S, 0, 1] = 1.0
    V = torch.zeros(1, T, 1, d, dtype=torch.float64)
    V[0, S:2 * S] = 1.0
    Q = torch.zeros(1, T, 1, d, dtype=torch.float64)
    Q[0, :, 0] = torch.tensor([x, y], dtype=torch.float64)
    _, sel, O = _full(Q, K, V, torch.eye(d, dtype=torch.float64), S, 2)
    want = 1.0 / (1.0 + math.exp(x - y))
    np.testing.assert_allclose(O[0, 2 * S:, 0], want, rtol=1e-14)
    assert list(sel["idx"][2 * S, 0]) == [0, 1]


def test_query_head_maps_to_kv_head_floor_h_over_G():
    """H=4, Hkv=2: heads 0,1 use kv head 0 and heads 2,3 use kv head 1, so the
    full problem equals two independent single-kv-head problems."""
    Q, K, V, W = _problem(18)
    _, _, O = _full(Q, K, V, W, 64, 3)
    for j in range(2):
        _, _, Oj = _full(Q[:, :, 2 * j:2 * j + 2].contiguous(), K[:, :, j:j + 1].contiguous(),
                         V[:, :, j:j + 1].contiguous(), W, 64, 3)
        np.testing.assert_array_equal(O[:, :, 2 * j:2 * j + 2], Oj)


def test_sampled_rows_and_gathered_attend_agree_with_full_run():
    p_T, S = 64 * 8 + 5, 64
    Q, K, V, W = _problem(19, B=2, T=p_T, dtype=torch.float32)
    Q, K, V, W = (x.to(torch.bfloat16) for x in (Q, K, V, W))
    rows_b = np.array([0, 1, 1, 0, 1])
    rows_t = np.array([70, 130, 511, 516, 300])
    a = oracle.forward_rows(Q, K, V, W, S, 3, 0.0, 0, rows_b, rows_t)
    Qr = Q[torch.as_tensor(rows_b), torch.as_tensor(rows_t)]
    O2 = oracle.attend_gathered(Qr, rows_b, K, V, S, a["sel"])
    np.testing.assert_array_equal(a["O"], O2)
    L = oracle.landmarks_stored(K, W, S, "bf16")
    rb_all = np.repeat(np.arange(2), p_T)
    rt_all = np.tile(np.arange(p_T), 2)
    sel_all = oracle.select(Q.reshape(-1, Q.shape[2], Q.shape[3]), rb_all, rt_all, L, S, 3, 0.0, Q.shape[2])
    for i, (b, t) in enumerate(zip(rows_b, rows_t)):
        np.testing.assert_array_equal(a["sel"]["idx"][i], sel_all["idx"][b * p_T + t])
