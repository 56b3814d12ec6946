"""Parity of the two selection variants (CUDA path through the C ABI) against
the oracle.

Landmark refiner (hsa_landmarks_refined): the refined landmarks element-wise,
then the whole forward on them (selection on the stored landmarks, output).
Its tolerance: one bf16 ulp of the stored value plus 2^-13 * max|L| for the
fp32 arithmetic of the chain (four d x d products, three S-long sums, a
softmax whose logits carry the products' rounding: each stage is bounded by
the fp32 accumulation bound 2^-17 of the plain landmark, and eight of them
add up to 2^-14; the factor 2 covers the softmax's sensitivity to its logits).

Quest scoring (HSA_FLAG_QUEST): the summaries must equal the oracle's exactly
(they are stored key values); the selection is checked against the oracle's
Quest selection on every row of small problems (all select paths: the tcgen05
kernel at d' = 128 and 256, the streaming and CUDA-core scans for decode, the
CUDA-core rows kernel for fp32 and under HSA_FLAG_SIMT), and the output
against the oracle's attention on that selection.  The decode-loop append
computes the summary of the chunk it completes."""
import math

import numpy as np
import pytest
import torch

import landmark_guided_chunk_b200 as hsa
import oracle
from landmark_guided_chunk_b200.inputs import Problem, make_inputs, torch_dtype
from tests import parity

pytestmark = pytest.mark.gpu


def _refine_weights(d, dtype, seed):
    g = torch.Generator(device="cuda").manual_seed(seed)
    ws = [(torch.randn(d, d, device="cuda", generator=g) / math.sqrt(d)) for _ in range(3)]
    ws[0] = ws[0] * 6.0   # W_q: a peaked in-chunk attention, so the softmax matters
    return [w.to(dtype) for w in ws]


def _all_rows(p):
    return np.repeat(np.arange(p.B), p.Tq), np.tile(np.arange(p.Tq), p.B)


def _check_rows(p, inp, L_gpu, sel_orc, idx, score, keff, O, rows):
    rb, rt = rows
    tb, tt = torch.as_tensor(rb, device="cuda"), torch.as_tensor(rt, device="cuda")
    ncand = np.minimum((rt + p.q_pos0) // p.S, p.C)
    g_idx, g_sc, g_ke = idx[tb, tt].cpu().numpy(), score[tb, tt].cpu().numpy(), keff[tb, tt].cpu().numpy()
    sel = parity.check_selection(g_idx, g_sc, g_ke, sel_orc, ncand, p.k, p.tau)
    Qr = inp["Q"][tb, tt].cpu()
    O_exp = parity.expected_output(Qr, rb, inp["K"], inp["V"], p.S, sel_orc, g_idx, g_ke, sel["tie_rows"])
    err = parity.check_output(O[tb, tt], O_exp, inp["Q"].dtype)
    return sel, err


REFINE_CASES = [
    Problem(B=2, Tq=64 * 20 + 37, Tkv=64 * 20 + 37, H=8, Hkv=2, d=128, S=64, k=8, dtype="bf16", name="bf16_d128"),
    Problem(B=1, Tq=32 * 40 + 5, Tkv=32 * 40 + 5, H=4, Hkv=4, d=64, S=32, k=5, tau=0.05, dtype="bf16",
            name="bf16_d64_s32_router"),
    Problem(B=1, Tq=128 * 12 + 100, Tkv=128 * 12 + 100, H=4, Hkv=2, d=64, S=128, k=4, dtype="f32",
            name="f32_s128"),
]


@pytest.mark.parametrize("p", REFINE_CASES, ids=lambda p: p.name)
def test_refined_landmarks_and_forward(p):
    torch.cuda.set_device(0)
    inp = make_inputs(p, seed=21, device="cuda")
    Q, K, V, W = inp["Q"], inp["K"], inp["V"], inp["W_L"]
    Wq, Wk, Wv = _refine_weights(p.d, Q.dtype, 22)
    O, L, idx, score, keff = hsa.forward(Q, K, V, W, p.S, p.k, p.tau, p.q_pos0, return_selection=True,
                                         refine=(Wq, Wk, Wv))
    torch.cuda.synchronize()
    L_orc = oracle.landmarks_refined(K.cpu(), W.cpu(), Wq.cpu(), Wk.cpu(), Wv.cpu(), p.S)
    L_orc_st = oracle.round_to(p.dtype, L_orc)
    g = L.double().cpu().numpy()
    atol = 2.0 ** -13 * float(np.abs(L_orc).max())
    if p.dtype == "bf16":
        bad = np.abs(g - L_orc_st) > parity.bf16_ulp(L_orc_st) * 1.0000001 + atol
    else:
        bad = np.abs(g - L_orc_st) > atol
    assert not bad.any(), f"{bad.sum()} refined landmark values off (worst {np.abs(g - L_orc_st).max():.3e})"
    # the refinement is not a no-op on these inputs
    L_plain = oracle.landmarks(K.cpu(), W.cpu(), p.S)
    assert np.abs(L_orc - L_plain).max() > 0.1 * np.abs(L_plain).max()
    rows = _all_rows(p)
    rb, rt = rows
    sel_orc = oracle.select(Q.cpu().reshape(p.B * p.Tq, p.H, p.d), rb, rt + p.q_pos0, g, p.S, p.k, p.tau, p.H,
                            want_all=True)
    _check_rows(p, inp, L, sel_orc, idx, score, keff, O, rows)


QUEST_CASES = [
    # tcgen05 scoring on the transformed problem: d' = 256 (64-chunk slices) and d' = 128
    Problem(B=2, Tq=64 * 24 + 29, Tkv=64 * 24 + 29, H=8, Hkv=2, d=128, S=64, k=8, dtype="bf16", name="bf16_d128_g4"),
    Problem(B=1, Tq=128 * 20 + 5, Tkv=128 * 20 + 5, H=8, Hkv=2, d=128, S=128, k=8, tau=0.02, dtype="bf16",
            name="bf16_d128_router"),
    Problem(B=1, Tq=32 * 60 + 9, Tkv=32 * 60 + 9, H=4, Hkv=4, d=64, S=32, k=6, dtype="bf16", name="bf16_d64_g1"),
    # CUDA-core rows kernel
    Problem(B=1, Tq=64 * 16 + 3, Tkv=64 * 16 + 3, H=6, Hkv=2, d=64, S=64, k=4, tau=0.1, dtype="f32",
            name="f32_router"),
    # decode: streaming scan (d' = 128) and the CUDA-core split scan (d' = 256)
    Problem(B=3, Tq=1, Tkv=64 * 2500 + 17, H=8, Hkv=2, d=64, S=64, k=8, q_pos0=64 * 2500 + 17, dtype="bf16",
            name="decode_d64"),
    Problem(B=2, Tq=1, Tkv=64 * 2200 + 3, H=8, Hkv=2, d=128, S=64, k=16, q_pos0=64 * 2200 + 3, dtype="bf16",
            name="decode_d128"),
]


def _quest_case(p, force_simt=False, seed=31):
    torch.cuda.set_device(0)
    inp = make_inputs(p, seed=seed, device="cuda")
    Q, K, V = inp["Q"], inp["K"], inp["V"]
    O, Lq, idx, score, keff = hsa.forward(Q, K, V, None, p.S, p.k, p.tau, p.q_pos0, return_selection=True,
                                          quest=True, force_simt=force_simt)
    torch.cuda.synchronize()
    Lq_orc = oracle.quest_summaries(K.cpu(), p.S)
    assert np.array_equal(Lq.double().cpu().numpy(), Lq_orc)
    rows = _all_rows(p)
    rb, rt = rows
    sel_orc = oracle.select_quest(Q.cpu().reshape(p.B * p.Tq, p.H, p.d), rb, rt + p.q_pos0, Lq_orc, p.S, p.k,
                                  p.tau, p.H, want_all=True)
    return _check_rows(p, inp, Lq, sel_orc, idx, score, keff, O, rows)


@pytest.mark.parametrize("p", QUEST_CASES, ids=lambda p: p.name)
def test_quest_selection_and_forward(p):
    prob = hsa.make_problem(p.B, p.Tq, p.Tkv, p.H, p.Hkv, p.d, p.S, p.k, p.q_pos0, p.tau, torch_dtype(p.dtype),
                            hsa._native.HSA_FLAG_QUEST)
    pl = hsa.plan(prob)
    if p.Tq >= 64 and p.dtype == "bf16":
        assert pl["select"][0] == "tensor"
    sel, err = _quest_case(p)
    assert sel["ties"] <= max(2, sel["exact"] // 200)


@pytest.mark.parametrize("p", [QUEST_CASES[0], QUEST_CASES[4]], ids=lambda p: p.name)
def test_quest_cuda_core_path(p):
    _quest_case(p, force_simt=True)


def test_quest_decode_append_writes_the_completed_chunk_summary():
    torch.cuda.set_device(0)
    B, Hkv, d, S, Tcap = 2, 2, 64, 32, 32 * 6
    T0 = 32 * 3 + 28
    p = Problem(B=B, Tq=T0, Tkv=Tcap, H=Hkv, Hkv=Hkv, d=d, S=S, k=2, dtype="bf16")
    inp = make_inputs(p, seed=41, device="cuda")
    K, V = inp["K"], inp["V"]
    Kc, Vc = K.clone(), V.clone()
    Kc[:, T0:] = 0
    Vc[:, T0:] = 0
    Lq = hsa.quest_summaries(Kc, S, kv_len=T0)
    for t in range(T0, T0 + 2 * S):
        if t >= Tcap:
            break
        hsa.decode_append(Kc, Vc, K[:, t].contiguous(), V[:, t].contiguous(), t, S, L=Lq, quest=True)
    torch.cuda.synchronize()
    n_done = min(Tcap, T0 + 2 * S) // S
    ref = oracle.quest_summaries(K[:, :n_done * S].cpu(), S)
    assert np.array_equal(Lq[:, :, :n_done].double().cpu().numpy(), ref)
