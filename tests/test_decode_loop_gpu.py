"""Decode loop on a cache that grows in place (hsa_decode_append), and the
K/V / landmark capacity (hsa_problem_t.kv_cap) it relies on.

HSA summary page, Implementation: every chunk has a landmark, so the decode
step that completes a chunk must produce that chunk's landmark before any later
query can retrieve it.  Each step appends one token per sequence into buffers
sized for the whole generation, and the forward of the next query reads them
with Tkv = the tokens cached so far.

Two references:
  * the oracle, on the step's rows (selection and output, as in the other
    parity tests), and
  * the same call on tightly packed copies of the cache: the kernels'
    arithmetic does not depend on the buffers' strides, so landmarks, indices
    and scores must be bit-identical to the tight call's, and O equal up to the
    order of its fp32 atomic additions.  This pins the capacity strides in each
    kernel path (tensor-core prefill, streaming decode scan and gather, CUDA-core).
"""
import numpy as np
import pytest
import torch

import landmark_guided_chunk_b200 as hsa
import oracle
from landmark_guided_chunk_b200.inputs import Problem, make_inputs
from tests import parity

pytestmark = pytest.mark.gpu


def _tight(x, n):
    return x[:, :n].contiguous()


def _same_output(O, Ot):
    """O of two calls that differ only in buffer strides.  The attention kernels add a
    row's chunk outputs with fp32 atomic reductions, whose order varies from call to
    call: the fp32 sums may differ by a few fp32 ulps of the terms' size (at most kmax
    terms, each below max|V|), which a bf16 O shows as one bf16 ulp, or as that
    absolute fp32 noise where the sum cancels to near zero.  Returns "" or a report."""
    a, b = O.double(), Ot.double()
    diff = (a - b).abs()
    floor = 1e-5 * max(float(a.abs().max()), float(b.abs().max()), 1e-30)
    if O.dtype == torch.bfloat16:
        ulp = torch.tensor(parity.bf16_ulp(np.maximum(a.abs().cpu().numpy(), b.abs().cpu().numpy())),
                           device=O.device)
        bad = diff > ulp * 1.0000001 + floor
    else:
        bad = diff > floor
    if not bool(bad.any()):
        return ""
    i = int(torch.argmax(diff))
    return f"{int(bad.sum())} of {diff.numel()} differ; max {float(diff.max()):.3g} at flat index {i}"


def _rand_W(d, dtype, seed):
    """A random W_L (decode-shaped inputs default to the identity), so that the
    incremental landmarks exercise the projection."""
    g = torch.Generator(device="cuda").manual_seed(seed)
    return (torch.randn(d, d, generator=g, device="cuda") / d ** 0.5).to(dtype)


def _oracle_step(Q, Kt, Vt, Lt, idx, sc, ke, S, k, tau, n):
    """Oracle check of one decode step (query at position n, B rows)."""
    B, _, H, d = Q.shape
    Hkv = Kt.shape[2]
    C = n // S
    rb, rt = np.arange(B), np.zeros(B, dtype=np.int64)
    Qr = Q[:, 0].cpu()
    orc = oracle.select(Qr, rb, rt + n, Lt.double().cpu().numpy(), S, k, tau, H, want_all=True)
    ncand = np.minimum((rt + n) // S, C)
    g_idx, g_ke = idx[:, 0].cpu().numpy(), ke[:, 0].cpu().numpy()
    sel = parity.check_selection(g_idx, sc[:, 0].cpu().numpy(), g_ke, orc, ncand, k, tau)
    O_exp = parity.expected_output(Qr, rb, Kt, Vt, S, orc, g_idx, g_ke, sel["tie_rows"])
    return O_exp


@pytest.mark.parametrize("dtype,H,Hkv,d,S,k,tau", [
    ("bf16", 8, 2, 128, 64, 4, 0.0),
    ("f32", 4, 4, 64, 32, 3, 0.05),
    ("bf16", 4, 1, 64, 128, 2, 0.0),
])
def test_decode_loop_matches_oracle_and_tight_cache(dtype, H, Hkv, d, S, k, tau):
    B, cap = 2, S * 12
    T0 = S * 10 - 14            # 14 steps before chunk 9 completes
    steps = S + 20              # so the loop completes two chunks
    full = Problem(B=B, Tq=steps, Tkv=cap, H=H, Hkv=Hkv, d=d, S=S, k=k, tau=tau, dtype=dtype)
    inp = make_inputs(full, seed=21, device="cuda")
    Qs, Kall, Vall = inp["Q"], inp["K"], inp["V"]
    W = _rand_W(d, Kall.dtype, 22)
    K, V = torch.zeros_like(Kall), torch.zeros_like(Vall)
    K[:, :T0] = Kall[:, :T0]
    V[:, :T0] = Vall[:, :T0]
    L = hsa.landmarks(K, W, S, kv_len=T0)
    assert L.shape == (B, Hkv, cap // S, d)
    completed = 0
    for s in range(steps):
        kv = T0 + s
        done = hsa.decode_append(K, V, Kall[:, kv].contiguous(), Vall[:, kv].contiguous(), kv, S, W, L)
        assert done == ((kv + 1) % S == 0)
        completed += int(done)
        n = kv + 1
        Q = Qs[:, s:s + 1].contiguous()
        O, _, idx, sc, ke = hsa.forward(Q, K, V, None, S, k, tau, q_pos0=n, L=L, landmarks_ready=True,
                                        return_selection=True, kv_len=n)
        Kt, Vt = _tight(Kall, n), _tight(Vall, n)
        Lt = hsa.landmarks(Kt, W, S)
        Ot, _, idxt, sct, ket = hsa.forward(Q, Kt, Vt, None, S, k, tau, q_pos0=n, L=Lt, landmarks_ready=True,
                                            return_selection=True)
        C = n // S
        assert torch.equal(L[:, :, :C], Lt), f"step {s}: incremental landmarks differ from a full recompute"
        assert torch.equal(idx, idxt) and torch.equal(ke, ket) and torch.equal(sc, sct), f"step {s}: selection"
        rep = _same_output(O, Ot)
        assert not rep, f"step {s}: output differs from the tight-cache call: {rep}"
        if s % 16 == 0 or n % S in (0, 1) or s == steps - 1:
            O_exp = _oracle_step(Q, Kt, Vt, Lt, idx, sc, ke, S, k, tau, n)
            parity.check_output(O[:, 0], O_exp, Q.dtype)
    assert completed == 2
    n = T0 + steps
    assert torch.equal(K[:, :n], Kall[:, :n]) and torch.equal(V[:, :n], Vall[:, :n])
    assert torch.all(K[:, n:] == 0) and torch.all(V[:, n:] == 0)
    parity.check_landmarks(L[:, :, :n // S], oracle.landmarks_stored(Kall[:, :n].cpu(), W.cpu(), S, dtype))


def test_decode_with_capacity_on_the_streaming_path():
    """One decode step at C >= 2048 (the streaming scan and the chunk gather) on
    buffers with room to spare: identical to the tight call, and to the oracle."""
    p = Problem(B=1, Tq=1, Tkv=64 * 2100 + 5, H=32, Hkv=8, d=128, S=64, k=16, q_pos0=64 * 2100 + 5,
                dtype="bf16")
    cap = p.Tkv + 300
    inp = make_inputs(p.with_(Tkv=cap), seed=5, device="cuda")
    Q, K, V = inp["Q"], inp["K"], inp["V"]
    W = _rand_W(p.d, K.dtype, 6)
    L = hsa.landmarks(K, W, p.S, kv_len=p.Tkv)
    prob = hsa.make_problem(p.B, 1, p.Tkv, p.H, p.Hkv, p.d, p.S, p.k, p.Tkv, 0.0, torch.bfloat16,
                            hsa._native.HSA_FLAG_LANDMARKS_READY, cap)
    assert hsa.plan(prob)["attend"] == ("mma_split", 1)
    O, _, idx, sc, ke = hsa.forward(Q, K, V, None, p.S, p.k, q_pos0=p.Tkv, L=L, landmarks_ready=True,
                                    return_selection=True, kv_len=p.Tkv)
    Kt, Vt = _tight(K, p.Tkv), _tight(V, p.Tkv)
    Lt = hsa.landmarks(Kt, W, p.S)
    Ot, _, idxt, sct, ket = hsa.forward(Q, Kt, Vt, None, p.S, p.k, q_pos0=p.Tkv, L=Lt, landmarks_ready=True,
                                        return_selection=True)
    assert torch.equal(L[:, :, :p.C], Lt)
    assert torch.equal(idx, idxt) and torch.equal(ke, ket) and torch.equal(sc, sct)
    assert not _same_output(O, Ot), _same_output(O, Ot)
    O_exp = _oracle_step(Q, Kt, Vt, Lt, idx, sc, ke, p.S, p.k, 0.0, p.Tkv)
    parity.check_output(O[:, 0], O_exp, Q.dtype)


@pytest.mark.parametrize("S,k,tau", [(64, 8, 0.0), (128, 4, 0.05)])
def test_prefill_with_capacity_matches_tight(S, k, tau):
    """Prefill over the first Tkv tokens of larger buffers (tensor-core scoring and
    chunk-major attention): identical to the tight call."""
    T = S * 30 + 17
    cap = T + 2 * S + 9
    p = Problem(B=2, Tq=T, Tkv=cap, H=8, Hkv=2, d=128, S=S, k=k, tau=tau, dtype="bf16")
    inp = make_inputs(p, seed=9, device="cuda")
    Qf, K, V = inp["Q"], inp["K"], inp["V"]
    W = _rand_W(p.d, K.dtype, 10)
    Q = Qf[:, :T].contiguous()
    O, L, idx, sc, ke = hsa.forward(Q, K, V, W, S, k, tau, return_selection=True, kv_len=T)
    assert L.shape[2] == cap // S
    Kt, Vt = _tight(K, T), _tight(V, T)
    Ot, Lt, idxt, sct, ket = hsa.forward(Q, Kt, Vt, W, S, k, tau, return_selection=True)
    prob = hsa.make_problem(p.B, T, T, p.H, p.Hkv, p.d, S, k, 0, tau, torch.bfloat16, 0, cap)
    assert hsa.plan(prob)["attend"][0] == "tensor" and hsa.plan(prob)["select"][0] == "tensor"
    assert torch.equal(L[:, :, :T // S], Lt)
    assert torch.equal(idx, idxt) and torch.equal(ke, ket) and torch.equal(sc, sct)
    rep = _same_output(O, Ot)
    assert not rep, rep
