"""Backward pass on the GPU (hsa_backward) against the oracle's backward.

HSA summary page, Implementation: the kept chunks' retrieval scores weight
their outputs, so the gradients flow through the in-chunk attention, the fusion
softmax, the group scores and the landmarks (mean-pooled keys times W_L); the
chunk choice itself is held fixed.  The forward runs on the GPU, and the oracle
differentiates the same selection on the same stored inputs, scoring on the
landmarks the library stored (their rounding counts as the identity on both
sides).

Tolerance, per gradient tensor, as max |gpu - oracle| / max |oracle|:
  * CUDA-core path (fp32, and bf16 with HSA_FLAG_SIMT or d = 64): 1e-4.  Both
    sides read the same stored values; the GPU accumulates in fp32 (its fusion
    weights come from the forward's fp32 scores, relative error ~1e-6; every
    sum has fp32 rounding ~6e-8 relative to its terms, a few thousand terms at
    most), measured 2e-7 .. 1e-6.
  * tensor-core path (bf16, d = 128, S 64 / 128): 1e-2.  dZ and w P are rounded
    once to bf16 (relative error <= 2^-9 = 1.95e-3) before the dQ, dK and dV
    contractions, as P is in the forward; every term of those sums carries
    one such factor, and the measured worst is 2.6e-3 of the tensor's scale.
    1e-2 (about 5 x 2^-9) bounds that with margin; e, the score path and dW_L
    stay fp32 (measured ~1e-6).
A dropped term or a wrong factor moves a gradient by O(1) of its scale (the
oracle pins show that), so both bounds still catch one.
"""
import numpy as np
import pytest
import torch

import landmark_guided_chunk_b200 as hsa
import oracle
from landmark_guided_chunk_b200.inputs import Problem, make_inputs, make_output_grad, workload

pytestmark = pytest.mark.gpu

TOL = 1e-4
TOL_TC = 1e-2


def _tc_path(p: Problem, force_simt=False) -> bool:
    return p.dtype == "bf16" and p.d == 128 and p.S in (64, 128) and not force_simt


def _close(name, got, ref, tol=TOL):
    got = got.double().cpu().numpy() if isinstance(got, torch.Tensor) else got
    scale = float(np.abs(ref).max()) if ref.size else 0.0
    err = float(np.abs(got - ref).max()) if ref.size else 0.0
    assert err <= tol * max(scale, 1e-30), f"{name}: max error {err:.3g} vs scale {scale:.3g} (tol {tol:g})"
    return err / max(scale, 1e-30)


def _run(p: Problem, seed: int, kv_len=None, W_random=True, force_simt=False):
    inp = make_inputs(p, seed=seed, device="cuda")
    Q, K, V, W = inp["Q"], inp["K"], inp["V"], inp["W_L"]
    if W_random and p.is_decode:
        g = torch.Generator(device="cuda").manual_seed(seed + 1)
        W = (torch.randn(p.d, p.d, generator=g, device="cuda") / p.d ** 0.5).to(K.dtype)
    dO = make_output_grad(p, seed=seed + 2, device="cuda")
    n = K.shape[1] if kv_len is None else kv_len
    O, L, idx, sc, ke = hsa.forward(Q, K, V, W, p.S, p.k, p.tau, q_pos0=p.q_pos0, return_selection=True,
                                    kv_len=kv_len)
    dQ, dK, dV, dW = hsa.backward(Q, K, V, W, L, idx, sc, ke, dO, p.S, p.k, p.tau, q_pos0=p.q_pos0, kv_len=kv_len,
                                  force_simt=force_simt)
    torch.cuda.synchronize()
    return dict(Q=Q, K=K, V=V, W=W, dO=dO, L=L, idx=idx, sc=sc, ke=ke, dQ=dQ, dK=dK, dV=dV, dW=dW, n=n)


def _oracle_rows(r, p, rows_b, rows_t):
    """Oracle backward over the listed query rows (all rows -> full dK, dV, dW)."""
    n, C = r["n"], r["n"] // p.S
    rb = torch.as_tensor(rows_b)
    rt = torch.as_tensor(rows_t)
    Qr = r["Q"][rb, rt].cpu()
    dOr = r["dO"][rb, rt].cpu().double().numpy()
    sel = {"idx": r["idx"][rb, rt].cpu().numpy(), "keff": r["ke"][rb, rt].cpu().numpy()}
    K = r["K"][:, :n].cpu()
    V = r["V"][:, :n].cpu()
    L = r["L"][:, :, :C].double().cpu().numpy()
    return oracle.backward(Qr, np.asarray(rows_b), K, V, r["W"].cpu(), L, p.S, sel, dOr)


def _full_check(p, r, tol):
    B, Tq = p.B, p.Tq
    rows_b = np.repeat(np.arange(B), Tq)
    rows_t = np.tile(np.arange(Tq), B)
    g = _oracle_rows(r, p, rows_b, rows_t)
    n = r["n"]
    errs = {"dQ": _close("dQ", r["dQ"].reshape(B * Tq, p.H, p.d), g["dQ"], tol),
            "dK": _close("dK", r["dK"][:, :n], g["dK"], tol),
            "dV": _close("dV", r["dV"][:, :n], g["dV"], tol),
            "dW": _close("dW", r["dW"], g["dW"], tol)}
    # tokens past the complete chunks (trailing partial chunk, spare capacity) get exactly 0
    c_end = (n // p.S) * p.S
    assert torch.all(r["dK"][:, c_end:] == 0) and torch.all(r["dV"][:, c_end:] == 0)
    return errs


CASES = {
    "tiny_f32": (workload("tiny_f32"), None, False),
    "bf16_gqa4_S64": (Problem(B=2, Tq=64 * 12 + 37, Tkv=64 * 12 + 37, H=8, Hkv=2, d=128, S=64, k=4, dtype="bf16"),
                      None, False),
    "bf16_gqa4_S64_simt": (Problem(B=2, Tq=64 * 12 + 37, Tkv=64 * 12 + 37, H=8, Hkv=2, d=128, S=64, k=4,
                                   dtype="bf16"), None, True),
    "bf16_router_S128_d64": (Problem(B=1, Tq=128 * 9 + 5, Tkv=128 * 9 + 5, H=4, Hkv=2, d=64, S=128, k=3, tau=0.05,
                                     dtype="bf16"), None, False),
    "bf16_router_S128_d128": (Problem(B=1, Tq=128 * 9 + 5, Tkv=128 * 9 + 5, H=8, Hkv=2, d=128, S=128, k=3,
                                      tau=0.05, dtype="bf16"), None, False),
    "bf16_G1_S64": (Problem(B=1, Tq=64 * 10 + 3, Tkv=64 * 10 + 3, H=2, Hkv=2, d=128, S=64, k=6, dtype="bf16"),
                    None, False),
    "bf16_G16_S128": (Problem(B=1, Tq=128 * 6 + 9, Tkv=128 * 6 + 9, H=16, Hkv=1, d=128, S=128, k=2, dtype="bf16"),
                      None, False),
    "f32_G16_S32_capacity": (Problem(B=1, Tq=32 * 20 + 7, Tkv=32 * 20 + 7 + 45, H=16, Hkv=1, d=64, S=32, k=5,
                                     dtype="f32"), 32 * 20 + 7, False),
    "bf16_capacity_S64": (Problem(B=2, Tq=64 * 9 + 20, Tkv=64 * 9 + 20 + 100, H=8, Hkv=2, d=128, S=64, k=3,
                                  dtype="bf16"), 64 * 9 + 20, False),
    "bf16_decode_rows": (Problem(B=3, Tq=1, Tkv=64 * 50 + 9, H=8, Hkv=2, d=128, S=64, k=8, q_pos0=64 * 50 + 9,
                                 dtype="bf16"), None, False),
    # the CUDA-core kernel's other shapes: fp32 at S = 128, d = 128; bf16 at S = 32 (no tensor-core
    # path) and at S = 128, d = 128 forced onto the CUDA cores
    "f32_S128_d128": (Problem(B=1, Tq=128 * 5 + 17, Tkv=128 * 5 + 17, H=4, Hkv=2, d=128, S=128, k=2, dtype="f32"),
                      None, False),
    "bf16_S32_d128": (Problem(B=1, Tq=32 * 20 + 7, Tkv=32 * 20 + 7, H=8, Hkv=2, d=128, S=32, k=4, dtype="bf16"),
                      None, False),
    "bf16_S128_d128_simt": (Problem(B=1, Tq=128 * 6 + 3, Tkv=128 * 6 + 3, H=4, Hkv=2, d=128, S=128, k=3,
                                    dtype="bf16"), None, True),
    # G = 16 over 73 chunks: tiles of 8 pairs, many tiles per chunk
    "bf16_G16_long": (Problem(B=1, Tq=4096 + 600, Tkv=4096 + 600, H=32, Hkv=2, d=128, S=64, k=2, dtype="bf16"),
                      None, False),
}


@pytest.mark.parametrize("case", list(CASES))
def test_backward_matches_oracle(case):
    p, kv_len, simt = CASES[case]
    r = _run(p, seed=40, kv_len=kv_len, force_simt=simt)
    if kv_len is not None:
        p = p.with_(Tkv=kv_len)
    if p.tau > 0:
        assert int((r["ke"] > p.k).sum()) > 0, "the router case must double some rows"
    _full_check(p, r, TOL_TC if _tc_path(p, simt) else TOL)


def test_backward_without_candidates_is_zero():
    p = Problem(B=2, Tq=50, Tkv=50, H=4, Hkv=2, d=64, S=64, k=2, dtype="bf16")   # no complete chunk
    r = _run(p, seed=3)
    for name in ("dQ", "dK", "dV", "dW"):
        assert torch.all(r[name] == 0), name


def test_backward_empty_batch():
    """B = 0: nothing to differentiate; dW_L (always allocated) comes back zeroed."""
    p = Problem(B=0, Tq=70, Tkv=70, H=4, Hkv=2, d=64, S=32, k=2, dtype="bf16")
    dt = torch.bfloat16
    Q = torch.empty(0, 70, 4, 64, dtype=dt, device="cuda")
    K = torch.empty(0, 70, 2, 64, dtype=dt, device="cuda")
    V = torch.empty_like(K)
    W = torch.randn(64, 64, device="cuda").to(dt)
    L = torch.empty(0, 2, 2, 64, dtype=dt, device="cuda")
    idx = torch.empty(0, 70, 2, 2, dtype=torch.int32, device="cuda")
    sc = torch.empty(0, 70, 2, 2, dtype=torch.float32, device="cuda")
    ke = torch.empty(0, 70, 2, dtype=torch.int32, device="cuda")
    dW = torch.full((64, 64), 7.0, device="cuda")
    out = (torch.empty(0, 70, 4, 64, device="cuda"), torch.empty(0, 70, 2, 64, device="cuda"),
           torch.empty(0, 70, 2, 64, device="cuda"), dW)
    hsa.backward(Q, K, V, W, L, idx, sc, ke, torch.empty_like(Q), p.S, p.k, out=out)
    torch.cuda.synchronize()
    assert torch.all(dW == 0)


def test_backward_prefill_full_size_sampled_rows():
    """The 65536-token bf16 prefill (H32 Hkv8 d128 S64 k16): dQ of sampled rows
    against the oracle on those rows alone (a row's dQ depends only on that row),
    and, for the whole problem, the sums the method fixes at any size: sum_t dV
    equals the summed dO of the rows that keep any chunk, and sum_t dK = 0
    (each chunk's keys sum to its landmark gradient times W_L^T, and the
    landmark gradients of a (batch, kv head) sum to zero)."""
    p = workload("prefill_bf16")
    r = _run(p, seed=7)
    rng = np.random.default_rng(8)
    rows_t = np.sort(np.concatenate([rng.choice(p.Tq, 24, replace=False), [p.S, p.Tq - 1]]))
    rows_b = np.zeros_like(rows_t)
    g = _oracle_rows(r, p, rows_b, rows_t)
    _close("dQ (sampled rows)", r["dQ"][0, torch.as_tensor(rows_t)], g["dQ"], TOL_TC)
    dO = r["dO"].double()
    kept = (r["ke"] > 0).double()                                       # [B,Tq,Hkv]
    dOg = dO.view(p.B, p.Tq, p.Hkv, p.G, p.d).sum(3)                     # [B,Tq,Hkv,d]
    expect = (dOg * kept.unsqueeze(-1)).sum(1)                           # [B,Hkv,d]
    got = r["dV"].double().sum(1)
    # w P is rounded to bf16 before the dV contraction: each kept row's share is off by at most
    # 2^-9 of its |dO| (its weights and probabilities sum to 1)
    bound = 2.0 ** -9 * (dOg.abs() * kept.unsqueeze(-1)).sum(1) + 1e-5 * float(r["dV"].double().abs().sum(1).max())
    assert bool(((got - expect).abs() <= bound).all())
    # dZ is rounded to bf16 as well: the per-chunk sums of its entries are zero only up to those
    # independent roundings, whose total grows like the square root of their count
    kscale = float(r["dK"].double().abs().sum(1).max())
    assert float(r["dK"].double().sum(1).abs().max()) <= 2.0 ** -9 * kscale
