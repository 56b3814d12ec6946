"""Backward pass on the GPU (hsa_backward) against the oracle's backward.

HSA summary page, Implementation: the kept chunks' retrieval scores weight
their outputs, so the gradients flow through the in-chunk attention, the fusion
softmax, the group scores and the landmarks (mean-pooled keys times W_L); the
chunk choice itself is held fixed.  The forward runs on the GPU, and the oracle
differentiates the same selection on the same stored inputs, scoring on the
landmarks the library stored (their rounding counts as the identity on both
sides).

Tolerance, per gradient tensor: max |gpu - oracle| <= 1e-4 * max |oracle|.  Both
sides read the same stored values; the GPU accumulates in fp32 (its fusion
weights come from the forward's fp32 scores, relative error ~1e-6; every sum
it forms has fp32 rounding ~6e-8 relative to its terms' magnitude, and the
largest sums have a few thousand terms), so 1e-4 of the tensor's scale covers
the accumulated rounding with a wide margin while a dropped term or wrong
factor (the oracle pins show those move a gradient by O(1) of its scale) fails.
"""
import numpy as np
import pytest
import torch

import landmark_guided_chunk_b200 as hsa
import oracle
from landmark_guided_chunk_b200.inputs import Problem, make_inputs, make_output_grad, workload

pytestmark = pytest.mark.gpu

TOL = 1e-4


def _close(name, got, ref):
    got = got.double().cpu().numpy() if isinstance(got, torch.Tensor) else got
    scale = float(np.abs(ref).max()) if ref.size else 0.0
    err = float(np.abs(got - ref).max()) if ref.size else 0.0
    assert err <= TOL * max(scale, 1e-30), f"{name}: max error {err:.3g} vs scale {scale:.3g}"
    return err / max(scale, 1e-30)


def _run(p: Problem, seed: int, kv_len=None, W_random=True):
    inp = make_inputs(p, seed=seed, device="cuda")
    Q, K, V, W = inp["Q"], inp["K"], inp["V"], inp["W_L"]
    if W_random and p.is_decode:
        g = torch.Generator(device="cuda").manual_seed(seed + 1)
        W = (torch.randn(p.d, p.d, generator=g, device="cuda") / p.d ** 0.5).to(K.dtype)
    dO = make_output_grad(p, seed=seed + 2, device="cuda")
    n = K.shape[1] if kv_len is None else kv_len
    O, L, idx, sc, ke = hsa.forward(Q, K, V, W, p.S, p.k, p.tau, q_pos0=p.q_pos0, return_selection=True,
                                    kv_len=kv_len)
    dQ, dK, dV, dW = hsa.backward(Q, K, V, W, L, idx, sc, ke, dO, p.S, p.k, p.tau, q_pos0=p.q_pos0, kv_len=kv_len)
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


def _full_check(p, r):
    B, Tq = p.B, p.Tq
    rows_b = np.repeat(np.arange(B), Tq)
    rows_t = np.tile(np.arange(Tq), B)
    g = _oracle_rows(r, p, rows_b, rows_t)
    n = r["n"]
    errs = {"dQ": _close("dQ", r["dQ"].reshape(B * Tq, p.H, p.d), g["dQ"]),
            "dK": _close("dK", r["dK"][:, :n], g["dK"]),
            "dV": _close("dV", r["dV"][:, :n], g["dV"]),
            "dW": _close("dW", r["dW"], g["dW"])}
    # tokens past the complete chunks (trailing partial chunk, spare capacity) get exactly 0
    c_end = (n // p.S) * p.S
    assert torch.all(r["dK"][:, c_end:] == 0) and torch.all(r["dV"][:, c_end:] == 0)
    return errs


@pytest.mark.parametrize("case", [
    "tiny_f32",
    "bf16_gqa4_S64",
    "bf16_router_S128",
    "f32_G16_S32_capacity",
    "bf16_decode_rows",
])
def test_backward_matches_oracle(case):
    kv_len = None
    if case == "tiny_f32":
        p = workload("tiny_f32")
    elif case == "bf16_gqa4_S64":
        p = Problem(B=2, Tq=64 * 12 + 37, Tkv=64 * 12 + 37, H=8, Hkv=2, d=128, S=64, k=4, dtype="bf16")
    elif case == "bf16_router_S128":
        p = Problem(B=1, Tq=128 * 9 + 5, Tkv=128 * 9 + 5, H=4, Hkv=2, d=64, S=128, k=3, tau=0.05, dtype="bf16")
    elif case == "f32_G16_S32_capacity":
        T = 32 * 20 + 7
        p = Problem(B=1, Tq=T, Tkv=T + 45, H=16, Hkv=1, d=64, S=32, k=5, dtype="f32")
        kv_len = T
    else:
        T = 64 * 50 + 9
        p = Problem(B=3, Tq=1, Tkv=T, H=8, Hkv=2, d=128, S=64, k=8, q_pos0=T, dtype="bf16")
    if kv_len is not None:
        inp_p = p
        r = _run(inp_p, seed=40, kv_len=kv_len)
        p = p.with_(Tkv=kv_len)
    else:
        r = _run(p, seed=40)
    if p.tau > 0:
        assert int((r["ke"] > p.k).sum()) > 0, "the router case must double some rows"
    _full_check(p, r)


def test_backward_without_candidates_is_zero():
    p = Problem(B=2, Tq=50, Tkv=50, H=4, Hkv=2, d=64, S=64, k=2, dtype="bf16")   # no complete chunk
    r = _run(p, seed=3)
    for name in ("dQ", "dK", "dV", "dW"):
        assert torch.all(r[name] == 0), name


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
    _close("dQ (sampled rows)", r["dQ"][0, torch.as_tensor(rows_t)], g["dQ"])
    dO = r["dO"].double()
    kept = (r["ke"] > 0).double()                                       # [B,Tq,Hkv]
    dOg = dO.view(p.B, p.Tq, p.Hkv, p.G, p.d).sum(3)                     # [B,Tq,Hkv,d]
    expect = (dOg * kept.unsqueeze(-1)).sum(1)                           # [B,Hkv,d]
    got = r["dV"].double().sum(1)
    scale = float(r["dV"].double().abs().sum(1).max())
    assert float((got - expect).abs().max()) <= 1e-5 * scale
    kscale = float(r["dK"].double().abs().sum(1).max())
    assert float(r["dK"].double().sum(1).abs().max()) <= 1e-5 * kscale
