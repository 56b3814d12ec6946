"""Failure detection on the GPU, without a fault or a hang.

Every mbarrier wait of the tensor-core kernels is bounded.  Under the test flag
HSA_FLAG_TEST_STALL the tcgen05 scoring kernel runs with a 0.1 ms limit and its
epilogue first waits on a barrier that nothing arrives on.  That wait runs out:
the waiter raises the CTA's abort flag and the status word, the producer drains
its TMA loads, the MMA thread commits and drains, and TMEM is freed.  The host
then reads HSA_ERR_TIMEOUT through hsa_get_device_status, and the next normal
call on the same workspace and stream must be clean and match the oracle."""
import ctypes

import numpy as np
import pytest
import torch

import landmark_guided_chunk_b200 as hsa
import oracle
from landmark_guided_chunk_b200 import _native
from landmark_guided_chunk_b200.inputs import Problem, make_inputs
from tests import parity

pytestmark = pytest.mark.gpu

P = Problem(B=2, Tq=64 * 12 + 5, Tkv=64 * 12 + 5, H=8, Hkv=2, d=128, S=64, k=4, tau=0.1, dtype="bf16",
            name="stall_probe")


def _select(prob, Q, L, out, ws):
    idx, score, keff = out
    st = torch.cuda.current_stream().cuda_stream
    P_ = hsa._p
    return _native.lib().hsa_select(ctypes.byref(prob), P_(Q), P_(L), P_(idx), P_(score), P_(keff), P_(ws),
                                    ws.numel(), st)


def _status(ws):
    return _native.lib().hsa_get_device_status(hsa._p(ws), ws.numel(), torch.cuda.current_stream().cuda_stream)


def test_scoring_wait_expiry_reports_timeout_and_the_next_call_is_clean():
    torch.cuda.set_device(0)
    p = P
    inp = make_inputs(p, seed=3, device="cuda")
    Q, K, W = inp["Q"], inp["K"], inp["W_L"]
    L = hsa.landmarks(K, W, p.S)
    base = hsa.make_problem(p.B, p.Tq, p.Tkv, p.H, p.Hkv, p.d, p.S, p.k, p.q_pos0, p.tau, torch.bfloat16)
    stall = hsa.make_problem(p.B, p.Tq, p.Tkv, p.H, p.Hkv, p.d, p.S, p.k, p.q_pos0, p.tau, torch.bfloat16,
                             _native.HSA_FLAG_TEST_STALL)
    assert hsa.plan(stall)["select"][0] == "tensor"
    ws = hsa.alloc_workspace(base)
    km = hsa.kmax_of(p.k, p.tau)
    mk = lambda: (torch.full((p.B, p.Tq, p.Hkv, km), -7, dtype=torch.int32, device="cuda"),  # noqa: E731
                  torch.full((p.B, p.Tq, p.Hkv, km), 7.0, dtype=torch.float32, device="cuda"),
                  torch.full((p.B, p.Tq, p.Hkv), -7, dtype=torch.int32, device="cuda"))

    # the stalled call launches normally; its kernel times out and winds down
    out = mk()
    assert _select(stall, Q, L, out, ws) == _native.HSA_OK
    assert _status(ws) == _native.HSA_ERR_TIMEOUT
    assert b"bounded device wait expired" in _native.lib().hsa_last_error()
    # the status word was cleared by the read; the context is usable
    assert _status(ws) == _native.HSA_OK
    torch.cuda.synchronize()

    # a normal call on the same workspace and stream: clean, and equal to the oracle's selection
    for _ in range(2):
        out = mk()
        assert _select(base, Q, L, out, ws) == _native.HSA_OK
        assert _status(ws) == _native.HSA_OK
        idx, score, keff = out
        rb, rt = np.repeat(np.arange(p.B), p.Tq), np.tile(np.arange(p.Tq), p.B)
        orc = oracle.select(Q.cpu().reshape(p.B * p.Tq, p.H, p.d), rb, rt + p.q_pos0, L.double().cpu().numpy(),
                            p.S, p.k, p.tau, p.H, want_all=True)
        ncand = np.minimum((rt + p.q_pos0) // p.S, p.C)
        parity.check_selection(idx.reshape(-1, p.Hkv, km).cpu().numpy(), score.reshape(-1, p.Hkv, km).cpu().numpy(),
                               keff.reshape(-1, p.Hkv).cpu().numpy(), orc, ncand, p.k, p.tau)


def test_timeout_is_per_call():
    """A timed-out call does not leak into the next one: each call clears the
    status word when it starts."""
    torch.cuda.set_device(0)
    p = P
    inp = make_inputs(p, seed=4, device="cuda")
    Q, K, W = inp["Q"], inp["K"], inp["W_L"]
    L = hsa.landmarks(K, W, p.S)
    base = hsa.make_problem(p.B, p.Tq, p.Tkv, p.H, p.Hkv, p.d, p.S, p.k, p.q_pos0, p.tau, torch.bfloat16)
    stall = hsa.make_problem(p.B, p.Tq, p.Tkv, p.H, p.Hkv, p.d, p.S, p.k, p.q_pos0, p.tau, torch.bfloat16,
                             _native.HSA_FLAG_TEST_STALL)
    ws = hsa.alloc_workspace(base)
    km = hsa.kmax_of(p.k, p.tau)
    out = (torch.empty(p.B, p.Tq, p.Hkv, km, dtype=torch.int32, device="cuda"),
           torch.empty(p.B, p.Tq, p.Hkv, km, dtype=torch.float32, device="cuda"),
           torch.empty(p.B, p.Tq, p.Hkv, dtype=torch.int32, device="cuda"))
    assert _select(stall, Q, L, out, ws) == _native.HSA_OK
    assert _select(base, Q, L, out, ws) == _native.HSA_OK   # not read in between
    assert _status(ws) == _native.HSA_OK
