"""hsa_select_noalloc: the selection stage for callers that cannot allocate
device memory (for example, code running under an allocator that must not be
re-entered).  Instead of a caller workspace it uses the library's own fixed
1 MiB device scratch.  Its output must equal hsa_select's (same kernels), on
two calls in a row (the scratch keeps the previous call's contents).

This file is collected last on purpose; it must also pass when run alone in a
fresh process."""
import ctypes

import pytest
import torch

import landmark_guided_chunk_b200 as hsa
from landmark_guided_chunk_b200 import _native
from landmark_guided_chunk_b200.inputs import Problem, make_inputs

pytestmark = pytest.mark.gpu

CASES = [
    # few rows with long scans: the split path, whose candidate lists live in the scratch
    Problem(B=3, Tq=1, Tkv=64 * 3000 + 17, H=8, Hkv=2, d=128, S=64, k=16, q_pos0=64 * 3000 + 17, dtype="bf16",
            name="decode_split"),
    # many rows: the tensor-core path, which only needs the scratch's status word
    Problem(B=1, Tq=64 * 40 + 9, Tkv=64 * 40 + 9, H=8, Hkv=2, d=128, S=64, k=8, tau=0.1, dtype="bf16",
            name="prefill_router"),
]


def _noalloc_call(p, Q, L, out):
    prob = hsa.make_problem(p.B, p.Tq, p.Tkv, p.H, p.Hkv, p.d, p.S, p.k, p.q_pos0, p.tau, Q.dtype)
    idx, score, keff = out
    st = torch.cuda.current_stream().cuda_stream
    return _native.lib().hsa_select_noalloc(ctypes.byref(prob), ctypes.c_void_p(Q.data_ptr()),
                                            ctypes.c_void_p(L.data_ptr()), ctypes.c_void_p(idx.data_ptr()),
                                            ctypes.c_void_p(score.data_ptr()), ctypes.c_void_p(keff.data_ptr()), st)


@pytest.mark.parametrize("p", CASES, ids=lambda p: p.name)
def test_noalloc_select_equals_workspace_select_twice(p):
    torch.cuda.set_device(0)
    inp = make_inputs(p, seed=11, device="cuda")
    Q, K, W = inp["Q"], inp["K"], inp["W_L"]
    L = hsa.landmarks(K, W, p.S)
    ref_idx, ref_score, ref_keff = hsa.select(Q, L, p.S, p.k, p.tau, p.q_pos0, Tkv=p.Tkv)
    for _ in range(2):
        out = (torch.full_like(ref_idx, -7), torch.full_like(ref_score, 7.0), torch.full_like(ref_keff, -7))
        assert _noalloc_call(p, Q, L, out) == _native.HSA_OK
        # the call's device-status word (in the static scratch) reports a clean run
        assert _native.lib().hsa_noalloc_status(torch.cuda.current_stream().cuda_stream) == _native.HSA_OK
        torch.cuda.synchronize()
        assert torch.equal(out[0], ref_idx)
        assert torch.equal(out[2], ref_keff)
        # same kernels, same order of arithmetic: the scores agree exactly
        assert torch.equal(out[1], ref_score)


def test_noalloc_select_rejects_a_problem_beyond_its_scratch():
    # 4096 decode rows x 32 slots (k = 16 with the router): the candidate lists need 1 MiB + the status word
    p = Problem(B=2048, Tq=1, Tkv=64 * 4096, H=2, Hkv=2, d=64, S=64, k=16, q_pos0=64 * 4096, tau=0.5, dtype="bf16")
    assert hsa.plan(hsa.make_problem(p.B, p.Tq, p.Tkv, p.H, p.Hkv, p.d, p.S, p.k, p.q_pos0, p.tau))["select"][0] \
        == "mma_split"
    prob = hsa.make_problem(p.B, p.Tq, p.Tkv, p.H, p.Hkv, p.d, p.S, p.k, p.q_pos0, p.tau)
    fake = ctypes.c_void_p(256)   # never dereferenced: the size check comes first
    rc = _native.lib().hsa_select_noalloc(ctypes.byref(prob), fake, fake, fake, fake, fake, None)
    assert rc == _native.HSA_ERR_WORKSPACE
    assert b"static scratch" in _native.lib().hsa_last_error()


def test_noalloc_timeout_is_reported_by_its_status_reader():
    """A device-side timeout inside hsa_select_noalloc lands in the static
    scratch's status word; hsa_noalloc_status reports it (the test flag makes
    the scoring kernel's wait run out, see tests/test_failure_gpu.py), and the
    next call is clean and equal to hsa_select."""
    torch.cuda.set_device(0)
    p = CASES[1]
    inp = make_inputs(p, seed=12, device="cuda")
    Q, K, W = inp["Q"], inp["K"], inp["W_L"]
    L = hsa.landmarks(K, W, p.S)
    st = torch.cuda.current_stream().cuda_stream
    ref_idx, ref_score, ref_keff = hsa.select(Q, L, p.S, p.k, p.tau, p.q_pos0, Tkv=p.Tkv)
    out = (torch.empty_like(ref_idx), torch.empty_like(ref_score), torch.empty_like(ref_keff))
    prob = hsa.make_problem(p.B, p.Tq, p.Tkv, p.H, p.Hkv, p.d, p.S, p.k, p.q_pos0, p.tau, Q.dtype,
                            _native.HSA_FLAG_TEST_STALL)
    rc = _native.lib().hsa_select_noalloc(ctypes.byref(prob), ctypes.c_void_p(Q.data_ptr()),
                                          ctypes.c_void_p(L.data_ptr()), ctypes.c_void_p(out[0].data_ptr()),
                                          ctypes.c_void_p(out[1].data_ptr()), ctypes.c_void_p(out[2].data_ptr()), st)
    assert rc == _native.HSA_OK
    assert _native.lib().hsa_noalloc_status(st) == _native.HSA_ERR_TIMEOUT
    assert _native.lib().hsa_noalloc_status(st) == _native.HSA_OK   # read and cleared
    assert _noalloc_call(p, Q, L, out) == _native.HSA_OK
    assert _native.lib().hsa_noalloc_status(st) == _native.HSA_OK
    assert torch.equal(out[0], ref_idx) and torch.equal(out[2], ref_keff) and torch.equal(out[1], ref_score)
