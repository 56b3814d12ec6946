"""The HSA_DEBUG build on the GPU: with every kernel-derived index checked on
the device (gathered tokens and chunks, TMA coordinates, accumulator offsets),
the prefill forward, the fused decode step and the backward run clean (status
word zero) and still match the oracle.  The library is chosen when the binding
loads, so the cases run in a child process with HSA_DEBUG=1."""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r"""
import torch
import landmark_guided_chunk_b200 as hsa
from landmark_guided_chunk_b200 import _native
from landmark_guided_chunk_b200.inputs import Problem, make_inputs, make_output_grad
from tests.test_parity_gpu import run_case, SMALL, DECODE_SMALL
from tests.test_backward_gpu import TOL_TC, _full_check, _run

assert _native.DEBUG and _native.lib().hsa_debug_checks() == 1
torch.cuda.set_device(0)
bwd = Problem(B=1, Tq=64 * 12 + 7, Tkv=64 * 12 + 7, H=8, Hkv=2, d=128, S=64, k=4, dtype="bf16", name="dbg_bwd")
cases = [q for q in SMALL if q.dtype == "bf16"][:2] + DECODE_SMALL[:1]
for p in cases:
    ready = p.is_decode
    run_case(p, landmarks_first=ready)       # parity with the oracle under the debug build
    # the same calls on a workspace whose status word is then read: no check may have fired
    inp = make_inputs(p, seed=0, device="cuda")
    Q, K, V, W = inp["Q"], inp["K"], inp["V"], inp["W_L"]
    prob = hsa.make_problem(p.B, p.Tq, p.Tkv, p.H, p.Hkv, p.d, p.S, p.k, p.q_pos0, p.tau, Q.dtype,
                            _native.HSA_FLAG_LANDMARKS_READY if ready else 0)
    ws = hsa.alloc_workspace(prob)
    L = hsa.landmarks(K, W, p.S) if ready else None
    O, L, idx, sc, ke = hsa.forward(Q, K, V, None if ready else W, p.S, p.k, p.tau, p.q_pos0, L=L,
                                    landmarks_ready=ready, return_selection=True, ws=ws)
    hsa.device_status(ws)
    if p.name == bwd.name or not ready:
        dO = make_output_grad(p, seed=2, device="cuda")
        bws = torch.empty(max(256, hsa.backward_workspace_size(prob)), dtype=torch.uint8, device="cuda")
        hsa.backward(Q, K, V, W, L, idx, sc, ke, dO, p.S, p.k, p.tau, q_pos0=p.q_pos0, ws=bws)
        hsa.device_status(bws)
errs = _full_check(bwd, _run(bwd, seed=5), TOL_TC)
print("debug build ok", max(errs.values()))
"""

@pytest.mark.gpu
def test_debug_build_runs_clean_against_the_oracle():
    lib = os.path.join(ROOT, "landmark_guided_chunk_b200", "libhsa_b200_debug.so")
    assert os.path.exists(lib), "build the debug library first (build.py --debug)"
    env = dict(os.environ, HSA_DEBUG="1", PYTHONPATH=ROOT)
    r = subprocess.run([sys.executable, "-c", CHILD], cwd=ROOT, env=env, capture_output=True, text=True,
                       timeout=900)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-3000:]
    assert "debug build ok" in r.stdout
