"""Run the HSA forward on one named workload (optionally resized) a few times.

Used to drive profilers on a single, small, reproducible case:

    python -m landmark_guided_chunk_b200.run_case --workload prefill_bf16 --T 16384 --iters 3
    python -m landmark_guided_chunk_b200.run_case --workload decode_1m --B 2 --ctx 262144 --iters 3
    python -m landmark_guided_chunk_b200.run_case --workload decode_1m --select-only --iters 3
    python -m landmark_guided_chunk_b200.run_case --workload prefill_bf16 --T 16384 --backward --iters 3

--backward runs one forward (with its selection), then the backward of that
selection --iters times.
--select-only runs the selection stage alone on the workload's query shapes and
random landmarks, with no K/V allocated (the decode_1m selection then needs
0.25 GiB on the device instead of 32 GiB).

Prints the per-stage kernel paths and the wall time of the last iteration.
"""
from __future__ import annotations

import argparse
import time

import torch

import landmark_guided_chunk_b200 as hsa
from landmark_guided_chunk_b200.inputs import make_inputs, workload


def select_only(p, args):
    g = torch.Generator(device="cuda").manual_seed(0)
    dt = torch.bfloat16 if p.dtype == "bf16" else torch.float32
    Q = torch.randn(p.B, p.Tq, p.H, p.d, device="cuda", generator=g).to(dt)
    L = (torch.randn(p.B, p.Hkv, p.C, p.d, device="cuda", generator=g) / 8).to(dt)
    prob = hsa.make_problem(p.B, p.Tq, p.Tkv, p.H, p.Hkv, p.d, p.S, p.k, p.q_pos0, p.tau, dt,
                            hsa._native.HSA_FLAG_SIMT if args.simt else 0)
    ws = hsa.alloc_workspace(prob)
    for _ in range(args.iters):
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        hsa.select(Q, L, p.S, p.k, p.tau, p.q_pos0, Tkv=p.Tkv, ws=ws, force_simt=args.simt)
        torch.cuda.synchronize()
        dt_s = time.perf_counter() - t0
    hsa.device_status(ws)
    print(f"{p.name} (select only): B{p.B} Tq{p.Tq} Tkv{p.Tkv} plan={hsa.plan(prob)} last={dt_s * 1e3:.3f} ms")


def backward(p, args, Q, K, V, W):
    from landmark_guided_chunk_b200.inputs import make_output_grad
    O, L, idx, sc, ke = hsa.forward(Q, K, V, W, p.S, p.k, p.tau, p.q_pos0, return_selection=True)
    dO = make_output_grad(p, seed=1, device="cuda")
    prob = hsa.make_problem(p.B, p.Tq, p.Tkv, p.H, p.Hkv, p.d, p.S, p.k, p.q_pos0, p.tau, Q.dtype,
                            hsa._native.HSA_FLAG_SIMT if args.simt else 0)
    ws = torch.empty(hsa.backward_workspace_size(prob), dtype=torch.uint8, device="cuda")
    f32 = dict(dtype=torch.float32, device="cuda")
    out = (torch.empty(Q.shape, **f32), torch.empty(K.shape, **f32), torch.empty(K.shape, **f32),
           torch.empty(p.d, p.d, **f32))
    for _ in range(args.iters):
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        hsa.backward(Q, K, V, W, L, idx, sc, ke, dO, p.S, p.k, p.tau, p.q_pos0, out=out, ws=ws, force_simt=args.simt)
        torch.cuda.synchronize()
        dt = time.perf_counter() - t0
    hsa.device_status(ws)
    print(f"{p.name} backward: B{p.B} Tq{p.Tq} Tkv{p.Tkv} simt={args.simt} last={dt * 1e3:.3f} ms")


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", default="prefill_bf16")
    ap.add_argument("--T", type=int, default=None, help="prefill length (Tq = Tkv)")
    ap.add_argument("--ctx", type=int, default=None, help="decode context length")
    ap.add_argument("--B", type=int, default=None)
    ap.add_argument("--iters", type=int, default=3)
    ap.add_argument("--simt", action="store_true", help="CUDA-core kernels only")
    ap.add_argument("--select-only", action="store_true", help="selection stage only, random landmarks, no K/V")
    ap.add_argument("--backward", action="store_true", help="one forward, then the backward --iters times")
    args = ap.parse_args()
    p = workload(args.workload)
    if args.B is not None:
        p = p.with_(B=args.B)
    if args.T is not None:
        p = p.with_(Tq=args.T, Tkv=args.T)
    if args.ctx is not None:
        p = p.with_(Tkv=args.ctx, q_pos0=args.ctx)
    torch.cuda.set_device(0)
    if args.select_only:
        select_only(p, args)
        return
    inp = make_inputs(p, seed=0, device="cuda")
    Q, K, V, W = inp["Q"], inp["K"], inp["V"], inp["W_L"]
    ready = p.is_decode
    L = hsa.landmarks(K, W, p.S) if ready else None
    prob = hsa.make_problem(p.B, p.Tq, p.Tkv, p.H, p.Hkv, p.d, p.S, p.k, p.q_pos0, p.tau, Q.dtype,
                            (hsa._native.HSA_FLAG_LANDMARKS_READY if ready else 0) |
                            (hsa._native.HSA_FLAG_SIMT if args.simt else 0))
    ws = hsa.alloc_workspace(prob)
    O = torch.empty_like(Q)
    if args.backward:
        backward(p, args, Q, K, V, W)
        return
    for _ in range(args.iters):
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        hsa.forward(Q, K, V, None if ready else W, p.S, p.k, p.tau, p.q_pos0, L=L, landmarks_ready=ready, O=O,
                    ws=ws, force_simt=args.simt)
        torch.cuda.synchronize()
        dt = time.perf_counter() - t0
    hsa.device_status(ws)
    print(f"{p.name}: B{p.B} Tq{p.Tq} Tkv{p.Tkv} plan={hsa.plan(prob)} last={dt * 1e3:.3f} ms")


if __name__ == "__main__":
    main()
