"""Multi-rank host paths on CPU: two gloo ranks on 127.0.0.1.

* bench.py's rank helpers: the reported time is the maximum over ranks, and
  every rank takes the same barrier.
* The data-parallel backward's exchange (landmark_guided_chunk_b200.dp): each
  rank differentiates its own sequence (the oracle's backward stands in for the
  kernels), and after allreduce_param_grads every rank holds the W_L gradient of
  the whole batch -- the oracle's backward over both sequences at once.
* Context-sharded decode (landmark_guided_chunk_b200.sharded), the method
  itself: each rank holds a contiguous range of a sequence's chunks, keeps its
  local top kmax with the router off (its candidates counted from
  sharded.local_q_pos), and contributes their scores, global chunk indices and
  per-chunk attention outputs -- computed here by the oracle -- through
  sharded.gather_shards.  Merging the gathered lists (top kmax of the union,
  ranked score descending then lower chunk, the gap router on the merged list,
  softmax weights over the kept scores) must reproduce the oracle's selection
  and output over the whole context.  The CUDA merge kernel itself is checked
  against the oracle in tests/test_sharded_gpu.py.
"""
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle

WORLD = 2


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _init(rank, port):
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=WORLD,
                            timeout=__import__("datetime").timedelta(seconds=60))


def _bench_helpers(rank, port):
    _init(rank, port)
    try:
        import bench
        bench.barrier(WORLD)
        assert bench.max_over_ranks(1.5 + rank, WORLD) == 1.5 + WORLD - 1
        bench.barrier(WORLD)
    finally:
        dist.destroy_process_group()


def test_bench_rank_helpers():
    mp.spawn(_bench_helpers, args=(_free_port(),), nprocs=WORLD, join=True)


def _shard_problem():
    rng = np.random.default_rng(77)
    B, H, Hkv, d, S = 1, 4, 2, 64, 32
    C = 37
    Tkv = C * S + 11                      # a trailing partial chunk, never a candidate
    Q = torch.tensor(rng.standard_normal((B, H, d)), dtype=torch.float64)
    K = torch.tensor(rng.standard_normal((B, Tkv, Hkv, d)), dtype=torch.float64)
    V = torch.tensor(rng.standard_normal((B, Tkv, Hkv, d)), dtype=torch.float64)
    W = torch.tensor(rng.standard_normal((d, d)) / d ** 0.5, dtype=torch.float64)
    return B, H, Hkv, d, S, C, Tkv, Q, K, V, W


def _chunk_outputs(Qr, rb, K, V, S, idx, keff):
    """o_i for every kept slot: the oracle's attention of a selection that keeps that chunk alone."""
    n, Hkv, km = idx.shape
    H, d = Qr.shape[1], Qr.shape[2]
    G = H // Hkv
    o = np.zeros((n, Hkv, km, G, d))
    for i in range(km):
        one = {"idx": np.full((n, Hkv, 1), -1, dtype=np.int32), "score": np.zeros((n, Hkv, 1)),
               "keff": np.zeros((n, Hkv), dtype=np.int32)}
        one["idx"][:, :, 0] = idx[:, :, i]
        one["keff"][:] = (keff > i).astype(np.int32)
        out = oracle.attend(Qr, rb, K, V, S, one).reshape(n, Hkv, G, d)
        o[:, :, i] = out
    return o


def _merge(score, gidx, keff, o, k, tau):
    """The merge rule over shard-major lists [P, n, Hkv, kmax(, G, d)]."""
    P, n, Hkv, km = gidx.shape
    G, d = o.shape[-2], o.shape[-1]
    O = np.zeros((n, Hkv, G, d))
    sel_idx = np.full((n, Hkv, km), -1)
    sel_ke = np.zeros((n, Hkv), dtype=np.int64)
    for r in range(n):
        for j in range(Hkv):
            cand = [(score[p, r, j, i], int(gidx[p, r, j, i]), p, i)
                    for p in range(P) for i in range(int(keff[p, r, j]))]
            cand.sort(key=lambda e: (-e[0], e[1]))
            cand = cand[:km]
            ke = min(k, len(cand))
            if tau > 0 and len(cand) > k:
                sk, sk1 = cand[k - 1][0], cand[k][0]
                if sk - sk1 < tau * abs(sk):
                    ke = min(2 * k, len(cand))
            s = np.array([c[0] for c in cand[:ke]])
            w = np.exp(s - s.max()) / np.exp(s - s.max()).sum() if ke else s
            for q in range(ke):
                O[r, j] += w[q] * o[cand[q][2], r, j, cand[q][3]]
            sel_idx[r, j, :ke] = [c[1] for c in cand[:ke]]
            sel_ke[r, j] = ke
    return O, sel_idx, sel_ke


def _sharded_method(rank, port, k, tau):
    _init(rank, port)
    try:
        from landmark_guided_chunk_b200 import sharded
        B, H, Hkv, d, S, C, Tkv, Q, K, V, W = _shard_problem()
        km = 2 * k if tau > 0 else k
        bounds = [0, 19, C]
        c0, c1 = bounds[rank], bounds[rank + 1]
        t1 = c1 * S if rank < WORLD - 1 else Tkv
        Kg, Vg = K[:, c0 * S:t1].contiguous(), V[:, c0 * S:t1].contiguous()
        Lg = oracle.landmarks(Kg, W, S)                       # this rank's chunks only
        rb = np.zeros(B, dtype=np.int64)
        qp = sharded.local_q_pos(Tkv, c0, S)
        sel = oracle.select(Q, rb, np.array([qp]), Lg, S, km, 0.0, H)
        gidx = np.where(sel["idx"] >= 0, sel["idx"] + c0, sel["idx"])
        o = _chunk_outputs(Q, rb, Kg, Vg, S, sel["idx"], sel["keff"])
        sc_all, ix_all, ke_all, o_all = sharded.gather_shards(
            (torch.tensor(sel["score"]), torch.tensor(gidx), torch.tensor(sel["keff"]), torch.tensor(o)))
        assert sc_all.shape[0] == WORLD and o_all.shape == (WORLD,) + o.shape
        O, sidx, ske = _merge(sc_all.numpy(), ix_all.numpy(), ke_all.numpy(), o_all.numpy(), k, tau)
        # the whole context on one "device"
        L = oracle.landmarks(K, W, S)
        ref = oracle.select(Q, rb, np.array([Tkv]), L, S, k, tau, H)
        O_ref = oracle.attend(Q, rb, K, V, S, ref).reshape(O.shape)
        assert np.array_equal(ske, ref["keff"]), (ske, ref["keff"])
        for j in range(Hkv):
            ke = int(ske[0, j])
            assert np.array_equal(sidx[0, j, :ke], ref["idx"][0, j, :ke]), (sidx[0, j], ref["idx"][0, j])
        assert np.max(np.abs(O - O_ref)) < 1e-12
    finally:
        dist.destroy_process_group()


def test_sharded_decode_method_two_ranks():
    mp.spawn(_sharded_method, args=(_free_port(), 4, 0.0), nprocs=WORLD, join=True)


def test_sharded_decode_method_two_ranks_router():
    mp.spawn(_sharded_method, args=(_free_port(), 3, 0.3), nprocs=WORLD, join=True)


def _dp_problem():
    rng = np.random.default_rng(91)
    B, T, H, Hkv, d, S = WORLD, 32 * 6 + 9, 4, 2, 16, 32
    Q = torch.tensor(rng.standard_normal((B, T, H, d)))
    K = torch.tensor(rng.standard_normal((B, T, Hkv, d)))
    V = torch.tensor(rng.standard_normal((B, T, Hkv, d)))
    W = torch.tensor(rng.standard_normal((d, d)) / d ** 0.5)
    dO = rng.standard_normal((B, T, H, d))
    return Q, K, V, W, dO, S


def _oracle_backward(Q, K, V, W, dO, S, k):
    B, T = Q.shape[:2]
    rb, rp = np.repeat(np.arange(B), T), np.tile(np.arange(T), B)
    Qr = Q.reshape(B * T, *Q.shape[2:])
    L = oracle.landmarks(K, W, S)
    sel = oracle.select(Qr, rb, rp, L, S, k, 0.0, Q.shape[2])
    return oracle.backward(Qr, rb, K, V, W, L, S, sel, dO.reshape(B * T, *dO.shape[2:]))


def _dp_backward(rank, port):
    _init(rank, port)
    try:
        from landmark_guided_chunk_b200 import dp
        Q, K, V, W, dO, S = _dp_problem()
        mine = _oracle_backward(Q[rank:rank + 1], K[rank:rank + 1], V[rank:rank + 1], W, dO[rank:rank + 1], S, 3)
        dW = torch.tensor(mine["dW"])
        dp.allreduce_param_grads(dW)
        whole = _oracle_backward(Q, K, V, W, dO, S, 3)
        assert np.allclose(dW.numpy(), whole["dW"], atol=1e-12, rtol=0)
        # the per-sequence gradients need no exchange: this rank's rows of the whole batch
        T = Q.shape[1]
        assert np.allclose(mine["dQ"], whole["dQ"][rank * T:(rank + 1) * T], atol=1e-12)
        assert np.allclose(mine["dK"][0], whole["dK"][rank], atol=1e-12)
        assert np.allclose(mine["dV"][0], whole["dV"][rank], atol=1e-12)
    finally:
        dist.destroy_process_group()


def test_data_parallel_backward_exchange_two_ranks():
    mp.spawn(_dp_backward, args=(_free_port(),), nprocs=WORLD, join=True)


def _oracle_forward(Q, K, V, W, S, k, tau):
    B, T, H, d = Q.shape
    rb, rt = np.repeat(np.arange(B), T), np.tile(np.arange(T), B)
    out = oracle.forward_rows(Q, K, V, W, S, k, tau, 0, rb, rt)
    return torch.tensor(out["O"]).reshape(B, T, H, d)


def _sharded_prefill(rank, port, B, Hkv, expect_kind):
    """The (b, kv head) split of a prefill: each rank computes its shard (the
    oracle stands in for the kernels) and one all-gather assembles O; it must
    equal the oracle over the whole problem, bit for bit (the units share nothing)."""
    _init(rank, port)
    try:
        from landmark_guided_chunk_b200 import sharded
        rng = np.random.default_rng(5)
        T, G, d, S, k = 32 * 7 + 5, 2, 16, 32, 3
        H = Hkv * G
        Q = torch.tensor(rng.standard_normal((B, T, H, d)), dtype=torch.float32)
        K = torch.tensor(rng.standard_normal((B, T, Hkv, d)), dtype=torch.float32)
        V = torch.tensor(rng.standard_normal((B, T, Hkv, d)), dtype=torch.float32)
        W = torch.tensor(rng.standard_normal((d, d)) / d ** 0.5, dtype=torch.float32)
        kind, Qr, Kr, Vr = sharded.shard_inputs(Q, K, V, WORLD, rank)
        assert kind == expect_kind
        O = sharded.sharded_prefill(Qr, Kr, Vr, W, S, k, 0.0, kind=kind, gather=True, forward_fn=_oracle_forward)
        ref = _oracle_forward(Q, K, V, W, S, k, 0.0)
        assert O.shape == ref.shape
        assert torch.equal(O, ref)
        mine = sharded.sharded_prefill(Qr, Kr, Vr, W, S, k, 0.0, kind=kind, forward_fn=_oracle_forward)
        a = rank * (Hkv // WORLD) * G if kind == "heads" else 0
        if kind == "heads":
            assert torch.equal(mine, ref[:, :, a:a + Qr.shape[2]])
        else:
            assert torch.equal(mine, ref[rank * (B // WORLD):(rank + 1) * (B // WORLD)])
    finally:
        dist.destroy_process_group()


def test_sharded_prefill_kv_head_split_two_ranks():
    mp.spawn(_sharded_prefill, args=(_free_port(), 1, 4, "heads"), nprocs=WORLD, join=True)


def test_sharded_prefill_batch_split_two_ranks():
    mp.spawn(_sharded_prefill, args=(_free_port(), 2, 3, "batch"), nprocs=WORLD, join=True)
