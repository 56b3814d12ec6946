"""Context-sharded decode on one GPU: the context's chunks are split into
nshard contiguous ranges, each shard's part runs on its own copy of its K, V
and landmarks, and the shard-major stack of their outputs (what the all-gather
of landmark_guided_chunk_b200.sharded leaves every rank) is merged.

HSA summary page, Implementation: the merged selection and output must be those
of one device holding the whole context.  They are checked against the oracle
on the whole context (selection exact up to near ties, output within the
dtype's tolerance) and against the single-device forward.
"""
import numpy as np
import pytest
import torch

import landmark_guided_chunk_b200 as hsa
import oracle
from landmark_guided_chunk_b200 import sharded
from landmark_guided_chunk_b200.inputs import Problem, make_inputs
from tests import parity

pytestmark = pytest.mark.gpu


def _split(C, nshard):
    return [round(g * C / nshard) for g in range(nshard + 1)]


@pytest.mark.parametrize("nshard,B,Tkv,k,tau,S", [
    (2, 2, 64 * 40 + 7, 8, 0.0, 64),
    (3, 1, 64 * 50 + 31, 4, 0.05, 64),        # router on: shards keep 2k, the merge decides
    (4, 1, 64 * 8400 + 5, 16, 0.0, 64),       # 2100 chunks per shard: each on the streaming scan
    (5, 2, 128 * 23, 6, 0.0, 128),            # uneven ranges, some shards with fewer than kmax chunks
])
def test_sharded_decode_matches_whole_context(nshard, B, Tkv, k, tau, S):
    p = Problem(B=B, Tq=1, Tkv=Tkv, H=8, Hkv=2, d=128, S=S, k=k, tau=tau, q_pos0=Tkv, dtype="bf16")
    inp = make_inputs(p, seed=31, device="cuda")
    Q, K, V = inp["Q"], inp["K"], inp["V"]
    g = torch.Generator(device="cuda").manual_seed(32)
    W = (torch.randn(p.d, p.d, generator=g, device="cuda") / p.d ** 0.5).to(K.dtype)
    L = hsa.landmarks(K, W, S)
    C = p.C
    bounds = _split(C, nshard)
    parts = []
    for sh in range(nshard):
        c0, c1 = bounds[sh], bounds[sh + 1]
        t1 = c1 * S if sh < nshard - 1 else Tkv   # the last shard also holds the trailing partial chunk
        Kg, Vg = K[:, c0 * S:t1].contiguous(), V[:, c0 * S:t1].contiguous()
        Lg = L[:, :, c0:c1].contiguous()
        parts.append(sharded.shard_partials(Q, Kg, Vg, Lg, S, k, tau, Tkv, c0))
    stacked = [torch.stack([pt[i] for pt in parts]) for i in range(4)]
    O, idx, sc, ke = hsa.merge_partials(*stacked, S, k, tau, dtype=Q.dtype, return_selection=True)

    # oracle on the whole context
    rb, rt = np.arange(B), np.zeros(B, dtype=np.int64)
    Qr = Q[:, 0].cpu()
    orc = oracle.select(Qr, rb, rt + Tkv, L.double().cpu().numpy(), S, k, tau, p.H, want_all=True)
    ncand = np.minimum((rt + Tkv) // S, C)
    g_idx, g_ke = idx[:, 0].cpu().numpy(), ke[:, 0].cpu().numpy()
    sel = parity.check_selection(g_idx, sc[:, 0].cpu().numpy(), g_ke, orc, ncand, k, tau)
    O_exp = parity.expected_output(Qr, rb, K, V, S, orc, g_idx, g_ke, sel["tie_rows"])
    parity.check_output(O[:, 0], O_exp, Q.dtype)

    # and the single-device forward: same selection wherever the cut is not a near tie
    Of, _, idxf, scf, kef = hsa.forward(Q, K, V, None, S, k, tau, q_pos0=Tkv, L=L, landmarks_ready=True,
                                        return_selection=True)
    tie = {(r, j) for (r, j) in sel["tie_rows"]}
    for b in range(B):
        for j in range(p.Hkv):
            if (b, j) in tie:
                continue
            assert int(ke[b, 0, j]) == int(kef[b, 0, j])
            assert torch.equal(idx[b, 0, j, :int(ke[b, 0, j])], idxf[b, 0, j, :int(kef[b, 0, j])])
    assert float((O.double() - Of.double()).abs().max()) <= 2e-2


def test_merge_rejects_mismatched_slots():
    o = torch.zeros(2, 1, 1, 2, 8, 4, 128, device="cuda")
    sc = torch.zeros(2, 1, 1, 2, 8, device="cuda")
    ix = torch.zeros(2, 1, 1, 2, 8, dtype=torch.int32, device="cuda")
    ke = torch.zeros(2, 1, 1, 2, dtype=torch.int32, device="cuda")
    with pytest.raises(ValueError):
        hsa.merge_partials(sc, ix, ke, o, 64, 8, tau=0.05)   # the router doubles k: 16 slots expected


@pytest.mark.parametrize("world", [2, 4])
def test_prefill_kv_head_shards_match_the_oracle(world):
    """The (b, kv head) split of one prefill sequence: every rank's shard, run
    through the CUDA forward on this device, against the oracle on that shard's
    rows (its kv heads' landmarks, selection and output)."""
    from landmark_guided_chunk_b200 import sharded
    p = Problem(B=1, Tq=64 * 20 + 13, Tkv=64 * 20 + 13, H=16, Hkv=4, d=128, S=64, k=8, dtype="bf16")
    inp = make_inputs(p, seed=9, device="cuda")
    Q, K, V, W = inp["Q"], inp["K"], inp["V"], inp["W_L"]
    outs = []
    for r in range(world):
        kind, Qr, Kr, Vr = sharded.shard_inputs(Q, K, V, world, r)
        assert kind == "heads"
        O, L, idx, sc, ke = hsa.forward(Qr, Kr, Vr, W, p.S, p.k, return_selection=True)
        torch.cuda.synchronize()
        B, T, Hr, d = Qr.shape
        rb, rt = np.repeat(np.arange(B), T), np.tile(np.arange(T), B)
        Lr = L.double().cpu().numpy()
        parity.check_landmarks(L, oracle.landmarks_stored(Kr.cpu(), W.cpu(), p.S, "bf16"))
        orc = oracle.select(Qr.cpu().reshape(B * T, Hr, d), rb, rt, Lr, p.S, p.k, 0.0, Hr, want_all=True)
        ncand = np.minimum(rt // p.S, p.C)
        sel = parity.check_selection(idx.reshape(-1, Kr.shape[2], p.k).cpu().numpy(),
                                     sc.reshape(-1, Kr.shape[2], p.k).cpu().numpy(),
                                     ke.reshape(-1, Kr.shape[2]).cpu().numpy(), orc, ncand, p.k, 0.0)
        O_exp = parity.expected_output(Qr.cpu().reshape(B * T, Hr, d), rb, Kr, Vr, p.S, orc,
                                       idx.reshape(-1, Kr.shape[2], p.k).cpu().numpy(),
                                       ke.reshape(-1, Kr.shape[2]).cpu().numpy(), sel["tie_rows"])
        parity.check_output(O.reshape(B * T, Hr, d), O_exp, torch.bfloat16)
        outs.append(O)
    # the shards tile the heads: together they are the single-device result's layout
    assert torch.cat(outs, dim=2).shape == Q.shape
