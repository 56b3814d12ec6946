"""Parity of the CUDA path (through the C ABI) against the CPU oracle.

Small problems are checked on every row.  They span several tiles, with ragged
tails, both dtypes, d 64/128, S 32/64/128, G 1..8 and the router.  The full
workloads are checked on sampled rows (prefill) or on every row (decode: the
oracle rebuilds all landmarks from the cache).
"""
import numpy as np
import pytest
import torch

import landmark_guided_chunk_b200 as hsa
import oracle
from landmark_guided_chunk_b200.inputs import Problem, make_inputs, workload
from tests import parity

pytestmark = pytest.mark.gpu


def _rows_all(p: Problem):
    return np.repeat(np.arange(p.B), p.Tq), np.tile(np.arange(p.Tq), p.B)


def _rows_sampled(p: Problem, n: int, seed: int = 0):
    rng = np.random.default_rng(seed)
    fixed = [0, p.S - 1, p.S, 2 * p.S - 1, 2 * p.S, p.Tq // 2, p.Tq - p.S, p.Tq - 1]
    t = np.array(sorted(set([x for x in fixed if 0 <= x < p.Tq] + list(rng.integers(0, p.Tq, n)))))
    b = rng.integers(0, p.B, t.size)
    return b, t


def _oracle_L(p: Problem, inp):
    K, W = inp["K"], inp["W_L"]
    if K.numel() * K.element_size() > (2 << 30):
        return oracle.landmarks_stored_sliced(K, W, p.S, p.dtype)
    return oracle.landmarks_stored(K.cpu(), W.cpu(), p.S, p.dtype)


def run_case(p: Problem, rows=None, seed=0, landmarks_first=False, force_simt=False, host=False):
    torch.manual_seed(seed)
    inp = make_inputs(p, seed=seed, device="cuda")
    Q, K, V, W = inp["Q"], inp["K"], inp["V"], inp["W_L"]
    if landmarks_first:
        L = hsa.landmarks(K, W, p.S)
        O, L, idx, score, keff = hsa.forward(Q, K, V, None, p.S, p.k, p.tau, p.q_pos0, L=L,
                                             landmarks_ready=True, return_selection=True, force_simt=force_simt)
    else:
        O, L, idx, score, keff = hsa.forward(Q, K, V, W, p.S, p.k, p.tau, p.q_pos0, return_selection=True,
                                             force_simt=force_simt)
    torch.cuda.synchronize()
    if host:
        # the same forward from page-locked host buffers (hsa_forward_host): its O is the one checked
        Qh, Kh, Vh, Wh = (x.cpu().pin_memory() for x in (Q, K, V, W))
        Oh = hsa.forward_host(Qh, Kh, Vh, Wh, p.S, p.k, p.tau, p.q_pos0)
        torch.cuda.synchronize()
        assert not Oh.is_cuda
        O = Oh.cuda()
    L_orc = _oracle_L(p, inp)
    lm = parity.check_landmarks(L, L_orc)
    rb, rt = rows if rows is not None else _rows_all(p)
    tb, tt = torch.as_tensor(rb, device="cuda"), torch.as_tensor(rt, device="cuda")
    Qr = Q[tb, tt].cpu()
    # The selection is checked on the landmarks the library stored (pinned element-wise to
    # the oracle's just above): a value next to a bf16 rounding boundary may be stored one
    # ulp either way, which moves a score by up to |q|.ulp, and that is a property of the
    # stored landmarks, not of the scoring or the top-k.
    L_lib = L.double().cpu().numpy()
    orc = oracle.select(Qr, rb, rt + p.q_pos0, L_lib, p.S, p.k, p.tau, p.H, want_all=True)
    ncand = np.minimum((rt + p.q_pos0) // p.S, p.C)
    g_idx, g_sc, g_ke = idx[tb, tt].cpu().numpy(), score[tb, tt].cpu().numpy(), keff[tb, tt].cpu().numpy()
    sel = parity.check_selection(g_idx, g_sc, g_ke, orc, ncand, p.k, p.tau)
    O_exp = parity.expected_output(Qr, rb, K, V, p.S, orc, g_idx, g_ke, sel["tie_rows"])
    err = parity.check_output(O[tb, tt], O_exp, Q.dtype)
    # End to end: the oracle's selection on its OWN landmarks.  Rows whose kept set
    # differs from the GPU's are those where a stored landmark's rounding (one ulp
    # either way) moved a score across the cut; the rate is reported, not asserted exact.
    orc_e2e = oracle.select(Qr, rb, rt + p.q_pos0, L_orc, p.S, p.k, p.tau, p.H)
    mism = parity.selection_mismatch_rate(g_idx, g_ke, orc_e2e)
    return {"inp": inp, "O": O, "L": L, "idx": idx, "keff": keff, "sel": sel, "lm": lm, "err": err,
            "orc": orc, "rows": (rb, rt), "e2e_mismatch": mism}


SMALL = [
    workload("tiny_f32"),
    Problem(B=2, Tq=64 * 40 + 37, Tkv=64 * 40 + 37, H=8, Hkv=2, d=128, S=64, k=16, dtype="bf16", name="bf16_g4"),
    Problem(B=1, Tq=128 * 24 + 5, Tkv=128 * 24 + 5, H=8, Hkv=2, d=128, S=128, k=8, tau=0.02, dtype="bf16",
            name="bf16_router"),
    Problem(B=1, Tq=128 * 24 + 5, Tkv=128 * 24 + 5, H=8, Hkv=2, d=128, S=128, k=8, tau=0.3, dtype="bf16",
            name="bf16_router_wide"),
    Problem(B=2, Tq=32 * 50 + 9, Tkv=32 * 50 + 9, H=4, Hkv=4, d=64, S=32, k=5, dtype="bf16", name="bf16_d64_s32"),
    Problem(B=1, Tq=64 * 30, Tkv=64 * 30, H=16, Hkv=2, d=64, S=64, k=32, dtype="f32", name="f32_g8_k32"),
    Problem(B=1, Tq=64 * 20 + 63, Tkv=64 * 20 + 63, H=6, Hkv=3, d=128, S=64, k=3, tau=0.05, dtype="f32",
            name="f32_router"),
]


# shapes on the tensor-core attention beyond prefill_bf16's: group sizes that do not divide the 128
# rows of a tile (padding rows), and head dim 64
ODD_GROUPS = [
    Problem(B=2, Tq=64 * 33 + 21, Tkv=64 * 33 + 21, H=8, Hkv=2, d=64, S=64, k=8, dtype="bf16", name="bf16_d64_s64"),
    Problem(B=1, Tq=128 * 14 + 77, Tkv=128 * 14 + 77, H=12, Hkv=2, d=64, S=128, k=6, tau=0.05, dtype="bf16",
            name="bf16_d64_s128_g6"),
    Problem(B=1, Tq=64 * 30 + 11, Tkv=64 * 30 + 11, H=12, Hkv=2, d=128, S=64, k=8, dtype="bf16", name="bf16_g6"),
    Problem(B=2, Tq=64 * 17 + 40, Tkv=64 * 17 + 40, H=6, Hkv=2, d=128, S=64, k=5, dtype="bf16", name="bf16_g3"),
    Problem(B=2, Tq=128 * 12 + 3, Tkv=128 * 12 + 3, H=12, Hkv=1, d=128, S=128, k=4, tau=0.05, dtype="bf16",
            name="bf16_g12_router"),
]


def _plan(p: Problem, simt=False):
    return hsa.plan(hsa.make_problem(p.B, p.Tq, p.Tkv, p.H, p.Hkv, p.d, p.S, p.k, p.q_pos0, p.tau,
                                     torch.bfloat16 if p.dtype == "bf16" else torch.float32,
                                     hsa._native.HSA_FLAG_SIMT if simt else 0))


@pytest.mark.parametrize("p", SMALL, ids=lambda p: p.name)
def test_small_prefill_all_rows(p):
    r = run_case(p)
    assert r["sel"]["ties"] <= max(2, r["sel"]["exact"] // 200)
    print(f"{p.name}: end-to-end selection mismatch vs the oracle's own landmarks: {r['e2e_mismatch']:.4f}")
    assert r["e2e_mismatch"] <= 0.05


@pytest.mark.parametrize("p", SMALL[:3], ids=lambda p: p.name)
def test_forward_from_host_buffers(p):
    """hsa_forward_host: inputs copied up, the whole forward, O copied down, all on one stream;
    O checked against the oracle like the device-buffer forward's."""
    run_case(p, host=True)


def test_forward_host_calls_in_flight_on_three_streams():
    """Six hsa_forward_host calls on three streams, each stream with its own device buffer and
    workspace, so one call's uploads overlap another's compute and download: each O equals the
    device-buffer forward of its own inputs (up to the order of the fp32 accumulator additions)."""
    p = SMALL[1]
    prob = hsa.make_problem(p.B, p.Tq, p.Tkv, p.H, p.Hkv, p.d, p.S, p.k, p.q_pos0, p.tau, torch.bfloat16)
    streams = [torch.cuda.Stream() for _ in range(3)]
    devs = [torch.empty(hsa.forward_host_bytes(prob), dtype=torch.uint8, device="cuda") for _ in streams]
    wss = [hsa.alloc_workspace(prob) for _ in streams]
    host_in, outs, expect = [], [], []
    for seed in range(6):
        inp = make_inputs(p, seed=100 + seed, device="cuda")
        dev_in = (inp["Q"], inp["K"], inp["V"], inp["W_L"])
        expect.append(hsa.forward(*dev_in, p.S, p.k, p.tau, p.q_pos0).float().cpu())
        host_in.append(tuple(x.cpu().pin_memory() for x in dev_in))
    torch.cuda.synchronize()
    for i, (Qh, Kh, Vh, Wh) in enumerate(host_in):
        j = i % 3
        outs.append(hsa.forward_host(Qh, Kh, Vh, Wh, p.S, p.k, p.tau, p.q_pos0, dev=devs[j], ws=wss[j],
                                     stream=streams[j]))
    torch.cuda.synchronize()
    for O, E in zip(outs, expect):
        # one bf16 ulp of the element, plus the fp32 summation-order error of up to kmax terms of |w o| < 8
        tol = 2.0 ** -7 * E.abs() + 16 * 8 * 2.0 ** -24
        assert torch.all((O.float() - E).abs() <= tol), (O.float() - E).abs().max()
    for ws in wss:
        hsa.device_status(ws)


@pytest.mark.parametrize("p", ODD_GROUPS, ids=lambda p: p.name)
def test_tensor_attention_other_shapes(p):
    assert _plan(p)["attend"][0] == "tensor"
    r = run_case(p)
    assert r["sel"]["ties"] <= max(2, r["sel"]["exact"] // 200)


@pytest.mark.parametrize("p", [q for q in SMALL if q.dtype == "bf16"], ids=lambda p: p.name)
def test_small_prefill_cuda_core_path(p):
    """The same bf16 cases on the CUDA-core kernels (HSA_FLAG_SIMT), so both
    paths stay pinned to the oracle."""
    assert _plan(p, simt=True)["select"][0] != "tensor"
    r = run_case(p, force_simt=True)
    assert r["sel"]["ties"] <= max(2, r["sel"]["exact"] // 200)


def test_tensor_core_paths_are_the_ones_planned():
    # many rows in bf16: tcgen05 scoring and chunk-major tcgen05 attention
    for name in ("prefill_bf16", "router_bf16", "prefill_bf16_d64"):
        assert _plan(workload(name))["select"][0] == "tensor"
        assert _plan(workload(name))["attend"][0] == "tensor"
    assert _plan(SMALL[1])["select"][0] == "tensor"
    # few rows in bf16: the single-launch gather kernel (TMA + mma.sync)
    assert tuple(_plan(workload("decode_1m"))["attend"]) == ("mma_split", 1)
    # long decode scans in bf16: the streaming mma.sync scan with the merge folded in
    assert tuple(_plan(workload("decode_1m"))["select"]) == ("mma_split", 1)
    assert tuple(_plan(DECODE_SMALL[3])["select"]) == ("mma_split", 1)
    # hsa_forward runs the decode scan and the gather as one launch; prefill does not fuse
    assert _plan(workload("decode_1m"))["forward_fused"] and _plan(workload("decode_16m"))["forward_fused"]
    assert not _plan(workload("prefill_bf16"))["forward_fused"]


DECODE_SMALL = [
    Problem(B=3, Tq=1, Tkv=64 * 3000 + 17, H=8, Hkv=2, d=128, S=64, k=16, q_pos0=64 * 3000 + 17, dtype="bf16",
            planted=3, name="decode_split"),
    Problem(B=2, Tq=1, Tkv=64 * 700 + 5, H=4, Hkv=1, d=64, S=64, k=4, q_pos0=64 * 700 + 5, dtype="bf16",
            planted=2, name="decode_rows"),
    Problem(B=2, Tq=1, Tkv=128 * 2500, H=8, Hkv=2, d=128, S=128, k=8, tau=0.02, q_pos0=128 * 2500, dtype="bf16",
            planted=2, name="decode_router"),
    Problem(B=2, Tq=1, Tkv=32 * 2400 + 31, H=16, Hkv=2, d=64, S=32, k=12, q_pos0=32 * 2400 + 31, dtype="bf16",
            planted=2, name="decode_s32_g8"),
    Problem(B=2, Tq=1, Tkv=64 * 2200 + 9, H=8, Hkv=2, d=128, S=64, k=24, q_pos0=64 * 2200 + 9, dtype="bf16",
            planted=2, name="decode_k24"),
]


# few rows (<= 2048) with Tq > 1: the slot-parallel attention, with every
# supported (d, S) and group sizes up to 16
FEW_ROWS = [
    Problem(B=1, Tq=32 * 30 + 7, Tkv=32 * 30 + 7, H=16, Hkv=1, d=64, S=32, k=6, dtype="bf16", name="few_d64_s32_g16"),
    Problem(B=2, Tq=128 * 6 + 3, Tkv=128 * 6 + 3, H=6, Hkv=1, d=128, S=128, k=3, tau=0.1, dtype="bf16",
            name="few_d128_s128_g6"),
    Problem(B=1, Tq=64 * 12, Tkv=64 * 12, H=8, Hkv=2, d=64, S=64, k=16, dtype="bf16", name="few_d64_s64_k_all"),
]


@pytest.mark.parametrize("p", FEW_ROWS, ids=lambda p: p.name)
def test_few_rows_slot_parallel_attention(p):
    assert p.B * p.Tq * p.Hkv <= 2048
    run_case(p)


@pytest.mark.parametrize("p", DECODE_SMALL, ids=lambda p: p.name)
def test_small_decode(p):
    r = run_case(p, landmarks_first=True)
    idx, keff = r["idx"].cpu().numpy(), r["keff"].cpu().numpy()
    for b in range(p.B):
        for c in r["inp"]["planted"][b].tolist():
            for j in range(p.Hkv):
                assert c in idx[b, 0, j, :keff[b, 0, j]], f"planted chunk {c} missed (b={b}, kv={j})"


def test_attend_stage_with_oracle_selection():
    """hsa_attend alone, fed the oracle's selection: isolates the attention and fusion kernels."""
    p = Problem(B=2, Tq=64 * 24 + 11, Tkv=64 * 24 + 11, H=8, Hkv=2, d=128, S=64, k=16, dtype="bf16")
    inp = make_inputs(p, seed=3, device="cuda")
    Q, K, V, W = inp["Q"], inp["K"], inp["V"], inp["W_L"]
    L = oracle.landmarks_stored(K.cpu(), W.cpu(), p.S, p.dtype)
    rb, rt = _rows_all(p)
    Qr = Q.reshape(-1, p.H, p.d).cpu()
    sel = oracle.select(Qr, rb, rt, L, p.S, p.k, 0.0, p.H)
    sh = (p.B, p.Tq, p.Hkv)
    idx = torch.as_tensor(sel["idx"]).reshape(*sh, p.kmax).cuda()
    sc = torch.as_tensor(sel["score"]).float().reshape(*sh, p.kmax).cuda()
    ke = torch.as_tensor(sel["keff"]).reshape(*sh).cuda()
    O = hsa.attend(Q, K, V, idx, sc, ke, p.S, p.k)
    O_exp = oracle.attend(Qr, rb, K.cpu(), V.cpu(), p.S, sel)
    parity.check_output(O.reshape(-1, p.H, p.d), O_exp, Q.dtype)


@pytest.mark.parametrize("Hkv,d,S,dtype", [
    (32, 128, 64, "bf16"),   # 512 vectors per token row: one row group, each thread streams two columns
    (8, 128, 128, "bf16"),   # 128 vectors: two row groups of 64 rows
    (2, 64, 32, "bf16"),     # 16 vectors: sixteen row groups of 2 rows (tail loop only)
    (3, 64, 64, "f32"),      # 48 vectors: five row groups, 64 rows not a multiple of 5
    (6, 128, 128, "bf16"),   # 96 vectors: two row groups, 64 idle threads
])
def test_landmark_pooling_layouts(Hkv, d, S, dtype):
    """hsa_landmarks alone over the row-group layouts its pooling pass picks
    (HSA summary page, Implementation: mean pooling of each chunk, then W_L)."""
    p = Problem(B=2, Tq=1, Tkv=S * 37 + 5, H=Hkv, Hkv=Hkv, d=d, S=S, k=4, q_pos0=S * 37 + 5, dtype=dtype)
    inp = make_inputs(p, seed=11, device="cuda")
    K, W = inp["K"], inp["W_L"]
    L = hsa.landmarks(K, W, S)
    torch.cuda.synchronize()
    assert L.shape == (p.B, Hkv, 37, d)
    parity.check_landmarks(L, oracle.landmarks_stored(K.cpu(), W.cpu(), S, dtype))


def test_select_stage_alone_matches_forward():
    p = Problem(B=1, Tq=64 * 33, Tkv=64 * 33, H=8, Hkv=2, d=128, S=64, k=16, dtype="bf16")
    inp = make_inputs(p, seed=4, device="cuda")
    Q, K, V, W = inp["Q"], inp["K"], inp["V"], inp["W_L"]
    L = hsa.landmarks(K, W, p.S)
    idx, sc, ke = hsa.select(Q, L, p.S, p.k)
    O, L2, idx2, sc2, ke2 = hsa.forward(Q, K, V, W, p.S, p.k, return_selection=True)
    assert torch.equal(L, L2) and torch.equal(idx, idx2) and torch.equal(ke, ke2) and torch.equal(sc, sc2)


def test_edges_no_chunks_and_short_sequences():
    for T in (0, 1, 63, 64, 65, 130):
        p = Problem(B=2, Tq=T, Tkv=T, H=4, Hkv=2, d=64, S=64, k=4, dtype="bf16")
        inp = make_inputs(p, seed=5, device="cuda")
        O, L, idx, sc, ke = hsa.forward(inp["Q"], inp["K"], inp["V"], inp["W_L"], 64, 4, return_selection=True)
        torch.cuda.synchronize()
        if T == 0:
            continue
        t = torch.arange(T, device="cuda")
        want_ke = torch.clamp(t // 64, max=T // 64).to(torch.int32).view(1, T, 1).expand(2, T, 2)
        assert torch.equal(ke, torch.minimum(want_ke, torch.tensor(4, device="cuda", dtype=torch.int32)))
        assert torch.all(O[:, :64] == 0)


def test_batch_zero_is_a_no_op():
    p = hsa.make_problem(0, 5, 5, 4, 2, 64, 64, 4)
    assert hsa.workspace_size(p) >= 256
    Q = torch.empty(0, 5, 4, 64, dtype=torch.bfloat16, device="cuda")
    K = torch.empty(0, 5, 2, 64, dtype=torch.bfloat16, device="cuda")
    O = hsa.forward(Q, K, K, torch.eye(64, dtype=torch.bfloat16, device="cuda"), 64, 4)
    assert O.shape == Q.shape


def test_device_status_is_clear_after_calls():
    p = Problem(B=1, Tq=256, Tkv=256, H=4, Hkv=2, d=64, S=64, k=2, dtype="bf16")
    inp = make_inputs(p, seed=6, device="cuda")
    prob = hsa.make_problem(1, 256, 256, 4, 2, 64, 64, 2)
    ws = hsa.alloc_workspace(prob)
    ws.fill_(0xFF)                      # garbage: every call clears the status word first
    hsa.forward(inp["Q"], inp["K"], inp["V"], inp["W_L"], 64, 2, ws=ws)
    hsa.device_status(ws)


# ------------------------------------------------------------------- full workloads (sampled rows)

@pytest.mark.parametrize("name", ["prefill_bf16", "router_bf16", "prefill_bf16_d64"])
def test_full_prefill_workload_sampled_rows(name):
    p = workload(name)
    r = run_case(p, rows=_rows_sampled(p, 192))
    # end-to-end against the oracle's own landmarks: only near-boundary landmark roundings
    # can move a selection, so nearly every sampled row keeps the same set
    print(f"{name}: end-to-end selection mismatch vs the oracle's own landmarks: {r['e2e_mismatch']:.4f}")
    assert r["e2e_mismatch"] <= 0.05
    if p.tau > 0:
        ke = r["keff"].cpu().numpy()
        frac = float(np.mean(ke[:, p.S * (p.k + 1):] > p.k))
        assert 0.05 < frac < 0.95, f"router doubled {frac:.3f} of rows"


@pytest.mark.parametrize("name", ["decode_1m", "decode_16m"])
def test_full_decode_workload(name):
    p = workload(name)
    r = run_case(p, landmarks_first=True)
    idx, keff = r["idx"].cpu().numpy(), r["keff"].cpu().numpy()
    for b in range(p.B):
        for c in r["inp"]["planted"][b].tolist():
            for j in range(p.Hkv):
                assert c in idx[b, 0, j, :keff[b, 0, j]], f"planted chunk {c} missed (b={b}, kv={j})"
    del r
    torch.cuda.empty_cache()


FUSED = [q for q in DECODE_SMALL if q.name in ("decode_split", "decode_router", "decode_s32_g8")]


@pytest.mark.parametrize("p", FUSED + [workload("decode_1m")], ids=lambda p: p.name)
def test_fused_decode_step_equals_select_then_attend(p):
    """The fused decode launch (scan, then each published row's gather) gives
    the selection of hsa_select bit for bit and the O of hsa_attend on it (up
    to the order of the fp32 accumulator additions), on the same workspace
    called repeatedly (its publication slots and counters are reset per call)."""
    prob = hsa.make_problem(p.B, p.Tq, p.Tkv, p.H, p.Hkv, p.d, p.S, p.k, p.q_pos0, p.tau, torch.bfloat16,
                            hsa._native.HSA_FLAG_LANDMARKS_READY)
    assert hsa.plan(prob)["forward_fused"], hsa.plan(prob)
    inp = make_inputs(p, seed=11, device="cuda")
    Q, K, V, W = inp["Q"], inp["K"], inp["V"], inp["W_L"]
    L = hsa.landmarks(K, W, p.S)
    ws = hsa.alloc_workspace(prob)
    idx, sc, ke = hsa.select(Q, L, p.S, p.k, p.tau, p.q_pos0, Tkv=p.Tkv, ws=ws)
    O_ref = hsa.attend(Q, K, V, idx, sc, ke, p.S, p.k, p.tau, p.q_pos0, ws=ws)
    hsa.device_status(ws)
    for rep in range(3):
        O, _, idx2, sc2, ke2 = hsa.forward(Q, K, V, None, p.S, p.k, p.tau, p.q_pos0, L=L, landmarks_ready=True,
                                           return_selection=True, ws=ws)
        hsa.device_status(ws)
        assert torch.equal(idx2, idx) and torch.equal(ke2, ke) and torch.equal(sc2, sc), f"repeat {rep}"
        err = (O.float() - O_ref.float()).abs().max().item()
        scale = O_ref.float().abs().max().item()
        assert err <= 2 ** -7 * max(scale, 1.0), f"repeat {rep}: fused O differs by {err} (max |O| {scale})"
    del inp, Q, K, V, L, ws
    torch.cuda.empty_cache()


def test_attend_skips_and_reports_out_of_range_selection():
    """A corrupt caller selection is never dereferenced: the slot is skipped and
    the status word turns the call into HSA_ERR_INVALID_ARG."""
    p = Problem(B=1, Tq=64 * 6, Tkv=64 * 6, H=4, Hkv=2, d=64, S=64, k=2, dtype="bf16")
    inp = make_inputs(p, seed=7, device="cuda")
    Q, K, V, W = inp["Q"], inp["K"], inp["V"], inp["W_L"]
    L = hsa.landmarks(K, W, p.S)
    idx, sc, ke = hsa.select(Q, L, p.S, p.k)
    prob = hsa.make_problem(p.B, p.Tq, p.Tkv, p.H, p.Hkv, p.d, p.S, p.k)
    ws = hsa.alloc_workspace(prob)
    hsa.attend(Q, K, V, idx, sc, ke, p.S, p.k, ws=ws)
    hsa.device_status(ws)
    bad = idx.clone()
    bad[0, -1, 0, 0] = 1 << 20
    hsa.attend(Q, K, V, bad, sc, ke, p.S, p.k, ws=ws)
    with pytest.raises(hsa.HSAError) as e:
        hsa.device_status(ws)
    assert e.value.status == hsa._native.HSA_ERR_INVALID_ARG
    ke2 = ke.clone()
    ke2[0, -1, 1] = 99
    hsa.attend(Q, K, V, idx, sc, ke2, p.S, p.k, ws=ws)
    with pytest.raises(hsa.HSAError):
        hsa.device_status(ws)
    hsa.attend(Q, K, V, idx, sc, ke, p.S, p.k, ws=ws)
    hsa.device_status(ws)


@pytest.mark.parametrize("nchunks", [1000, 5000])
def test_scoring_prefill_continuation_over_a_long_context(nchunks):
    """A prefill continuation (128 new queries after a long cached context) on the
    tcgen05 scoring kernel: few M-tiles, each scanning thousands of chunks in many
    N-slices.  Checked on every row."""
    p = Problem(B=1, Tq=128, Tkv=64 * nchunks + 7, H=8, Hkv=2, d=128, S=64, k=16, tau=0.0,
                q_pos0=64 * nchunks + 7 - 128, dtype="bf16")
    prob = hsa.make_problem(p.B, p.Tq, p.Tkv, p.H, p.Hkv, p.d, p.S, p.k, p.q_pos0, p.tau, torch.bfloat16)
    assert hsa.plan(prob)["select"][0] == "tensor"
    inp = make_inputs(p, seed=13, device="cuda")
    Q, K, W = inp["Q"], inp["K"], inp["W_L"]
    L = hsa.landmarks(K, W, p.S)
    idx, score, keff = hsa.select(Q, L, p.S, p.k, p.tau, p.q_pos0, Tkv=p.Tkv)
    torch.cuda.synchronize()
    rb, rt = _rows_all(p)
    orc = oracle.select(Q.cpu().reshape(p.B * p.Tq, p.H, p.d), rb, rt + p.q_pos0, L.double().cpu().numpy(), p.S,
                        p.k, p.tau, p.H, want_all=True)
    ncand = np.minimum((rt + p.q_pos0) // p.S, p.C)
    sel = parity.check_selection(idx.reshape(-1, p.Hkv, p.k).cpu().numpy(), score.reshape(-1, p.Hkv, p.k).cpu().numpy(),
                                 keff.reshape(-1, p.Hkv).cpu().numpy(), orc, ncand, p.k, p.tau)
    assert sel["ties"] <= max(2, sel["exact"] // 100)
