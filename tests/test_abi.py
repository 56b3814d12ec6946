"""The C ABI on the host: the library loads, exports every entry point that
include/hsa.h declares, and rejects bad calls before launching anything."""
import ctypes
import os
import re

import pytest

import landmark_guided_chunk_b200 as hsa
from landmark_guided_chunk_b200 import _native

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    txt = open(os.path.join(ROOT, "include", "hsa.h")).read()
    return re.findall(r"HSA_API\s+[\w\s\*]+?\b(hsa_\w+)\s*\(", txt)


def test_library_exports_every_declared_symbol():
    names = _declared()
    assert len(names) >= 9
    lib = _native.lib()
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(_native.EXPORTED)
    assert lib.hsa_abi_version() == 6
    assert lib.hsa_debug_checks() == (1 if _native.DEBUG else 0)


def test_debug_library_exports_every_declared_symbol():
    """The HSA_DEBUG build (device-side index checks) has the same ABI and says so."""
    path = os.path.join(ROOT, "landmark_guided_chunk_b200", "libhsa_b200_debug.so")
    if not os.path.exists(path):
        from landmark_guided_chunk_b200 import build
        build.build(debug=True)
    dbg = ctypes.CDLL(path)
    for n in _declared():
        assert hasattr(dbg, n), n
    dbg.hsa_abi_version.restype = ctypes.c_int
    dbg.hsa_debug_checks.restype = ctypes.c_int
    assert dbg.hsa_abi_version() == 6
    assert dbg.hsa_debug_checks() == 1


def test_status_strings():
    lib = _native.lib()
    for s in range(6):
        assert lib.hsa_status_string(s).startswith(b"HSA_")


def _prob(**kw):
    base = dict(B=1, Tq=128, Tkv=128, H=4, Hkv=2, d=64, S=64, k=4, q_pos0=0, tau=0.0, dtype=torch_bf16(), flags=0)
    base.update(kw)
    return hsa.make_problem(**base)


def torch_bf16():
    import torch
    return torch.bfloat16


@pytest.mark.parametrize("kw,status", [
    (dict(H=5), _native.HSA_ERR_INVALID_ARG),
    (dict(B=-1), _native.HSA_ERR_INVALID_ARG),
    (dict(k=0), _native.HSA_ERR_INVALID_ARG),
    (dict(tau=-0.1), _native.HSA_ERR_INVALID_ARG),
    (dict(tau=float("nan")), _native.HSA_ERR_INVALID_ARG),
    (dict(tau=float("inf")), _native.HSA_ERR_INVALID_ARG),
    (dict(q_pos0=-3), _native.HSA_ERR_INVALID_ARG),
    (dict(flags=64), _native.HSA_ERR_INVALID_ARG),
    (dict(d=96), _native.HSA_ERR_UNSUPPORTED),
    (dict(S=48), _native.HSA_ERR_UNSUPPORTED),
    (dict(k=33), _native.HSA_ERR_UNSUPPORTED),
    (dict(k=17, tau=0.1), _native.HSA_ERR_UNSUPPORTED),
    (dict(H=34, Hkv=2), _native.HSA_ERR_UNSUPPORTED),
    (dict(Tkv=128, kv_cap=127), _native.HSA_ERR_INVALID_ARG),
])
def test_workspace_size_rejects_bad_problems(kw, status):
    with pytest.raises(hsa.HSAError) as e:
        hsa.workspace_size(_prob(**kw))
    assert e.value.status == status


def test_workspace_size_grows_with_rows_and_is_aligned():
    a = hsa.workspace_size(_prob(Tq=4096, Tkv=4096))
    b = hsa.workspace_size(_prob(Tq=8192, Tkv=8192))
    assert a >= 256 and b > a and a % 256 == 0 and b % 256 == 0


def _call_forward(prob, Q=16, K=16, V=16, W=16, L=16, O=16, ws=256, ws_bytes=1 << 30):
    lib = _native.lib()
    P = lambda x: None if x is None else ctypes.c_void_p(x)
    return lib.hsa_forward(ctypes.byref(prob), P(Q), P(K), P(V), P(W), P(L), None, None, None, P(O), P(ws),
                           ws_bytes, None)


def test_forward_validates_pointers_before_launch():
    """Fake, never-dereferenced addresses: every call below must fail in host validation."""
    p = _prob()
    assert _call_forward(p, Q=None) == _native.HSA_ERR_INVALID_ARG
    assert _call_forward(p, K=24) == _native.HSA_ERR_INVALID_ARG            # misaligned
    assert _call_forward(p, O=None) == _native.HSA_ERR_INVALID_ARG
    assert _call_forward(p, W=None) == _native.HSA_ERR_INVALID_ARG
    assert _call_forward(p, ws=None) == _native.HSA_ERR_WORKSPACE
    assert _call_forward(p, ws=272) == _native.HSA_ERR_WORKSPACE            # not 256-aligned
    assert _call_forward(p, ws_bytes=64) == _native.HSA_ERR_WORKSPACE
    assert b"workspace" in _native.lib().hsa_last_error()
    ready = _prob(flags=_native.HSA_FLAG_LANDMARKS_READY)
    assert _call_forward(ready, W=None, L=None) == _native.HSA_ERR_INVALID_ARG   # L is required


def _host_bytes(prob):
    n = ctypes.c_size_t()
    assert _native.lib().hsa_forward_host_bytes(ctypes.byref(prob), ctypes.byref(n)) == _native.HSA_OK
    return n.value


def test_forward_host_bytes_is_the_sum_of_its_aligned_copies():
    """Q, K, V, W_L, the landmarks and O, each rounded up to 256 bytes (bf16: 2 bytes an element)."""
    up = lambda n: (n + 255) // 256 * 256
    B, T, H, Hkv, d, S = 2, 1000, 4, 2, 64, 64
    q = B * T * H * d * 2
    kv = B * 1024 * Hkv * d * 2                                           # K and V copied whole (Tcap = 1024)
    lm = B * Hkv * (1024 // S) * d * 2
    p = _prob(B=B, Tq=T, Tkv=T, H=H, Hkv=Hkv, d=d, S=S, kv_cap=1024)
    assert _host_bytes(p) == up(q) + 2 * up(kv) + up(d * d * 2) + up(lm) + up(q)
    quest = _prob(B=B, Tq=T, Tkv=T, H=H, Hkv=Hkv, d=d, S=S, kv_cap=1024, flags=_native.HSA_FLAG_QUEST)
    assert _host_bytes(quest) == up(q) + 2 * up(kv) + up(2 * lm) + up(q)  # no W_L, summaries of width 2d
    assert _host_bytes(_prob(B=0)) == 64 * 64 * 2                          # W_L alone


def _call_forward_host(prob, Q=16, K=16, V=16, W=16, O=16, dev=256, dev_bytes=None, ws=256, ws_bytes=1 << 30):
    P = lambda x: None if x is None else ctypes.c_void_p(x)
    dev_bytes = _host_bytes(prob) if dev_bytes is None else dev_bytes
    return _native.lib().hsa_forward_host(ctypes.byref(prob), P(Q), P(K), P(V), P(W), P(O), P(dev), dev_bytes,
                                          P(ws), ws_bytes, None)


def test_forward_host_validates_before_enqueueing():
    """Fake, never-dereferenced addresses: every call below must fail in host validation."""
    p = _prob()
    for kw in (dict(Q=None), dict(K=None), dict(V=None), dict(W=None), dict(O=None), dict(dev=None),
               dict(dev=272), dict(dev_bytes=_host_bytes(p) - 1)):
        assert _call_forward_host(p, **kw) == _native.HSA_ERR_INVALID_ARG, kw
    assert b"device buffer" in _native.lib().hsa_last_error()
    assert _call_forward_host(p, ws=None) == _native.HSA_ERR_WORKSPACE
    assert _call_forward_host(p, ws_bytes=64) == _native.HSA_ERR_WORKSPACE
    ready = _prob(flags=_native.HSA_FLAG_LANDMARKS_READY)
    assert _call_forward_host(ready) == _native.HSA_ERR_INVALID_ARG
    assert b"LANDMARKS_READY" in _native.lib().hsa_last_error()
    quest = _prob(flags=_native.HSA_FLAG_QUEST)                            # Quest reads no W_L ...
    assert _call_forward_host(quest, W=None, dev=None) == _native.HSA_ERR_INVALID_ARG
    assert b"device buffer" in _native.lib().hsa_last_error()             # ... so only the buffer is missing


def _call_append(prob, kn=16, vn=16, K=16, V=16, W=16, L=16):
    P = lambda x: None if x is None else ctypes.c_void_p(x)
    return _native.lib().hsa_decode_append(ctypes.byref(prob), P(kn), P(vn), P(K), P(V), P(W), P(L), None)


def test_decode_append_validates_before_launch():
    """Fake, never-dereferenced addresses: every call below must fail in host validation."""
    full = _prob(Tq=1, Tkv=256, kv_cap=256, q_pos0=256)
    assert _call_append(full) == _native.HSA_ERR_INVALID_ARG                # no room to append
    assert b"no room" in _native.lib().hsa_last_error()
    tight = _prob(Tq=1, Tkv=130, kv_cap=0, q_pos0=130)                      # kv_cap 0 = Tkv: full too
    assert _call_append(tight) == _native.HSA_ERR_INVALID_ARG
    p = _prob(Tq=1, Tkv=130, kv_cap=256, q_pos0=130)
    assert _call_append(p, kn=None) == _native.HSA_ERR_INVALID_ARG
    assert _call_append(p, V=24) == _native.HSA_ERR_INVALID_ARG              # misaligned
    completes = _prob(Tq=1, Tkv=127, kv_cap=256, q_pos0=127)                 # token 127 completes chunk 1
    assert _call_append(completes, W=None) == _native.HSA_ERR_INVALID_ARG
    assert _call_append(completes, L=None) == _native.HSA_ERR_INVALID_ARG


def test_null_problem_and_status_reader():
    lib = _native.lib()
    n = ctypes.c_size_t()
    assert lib.hsa_workspace_size(None, ctypes.byref(n)) == _native.HSA_ERR_INVALID_ARG
    assert lib.hsa_get_device_status(None, 0, None) == _native.HSA_ERR_WORKSPACE


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    monkeypatch.setattr(_native, "_lib", None)
    monkeypatch.setattr(_native, "LIB_PATH", str(tmp_path / "nope.so"))
    with pytest.raises(RuntimeError, match="not built"):
        _native.lib()


def _call_backward(prob, ws_bytes=1 << 20, **ptrs):
    names = ("Q", "K", "V", "W", "L", "idx", "score", "keff", "dO", "dQ", "dK", "dV", "dW", "ws")
    vals = {n: 256 for n in names}
    vals.update(ptrs)
    P = lambda x: None if x is None else ctypes.c_void_p(x)
    return _native.lib().hsa_backward(ctypes.byref(prob), *[P(vals[n]) for n in names[:-1]], P(vals["ws"]),
                                      ws_bytes, None)


def test_backward_workspace_and_validation_before_launch():
    """hsa_backward_workspace_size is host arithmetic; every call below fails in host
    validation (fake, never-dereferenced addresses)."""
    p = _prob()
    n = ctypes.c_size_t()
    assert _native.lib().hsa_backward_workspace_size(ctypes.byref(p), ctypes.byref(n)) == _native.HSA_OK
    rows, kmax, G, C = 128 * 2, 4, 2, 2
    assert n.value >= rows * kmax * (4 + 4 * G + 4) + 2 * C * 64 * 4
    assert _call_backward(p, dO=None) == _native.HSA_ERR_INVALID_ARG
    assert b"dO" in _native.lib().hsa_last_error()
    assert _call_backward(p, dK=24) == _native.HSA_ERR_INVALID_ARG             # misaligned
    assert _call_backward(p, ws=None) == _native.HSA_ERR_WORKSPACE
    assert _call_backward(p, ws_bytes=16) == _native.HSA_ERR_WORKSPACE
    assert _call_backward(p, ws=256 + 16) == _native.HSA_ERR_WORKSPACE        # not 256-byte aligned
    assert _call_backward(_prob(H=5)) == _native.HSA_ERR_INVALID_ARG


def test_quest_flag_host_rules():
    """Quest scoring: the workspace holds the transformed query rows, the plan adds
    their kernel, and the calls that do not implement it refuse before launching."""
    plain, quest = _prob(), _prob(flags=_native.HSA_FLAG_QUEST)
    assert hsa.workspace_size(quest) >= hsa.workspace_size(plain) + 128 * 2 * 2 * 2 * 64 * 2
    assert hsa.plan(quest)["select"][1] == hsa.plan(plain)["select"][1] + 1
    n = ctypes.c_size_t(0)
    assert _native.lib().hsa_backward_workspace_size(ctypes.byref(quest), ctypes.byref(n)) == \
        _native.HSA_ERR_UNSUPPORTED
    fake = ctypes.c_void_p(256)
    assert _native.lib().hsa_select_noalloc(ctypes.byref(quest), fake, fake, fake, fake, fake, None) == \
        _native.HSA_ERR_UNSUPPORTED
    assert _native.lib().hsa_landmarks_refined(ctypes.byref(quest), fake, fake, fake, fake, fake, fake, None) == \
        _native.HSA_ERR_INVALID_ARG
    # the refiner needs every weight
    assert _native.lib().hsa_landmarks_refined(ctypes.byref(plain), fake, fake, fake, None, fake, fake, None) == \
        _native.HSA_ERR_INVALID_ARG


def test_fused_decode_plan_host_rules():
    """hsa_forward fuses the decode scan and the gather only for decode-shaped bf16 problems
    with long contexts that both kernels support, never under Quest scoring, and the
    fused plan adds no attention launch.  The workspace grows by the unit descriptors."""
    from landmark_guided_chunk_b200.inputs import workload
    bf16 = torch_bf16()

    def plan_of(p, flags=0):
        return hsa.plan(hsa.make_problem(p.B, p.Tq, p.Tkv, p.H, p.Hkv, p.d, p.S, p.k, p.q_pos0, p.tau, bf16, flags))

    for name in ("decode_1m", "decode_16m"):
        pl = plan_of(workload(name))
        assert pl["forward_fused"] and pl["select"] == ("mma_split", 1) and pl["attend"] == ("mma_split", 1)
        assert not plan_of(workload(name), _native.HSA_FLAG_QUEST)["forward_fused"]
        assert not plan_of(workload(name), _native.HSA_FLAG_SIMT)["forward_fused"]
    assert not plan_of(workload("prefill_bf16"))["forward_fused"]
    # a short context (under 2048 candidate chunks) takes the per-row scan: no fusion
    short = workload("decode_1m").with_(Tkv=64 * 1500, q_pos0=64 * 1500)
    assert not plan_of(short)["forward_fused"]
    # so many rows that the scan needs more CTAs than there are SMs: they could not all be resident
    # at once, so the scan and the gather stay two launches
    wide = workload("decode_1m").with_(B=64, Tkv=64 * 4096, q_pos0=64 * 4096)
    assert plan_of(wide)["select"][0] == "mma_split" and not plan_of(wide)["forward_fused"]
    # the fused layout holds one 8-byte descriptor per (row, slot) on top of the unfused one
    p = workload("decode_1m")
    fused = hsa.workspace_size(hsa.make_problem(p.B, p.Tq, p.Tkv, p.H, p.Hkv, p.d, p.S, p.k, p.q_pos0, p.tau, bf16))
    assert fused >= p.B * p.Hkv * p.k * 8
