"""B200-native Hierarchical Sparse Attention (HSA) forward path.

Method: "Every Token Counts 16m Context" (HSA summary page), Core Technique
and Implementation.  The sequence is cut into chunks of S tokens, each with a
landmark (the mean of its keys times W_L).  Each query keeps the top-k
strictly-past chunks by landmark score, attends inside each kept chunk, and
fuses the chunk outputs by the softmax of their retrieval scores.  The gap
router of the value-of-information router page optionally doubles k.

Python surface over the C ABI in include/hsa.h (libhsa_b200.so).  Torch
supplies device memory and the current stream.  Every step runs in the CUDA
kernels of that library, and there is no CPU or PyTorch fallback.
"""
from __future__ import annotations

import ctypes

import torch

from . import _native
from ._native import HSAError, hsa_problem_t

__all__ = ["make_problem", "plan", "workspace_size", "alloc_workspace", "landmarks", "landmarks_refined",
           "quest_summaries", "select", "select_noalloc", "attend", "forward", "forward_host",
           "forward_host_bytes", "decode_append", "attend_partials", "merge_partials", "device_status", "HSAError",
           "hsa_problem_t", "kmax_of", "backward", "backward_workspace_size"]

_DT = {torch.float32: _native.HSA_F32, torch.bfloat16: _native.HSA_BF16}


def make_problem(B, Tq, Tkv, H, Hkv, d, S, k, q_pos0=0, tau=0.0, dtype=torch.bfloat16, flags=0,
                 kv_cap=0) -> hsa_problem_t:
    """Tkv = cached tokens; kv_cap = tokens the K/V buffers hold per sequence (0 = Tkv)."""
    if dtype not in _DT:
        raise TypeError(f"dtype {dtype} not supported (float32, bfloat16)")
    return hsa_problem_t(B, Tq, Tkv, H, Hkv, d, S, k, q_pos0, tau, _DT[dtype], flags, kv_cap)


def plan(prob: hsa_problem_t) -> dict:
    """Kernel path and launch count of each stage for this problem (nothing is launched)."""
    pl = _native.hsa_plan_t()
    _native.check(_native.lib().hsa_plan(ctypes.byref(prob), ctypes.byref(pl)), "hsa_plan")
    names = _native.PATH_NAMES
    return {"landmarks": (names[pl.landmark_path], pl.landmark_kernels),
            "select": (names[pl.select_path], pl.select_kernels),
            "attend": (names[pl.attend_path], pl.attend_kernels),
            "forward_fused": bool(pl.forward_fused)}


def kmax_of(k: int, tau: float) -> int:
    return 2 * k if tau > 0 else k


def workspace_size(prob: hsa_problem_t) -> int:
    n = ctypes.c_size_t(0)
    _native.check(_native.lib().hsa_workspace_size(ctypes.byref(prob), ctypes.byref(n)), "hsa_workspace_size")
    return int(n.value)


def alloc_workspace(prob: hsa_problem_t, device=None) -> torch.Tensor:
    """A uint8 device buffer of hsa_workspace_size bytes (torch allocations are 256-byte aligned)."""
    n = max(256, workspace_size(prob))
    ws = torch.empty(n, dtype=torch.uint8, device=device if device is not None else "cuda")
    assert ws.data_ptr() % 256 == 0
    return ws


def _stream(t: torch.Tensor) -> int:
    return torch.cuda.current_stream(t.device).cuda_stream


def _dev(*ts):
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("all tensors must be CUDA tensors")
        if t is not None and not t.is_contiguous():
            raise ValueError("all tensors must be contiguous")


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def landmarks(K: torch.Tensor, W_L: torch.Tensor, S: int, L: torch.Tensor | None = None,
              kv_len: int | None = None) -> torch.Tensor:
    """L [B,Hkv,Tcap//S,d] = mean of each complete chunk's keys times W_L (rounded once to K's
    dtype), for the chunks of the first kv_len tokens (default: all Tcap = K.shape[1])."""
    _dev(K, W_L, L)
    B, Tcap, Hkv, d = K.shape
    Tkv = Tcap if kv_len is None else kv_len
    if L is None:
        L = torch.empty(B, Hkv, Tcap // S, d, dtype=K.dtype, device=K.device)
    prob = make_problem(B, 0, Tkv, Hkv, Hkv, d, S, 1, 0, 0.0, K.dtype, kv_cap=Tcap)
    _native.check(_native.lib().hsa_landmarks(ctypes.byref(prob), _p(K), _p(W_L), _p(L), _stream(K)),
                  "hsa_landmarks")
    return L


def landmarks_refined(K: torch.Tensor, W_L: torch.Tensor, W_q: torch.Tensor, W_k: torch.Tensor, W_v: torch.Tensor,
                      S: int, L: torch.Tensor | None = None, kv_len: int | None = None) -> torch.Tensor:
    """Refined landmarks [B,Hkv,Tcap//S,d]: the pooled landmark L0 = mean(K_c) W_L plus one head of
    cross-attention from it to the chunk's keys, softmax((L0 W_q)(K_c W_k)^T / sqrt(d)) K_c W_v."""
    _dev(K, W_L, W_q, W_k, W_v, L)
    B, Tcap, Hkv, d = K.shape
    Tkv = Tcap if kv_len is None else kv_len
    if L is None:
        L = torch.empty(B, Hkv, Tcap // S, d, dtype=K.dtype, device=K.device)
    prob = make_problem(B, 0, Tkv, Hkv, Hkv, d, S, 1, 0, 0.0, K.dtype, kv_cap=Tcap)
    _native.check(_native.lib().hsa_landmarks_refined(ctypes.byref(prob), _p(K), _p(W_L), _p(W_q), _p(W_k), _p(W_v),
                                                      _p(L), _stream(K)), "hsa_landmarks_refined")
    return L


def quest_summaries(K: torch.Tensor, S: int, Lq: torch.Tensor | None = None, kv_len: int | None = None) -> torch.Tensor:
    """Quest chunk summaries Lq [B,Hkv,Tcap//S,2d]: the channel-wise max of each complete chunk's
    keys, then the channel-wise min (hsa_landmarks under HSA_FLAG_QUEST)."""
    _dev(K, Lq)
    B, Tcap, Hkv, d = K.shape
    Tkv = Tcap if kv_len is None else kv_len
    if Lq is None:
        Lq = torch.empty(B, Hkv, Tcap // S, 2 * d, dtype=K.dtype, device=K.device)
    prob = make_problem(B, 0, Tkv, Hkv, Hkv, d, S, 1, 0, 0.0, K.dtype, _native.HSA_FLAG_QUEST, kv_cap=Tcap)
    _native.check(_native.lib().hsa_landmarks(ctypes.byref(prob), _p(K), None, _p(Lq), _stream(K)), "hsa_landmarks")
    return Lq


def _prob_from(Q, Tkv, Hkv, S, k, tau, q_pos0, flags=0, kv_cap=0):
    B, Tq, H, d = Q.shape
    return make_problem(B, Tq, Tkv, H, Hkv, d, S, k, q_pos0, tau, Q.dtype, flags, kv_cap)


def _l_cap(Tkv, Ccap, S):
    """kv_cap whose chunk stride is L's Ccap (L may hold more chunks than Tkv has)."""
    return max(Tkv, Ccap * S)


def select(Q, L, S, k, tau=0.0, q_pos0=0, Tkv=None, ws=None, force_simt=False, quest=False):
    """Top-k chunk selection.  Returns (idx int32, score fp32 [B,Tq,Hkv,kmax], keff int32 [B,Tq,Hkv]).
    quest: L holds Quest chunk summaries [B,Hkv,C,2d] and the scores are Quest's bounds."""
    _dev(Q, L, ws)
    B, Tq, H, d = Q.shape
    Hkv, C = L.shape[1], L.shape[2]
    Tkv = Tkv if Tkv is not None else C * S
    flags = (_native.HSA_FLAG_SIMT if force_simt else 0) | (_native.HSA_FLAG_QUEST if quest else 0)
    prob = _prob_from(Q, Tkv, Hkv, S, k, tau, q_pos0, flags, _l_cap(Tkv, C, S))
    km = kmax_of(k, tau)
    idx = torch.empty(B, Tq, Hkv, km, dtype=torch.int32, device=Q.device)
    score = torch.empty(B, Tq, Hkv, km, dtype=torch.float32, device=Q.device)
    keff = torch.empty(B, Tq, Hkv, dtype=torch.int32, device=Q.device)
    if ws is None:
        ws = alloc_workspace(prob, Q.device)
    _native.check(_native.lib().hsa_select(ctypes.byref(prob), _p(Q), _p(L), _p(idx), _p(score), _p(keff),
                                           _p(ws), ws.numel(), _stream(Q)), "hsa_select")
    return idx, score, keff


def select_noalloc(Q, L, S, k, tau=0.0, q_pos0=0, Tkv=None, out=None):
    """hsa_select without a workspace: the library's own fixed 1 MiB device
    scratch is used instead (see include/hsa.h for who needs this and its
    limits).  out, if given, is (idx, score, keff) to fill; they are allocated
    here otherwise."""
    _dev(Q, L)
    B, Tq, H, d = Q.shape
    Hkv, C = L.shape[1], L.shape[2]
    Tkv = Tkv if Tkv is not None else C * S
    prob = _prob_from(Q, Tkv, Hkv, S, k, tau, q_pos0, 0, _l_cap(Tkv, C, S))
    km = kmax_of(k, tau)
    if out is None:
        out = (torch.empty(B, Tq, Hkv, km, dtype=torch.int32, device=Q.device),
               torch.empty(B, Tq, Hkv, km, dtype=torch.float32, device=Q.device),
               torch.empty(B, Tq, Hkv, dtype=torch.int32, device=Q.device))
    idx, score, keff = out
    _dev(idx, score, keff)
    _native.check(_native.lib().hsa_select_noalloc(ctypes.byref(prob), _p(Q), _p(L), _p(idx), _p(score), _p(keff),
                                                   _stream(Q)), "hsa_select_noalloc")
    return idx, score, keff


def attend(Q, K, V, idx, score, keff, S, k, tau=0.0, q_pos0=0, O=None, ws=None, force_simt=False, kv_len=None):
    """Chunk attention + fusion for a given selection.  Returns O [B,Tq,H,d].  kv_len: cached
    tokens when the K/V buffers hold more (default: all of K.shape[1])."""
    _dev(Q, K, V, idx, score, keff, O, ws)
    Tcap = K.shape[1]
    prob = _prob_from(Q, Tcap if kv_len is None else kv_len, K.shape[2], S, k, tau, q_pos0,
                      _native.HSA_FLAG_SIMT if force_simt else 0, Tcap)
    if O is None:
        O = torch.empty_like(Q)
    if ws is None:
        ws = alloc_workspace(prob, Q.device)
    _native.check(_native.lib().hsa_attend(ctypes.byref(prob), _p(Q), _p(K), _p(V), _p(idx), _p(score),
                                           _p(keff), _p(O), _p(ws), ws.numel(), _stream(Q)), "hsa_attend")
    return O


def forward(Q, K, V, W_L, S, k, tau=0.0, q_pos0=0, L=None, landmarks_ready=False, O=None, ws=None,
            return_selection=False, force_simt=False, kv_len=None, quest=False, refine=None):
    """The whole HSA forward.  Returns O, or (O, L, idx, score, keff) with return_selection.
    force_simt runs the CUDA-core kernels even where tensor-core ones exist (for A/B tests).
    kv_len: cached tokens when the K/V buffers (and L) hold more, as in a decode loop (default:
    all of K.shape[1]); L is then [B, Hkv, K.shape[1] // S, d].
    quest: Quest block scoring (L = chunk summaries [.., 2d], W_L unused).
    refine: (W_q, W_k, W_v) -- the landmarks are the refined ones (hsa_landmarks_refined), then
    the forward runs on them."""
    _dev(Q, K, V, W_L, L, O, ws)
    B, Tq, H, d = Q.shape
    Tcap, Hkv = K.shape[1], K.shape[2]
    Tkv = Tcap if kv_len is None else kv_len
    if refine is not None:
        if quest or landmarks_ready:
            raise ValueError("refine makes the landmarks: not with quest or landmarks_ready")
        L = landmarks_refined(K, W_L, *refine, S, L=L, kv_len=kv_len)
        landmarks_ready = True
    flags = ((_native.HSA_FLAG_LANDMARKS_READY if landmarks_ready else 0) |
             (_native.HSA_FLAG_SIMT if force_simt else 0) | (_native.HSA_FLAG_QUEST if quest else 0))
    prob = _prob_from(Q, Tkv, Hkv, S, k, tau, q_pos0, flags, Tcap)
    if L is None:
        if landmarks_ready:
            raise ValueError("landmarks_ready needs L")
        L = torch.empty(B, Hkv, Tcap // S, 2 * d if quest else d, dtype=Q.dtype, device=Q.device)
    if O is None:
        O = torch.empty_like(Q)
    if ws is None:
        ws = alloc_workspace(prob, Q.device)
    sel = (None, None, None)
    if return_selection:
        km = kmax_of(k, tau)
        sel = (torch.empty(B, Tq, Hkv, km, dtype=torch.int32, device=Q.device),
               torch.empty(B, Tq, Hkv, km, dtype=torch.float32, device=Q.device),
               torch.empty(B, Tq, Hkv, dtype=torch.int32, device=Q.device))
    _native.check(_native.lib().hsa_forward(ctypes.byref(prob), _p(Q), _p(K), _p(V), _p(W_L), _p(L),
                                            _p(sel[0]), _p(sel[1]), _p(sel[2]), _p(O), _p(ws), ws.numel(),
                                            _stream(Q)), "hsa_forward")
    if return_selection:
        return (O, L) + sel
    return O


def forward_host_bytes(prob: hsa_problem_t) -> int:
    """hsa_forward_host_bytes: device bytes that hsa_forward_host keeps its copies in."""
    n = ctypes.c_size_t(0)
    _native.check(_native.lib().hsa_forward_host_bytes(ctypes.byref(prob), ctypes.byref(n)), "hsa_forward_host_bytes")
    return int(n.value)


def forward_host(Q, K, V, W_L, S, k, tau=0.0, q_pos0=0, O=None, dev=None, ws=None, stream=None, quest=False,
                 device=None):
    """hsa_forward_host: the whole forward on HOST tensors (CPU, contiguous; page-locked ones make the
    copies asynchronous).  Q [B,Tq,H,d], K and V [B,Tcap,Hkv,d], W_L [d,d] (None with quest).  Returns
    O (a CPU tensor, written when `stream` reaches the call: synchronize before reading it).  dev and
    ws are device uint8 buffers of forward_host_bytes(prob) and workspace_size(prob) bytes, made on
    `device` (default: the current CUDA device) when None; calls in flight on different streams need
    their own.  stream: a torch.cuda.Stream (default: the device's current stream)."""
    for t in (Q, K, V, W_L, O):
        if t is not None and (t.is_cuda or not t.is_contiguous()):
            raise ValueError("forward_host takes contiguous host (CPU) tensors")
    B, Tq, H, d = Q.shape
    Tcap, Hkv = K.shape[1], K.shape[2]
    prob = _prob_from(Q, Tcap, Hkv, S, k, tau, q_pos0, _native.HSA_FLAG_QUEST if quest else 0, Tcap)
    dev_t = torch.device(device) if device is not None else torch.device("cuda", torch.cuda.current_device())
    if dev is None:
        dev = torch.empty(max(256, forward_host_bytes(prob)), dtype=torch.uint8, device=dev_t)
    if ws is None:
        ws = alloc_workspace(prob, dev_t)
    if O is None:
        O = torch.empty(Q.shape, dtype=Q.dtype, pin_memory=Q.is_pinned())
    st = stream if stream is not None else torch.cuda.current_stream(dev_t)
    _native.check(_native.lib().hsa_forward_host(ctypes.byref(prob), _p(Q), _p(K), _p(V), _p(W_L), _p(O),
                                                 _p(dev), dev.numel(), _p(ws), ws.numel(), st.cuda_stream),
                  "hsa_forward_host")
    return O


def decode_append(K, V, k_new, v_new, kv_len, S, W_L=None, L=None, quest=False) -> bool:
    """One decode step's cache update: K[:, kv_len] = k_new and V[:, kv_len] = v_new
    (k_new, v_new [B, Hkv, d]; K, V [B, Tcap, Hkv, d] with kv_len < Tcap), and, when that
    completes a chunk, its landmark into L [B, Hkv, Tcap // S, d] (quest: its Quest summary
    into L [B, Hkv, Tcap // S, 2d]).  Returns whether a chunk was completed (L, and W_L unless
    quest, are needed then)."""
    _dev(K, V, k_new, v_new, W_L, L)
    B, Tcap, Hkv, d = K.shape
    prob = make_problem(B, 1, kv_len, Hkv, Hkv, d, S, 1, kv_len, 0.0, K.dtype,
                        _native.HSA_FLAG_QUEST if quest else 0, Tcap)
    _native.check(_native.lib().hsa_decode_append(ctypes.byref(prob), _p(k_new), _p(v_new), _p(K), _p(V),
                                                   _p(W_L), _p(L), _stream(K)), "hsa_decode_append")
    return (kv_len + 1) % S == 0


def attend_partials(Q, K, V, idx, keff, S, k, tau=0.0, q_pos0=0, kv_len=None, out=None, ws=None):
    """One shard's chunk outputs for its selection, without fusion: o [B,Tq,Hkv,kmax,G,d] fp32,
    o[b,t,j,i,g] = softmax(q_{jG+g} K_{c_i}^T / sqrt(d)) V_{c_i} for i < keff (others unwritten).
    idx holds the shard's local chunk indices."""
    _dev(Q, K, V, idx, keff, out, ws)
    B, Tq, H, d = Q.shape
    Tcap, Hkv = K.shape[1], K.shape[2]
    prob = _prob_from(Q, Tcap if kv_len is None else kv_len, Hkv, S, k, tau, q_pos0, 0, Tcap)
    km = kmax_of(k, tau)
    if out is None:
        out = torch.empty(B, Tq, Hkv, km, H // Hkv, d, dtype=torch.float32, device=Q.device)
    if ws is None:
        ws = alloc_workspace(prob, Q.device)
    _native.check(_native.lib().hsa_attend_partials(ctypes.byref(prob), _p(Q), _p(K), _p(V), _p(idx), _p(keff),
                                                    _p(out), _p(ws), ws.numel(), _stream(Q)),
                  "hsa_attend_partials")
    return out


def merge_partials(score, idx, keff, o_part, S, k, tau=0.0, dtype=torch.bfloat16, O=None,
                   return_selection=False):
    """Merge of nshard shards' selections and partial outputs, concatenated shard-major
    (score, idx [P,B,Tq,Hkv,kmax] with global chunk indices, keff [P,B,Tq,Hkv],
    o_part [P,B,Tq,Hkv,kmax,G,d]) into O [B,Tq,H,d] of dtype, and with return_selection
    also the merged (idx, score, keff)."""
    _dev(score, idx, keff, o_part, O)
    P, B, Tq, Hkv, km, G, d = o_part.shape
    if km != kmax_of(k, tau):
        raise ValueError(f"partials hold {km} slots per row, but k={k}, tau={tau} merge into {kmax_of(k, tau)}")
    H = Hkv * G
    prob = make_problem(B, Tq, 0, H, Hkv, d, S, k, 0, tau, dtype)
    if O is None:
        O = torch.empty(B, Tq, H, d, dtype=dtype, device=o_part.device)
    sel = (None, None, None)
    if return_selection:
        sel = (torch.empty(B, Tq, Hkv, km, dtype=torch.int32, device=o_part.device),
               torch.empty(B, Tq, Hkv, km, dtype=torch.float32, device=o_part.device),
               torch.empty(B, Tq, Hkv, dtype=torch.int32, device=o_part.device))
    _native.check(_native.lib().hsa_merge_partials(ctypes.byref(prob), P, _p(score), _p(idx), _p(keff), _p(o_part),
                                                   _p(O), _p(sel[0]), _p(sel[1]), _p(sel[2]), _stream(o_part)),
                  "hsa_merge_partials")
    return (O,) + sel if return_selection else O


def backward_workspace_size(prob: hsa_problem_t) -> int:
    n = ctypes.c_size_t()
    _native.check(_native.lib().hsa_backward_workspace_size(ctypes.byref(prob), ctypes.byref(n)),
                  "hsa_backward_workspace_size")
    return int(n.value)


def backward(Q, K, V, W_L, L, idx, score, keff, dO, S, k, tau=0.0, q_pos0=0, kv_len=None, out=None, ws=None,
             force_simt=False):
    """Gradients (dQ, dK, dV, dW_L), fp32, of the forward with its selection (idx, score,
    keff) held fixed, for the output gradient dO [B,Tq,H,d].  L: the landmarks the forward
    scored ([B, Hkv, K.shape[1] // S, d]).  kv_len as in forward.  out: optional preallocated
    (dQ, dK, dV, dW_L); ws: optional workspace (uint8, 256-byte aligned).  force_simt runs the
    fp32 CUDA-core attention backward where the tensor-core one would apply (bf16, d 128)."""
    _dev(Q, K, V, W_L, L, idx, score, keff, dO, ws)
    B, Tq, H, d = Q.shape
    Tcap, Hkv = K.shape[1], K.shape[2]
    Tkv = Tcap if kv_len is None else kv_len
    if dO.shape != Q.shape or dO.dtype != Q.dtype:
        raise ValueError(f"dO must match Q ({tuple(Q.shape)}, {Q.dtype}); got {tuple(dO.shape)}, {dO.dtype}")
    prob = _prob_from(Q, Tkv, Hkv, S, k, tau, q_pos0, _native.HSA_FLAG_SIMT if force_simt else 0, Tcap)
    if out is None:
        f32 = dict(dtype=torch.float32, device=Q.device)
        out = (torch.empty(B, Tq, H, d, **f32), torch.empty(B, Tcap, Hkv, d, **f32),
               torch.empty(B, Tcap, Hkv, d, **f32), torch.empty(d, d, **f32))
    dQ, dK, dV, dW = out
    _dev(dQ, dK, dV, dW)
    if ws is None:
        ws = torch.empty(max(256, backward_workspace_size(prob)), dtype=torch.uint8, device=Q.device)
    _native.check(_native.lib().hsa_backward(ctypes.byref(prob), _p(Q), _p(K), _p(V), _p(W_L), _p(L), _p(idx),
                                             _p(score), _p(keff), _p(dO), _p(dQ), _p(dK), _p(dV), _p(dW), _p(ws),
                                             ws.numel(), _stream(Q)), "hsa_backward")
    return dQ, dK, dV, dW


def device_status(ws: torch.Tensor) -> None:
    """Synchronise and raise HSAError if a bounded device wait expired on this workspace."""
    _native.check(_native.lib().hsa_get_device_status(_p(ws), ws.numel(), _stream(ws)),
                  "hsa_get_device_status")
