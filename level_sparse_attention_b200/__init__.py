"""Python binding of libpsa.so, the B200 (sm_100a) Pyramid Sparse Attention
forward pass.  Argument marshalling only: every step runs in the library's CUDA
kernels; torch supplies device memory and the current stream.

The entry points mirror include/psa.h one to one (build_pyramid,
score_and_mask, attention_fwd, forward, workspace_size, check_device); the
helper ``psa_forward`` allocates the outputs and the workspace with torch.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional, Sequence, Tuple

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libpsa.so")
# the same library compiled with PSA_DEBUG (device-side work-list bounds checks)
DEBUG_LIB_PATH = os.path.join(_HERE, "libpsa_debug.so")

F32, BF16 = 0, 1
_STATUS = {0: "ok", 1: "invalid argument", 2: "unsupported configuration", 3: "misaligned",
           4: "workspace too small", 5: "CUDA error", 6: "device timeout",
           7: "level map corrected", 8: "work list out of bounds (debug build)"}


class PSAError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} (status {status})")


class Params(ctypes.Structure):
    """Mirror of psa_params_t."""
    _fields_ = [("B", ctypes.c_int), ("Hq", ctypes.c_int), ("Hkv", ctypes.c_int),
                ("N", ctypes.c_int), ("d", ctypes.c_int), ("q_blk", ctypes.c_int),
                ("kv_blk", ctypes.c_int), ("n_levels", ctypes.c_int),
                ("pool", ctypes.c_int * 4), ("tau", ctypes.c_float * 4),
                ("causal", ctypes.c_int), ("forced_prefix_tokens", ctypes.c_int),
                ("scale", ctypes.c_float), ("dtype", ctypes.c_int), ("assign", ctypes.c_int),
                ("sim_threshold", ctypes.c_float)]


_lib = None
_debug_lib = None


def lib() -> ctypes.CDLL:
    """Load libpsa.so (built by ``python -m level_sparse_attention_b200.build``).
    There is no fallback: a missing library is an error."""
    global _lib
    if _lib is None:
        _lib = _load(LIB_PATH)
    return _lib


def debug_lib() -> ctypes.CDLL:
    """Load libpsa_debug.so, the PSA_DEBUG build of the same sources (built by
    ``python -m level_sparse_attention_b200.build --debug``)."""
    global _debug_lib
    if _debug_lib is None:
        _debug_lib = _load(DEBUG_LIB_PATH)
    return _debug_lib


def _load(path: str) -> ctypes.CDLL:
    if True:
        if not os.path.exists(path):
            raise ImportError(f"{path} is missing; run python -m level_sparse_attention_b200.build")
        L = ctypes.CDLL(path)
        P, vp, sz = ctypes.POINTER(Params), ctypes.c_void_p, ctypes.c_size_t
        sigs = {
            "psa_workspace_size": (sz, [P]),
            "psa_build_pyramid": (ctypes.c_int, [P, vp, vp, vp, sz, vp]),
            "psa_score_and_mask": (ctypes.c_int, [P, vp, vp, sz, vp, vp, vp]),
            "psa_attention_fwd": (ctypes.c_int, [P, vp, vp, vp, vp, sz, vp, vp, vp, vp]),
            "psa_forward": (ctypes.c_int, [P, vp, vp, vp, vp, vp, vp, vp, sz, vp]),
            "psa_check_device": (ctypes.c_int, [P, vp, sz, vp]),
            "psa_forward_noalloc": (ctypes.c_int, [P, vp, vp, vp, vp, vp, vp, vp]),
            "psa_status_string": (ctypes.c_char_p, [ctypes.c_int]),
            "psa_selftest_wait_timeout": (ctypes.c_int, [P, vp, sz, ctypes.c_uint64, vp]),
            "psa_forward_host": (ctypes.c_int, [P, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz,
                                                ctypes.c_int, vp, vp, vp]),
            "psa_backward_workspace_size": (sz, [P]),
            "psa_debug_build": (ctypes.c_int, []),
            "psa_backward": (ctypes.c_int, [P, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp, sz, vp, vp,
                                            vp, vp]),
        }
        for name, (res, args) in sigs.items():
            fn = getattr(L, name)
            fn.restype, fn.argtypes = res, args
    return L


EXPORTED = ("psa_workspace_size", "psa_build_pyramid", "psa_score_and_mask",
            "psa_attention_fwd", "psa_forward", "psa_check_device", "psa_status_string",
            "psa_forward_noalloc", "psa_selftest_wait_timeout", "psa_forward_host",
            "psa_backward_workspace_size", "psa_backward", "psa_debug_build")


def status_string(status: int) -> str:
    try:
        return lib().psa_status_string(status).decode()
    except ImportError:
        return _STATUS.get(status, "unknown")


ASSIGN_THRESHOLD, ASSIGN_QUANTILE = 0, 1


def make_params(B: int, Hq: int, Hkv: int, N: int, d: int, q_blk: int = 128, kv_blk: int = 64,
                tau: Sequence[float] = (0.6, 0.8, 0.9, 0.97), causal: bool = False,
                forced_prefix_tokens: int = 0, scale: float = 0.0,
                dtype: torch.dtype = torch.bfloat16, assign: int = ASSIGN_THRESHOLD,
                sim_threshold: float = -1.0) -> Params:
    """psa_params_t for the arguments; ``sim_threshold`` > -1 turns on the
    cosine-similarity constraint on the pyramid levels."""
    p = Params()
    p.B, p.Hq, p.Hkv, p.N, p.d = B, Hq, Hkv, N, d
    p.q_blk, p.kv_blk, p.n_levels = q_blk, kv_blk, 4
    for i in range(4):
        p.pool[i] = 1 << i
        p.tau[i] = float(tau[i])
    p.causal, p.forced_prefix_tokens, p.scale = int(bool(causal)), forced_prefix_tokens, scale
    p.dtype = BF16 if dtype == torch.bfloat16 else F32
    p.assign = int(assign)
    p.sim_threshold = float(sim_threshold)
    return p


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _check(status: int, where: str) -> None:
    if status != 0:
        raise PSAError(status, where)


def workspace_size(p: Params) -> int:
    return int(lib().psa_workspace_size(ctypes.byref(p)))


def new_workspace(p: Params, device="cuda") -> torch.Tensor:
    n = workspace_size(p)
    if n == 0:
        raise PSAError(1, "psa_workspace_size")
    return torch.zeros(n, dtype=torch.uint8, device=device)


def build_pyramid(p: Params, K: torch.Tensor, V: torch.Tensor, ws: torch.Tensor, stream=None):
    _check(lib().psa_build_pyramid(ctypes.byref(p), _ptr(K), _ptr(V), _ptr(ws), ws.numel(),
                                   _stream(stream)), "psa_build_pyramid")


def score_and_mask(p: Params, Q: torch.Tensor, ws: torch.Tensor,
                   level_map: Optional[torch.Tensor] = None,
                   block_mass: Optional[torch.Tensor] = None, stream=None):
    _check(lib().psa_score_and_mask(ctypes.byref(p), _ptr(Q), _ptr(ws), ws.numel(),
                                    _ptr(level_map), _ptr(block_mass), _stream(stream)),
           "psa_score_and_mask")


def attention_fwd(p: Params, Q, K, V, ws, O, lse=None, level_map=None, stream=None):
    _check(lib().psa_attention_fwd(ctypes.byref(p), _ptr(Q), _ptr(K), _ptr(V), _ptr(ws),
                                   ws.numel(), _ptr(level_map), _ptr(O), _ptr(lse),
                                   _stream(stream)), "psa_attention_fwd")


def forward(p: Params, Q, K, V, O, ws, lse=None, level_map=None, stream=None):
    _check(lib().psa_forward(ctypes.byref(p), _ptr(Q), _ptr(K), _ptr(V), _ptr(O), _ptr(lse),
                             _ptr(level_map), _ptr(ws), ws.numel(), _stream(stream)),
           "psa_forward")


def host_groups(p: Params) -> int:
    """A head-group count for forward_host: up to 8 groups of whole GQA groups,
    or the KV heads' query heads split evenly when there are fewer KV heads."""
    if p.Hkv >= 8:
        return 8
    grp = p.Hq // p.Hkv
    per = max(1, min(grp, 8 // p.Hkv))
    return p.Hkv * per


def forward_host(p: Params, hQ, hK, hV, hO, Q, K, V, O, ws, h2d_stream, d2h_stream,
                 hlse=None, lse=None, groups: Optional[int] = None, stream=None):
    """psa_forward_host: the forward pass from (pinned) host tensors hQ, hK,
    hV into hO (and hlse), with per-head-group copies on the two copy streams
    pipelined behind the kernels on `stream`.  Q, K, V, O (and lse): device
    buffers for the whole problem."""
    g = host_groups(p) if groups is None else groups
    _check(lib().psa_forward_host(ctypes.byref(p), _ptr(hQ), _ptr(hK), _ptr(hV), _ptr(hO),
                                  _ptr(hlse), _ptr(Q), _ptr(K), _ptr(V), _ptr(O), _ptr(lse),
                                  _ptr(ws), ws.numel(), int(g), _stream(stream),
                                  _stream(h2d_stream), _stream(d2h_stream)), "psa_forward_host")


def backward_workspace_size(p: Params) -> int:
    return int(lib().psa_backward_workspace_size(ctypes.byref(p)))


def new_backward_workspace(p: Params, device="cuda") -> torch.Tensor:
    n = backward_workspace_size(p)
    if n == 0:
        raise PSAError(1, "psa_backward_workspace_size")
    return torch.empty(n, dtype=torch.uint8, device=device)


def backward(p: Params, Q, K, V, O, lse, dO, ws, bws, dQ, dK, dV, level_map=None, stream=None):
    """psa_backward: dQ, dK, dV of the pyramid attention with the map held
    fixed.  ``ws`` is the forward workspace (its work list is used unless
    ``level_map`` is given); ``bws`` the backward scratch."""
    _check(lib().psa_backward(ctypes.byref(p), _ptr(Q), _ptr(K), _ptr(V), _ptr(O), _ptr(lse),
                              _ptr(dO), _ptr(level_map), _ptr(ws), ws.numel(), _ptr(bws),
                              bws.numel(), _ptr(dQ), _ptr(dK), _ptr(dV), _stream(stream)),
           "psa_backward")


def forward_noalloc(p: Params, Q, K, V, O, lse=None, level_map=None, stream=None):
    """psa_forward without a workspace: the library's own 32 MiB device array
    serves as scratch (no allocation; calls must not overlap on the GPU)."""
    _check(lib().psa_forward_noalloc(ctypes.byref(p), _ptr(Q), _ptr(K), _ptr(V), _ptr(O),
                                     _ptr(lse), _ptr(level_map), _stream(stream)),
           "psa_forward_noalloc")


def check_device(p: Params, ws: torch.Tensor, stream=None):
    _check(lib().psa_check_device(ctypes.byref(p), _ptr(ws), ws.numel(), _stream(stream)),
           "psa_check_device")


def selftest_wait_timeout(p: Params, ws: torch.Tensor, limit_ns: int, stream=None):
    """Enqueue the failure-path self-test: a bounded wait that runs out after
    ``limit_ns`` and records a timeout in the workspace's error word, which
    the next check_device reports as PSA_ERR_DEVICE_TIMEOUT."""
    _check(lib().psa_selftest_wait_timeout(ctypes.byref(p), _ptr(ws), ws.numel(), int(limit_ns),
                                           _stream(stream)), "psa_selftest_wait_timeout")


def map_shape(p: Params) -> Tuple[int, int, int, int]:
    return (p.B, p.Hq, -(-p.N // p.q_blk), -(-p.N // p.kv_blk))


def psa_forward(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, q_blk: int = 128,
                kv_blk: int = 64, tau: Sequence[float] = (0.6, 0.8, 0.9, 0.97),
                causal: bool = False, forced_prefix_tokens: int = 0, scale: float = 0.0,
                return_map: bool = False, workspace: Optional[torch.Tensor] = None,
                assign: int = ASSIGN_THRESHOLD):
    """PSA forward on CUDA tensors q [B, Hq, N, d], k/v [B, Hkv, N, d]
    (contiguous, bf16 or fp32).  Returns (O, lse) or (O, lse, level_map)."""
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    p = make_params(B, Hq, Hkv, N, d, q_blk, kv_blk, tau, causal, forced_prefix_tokens, scale,
                    q.dtype, assign)
    ws = workspace if workspace is not None else new_workspace(p, q.device)
    O = torch.empty_like(q)
    lse = torch.empty((B, Hq, N), dtype=torch.float32, device=q.device)
    lm = torch.empty(map_shape(p), dtype=torch.int8, device=q.device) if return_map else None
    forward(p, q.contiguous(), k.contiguous(), v.contiguous(), O, ws, lse, lm)
    return (O, lse, lm) if return_map else (O, lse)


class _PSAFunction(torch.autograd.Function):
    """psa_forward in the forward pass; psa_backward, on the map the forward
    pass chose (held fixed), in the backward pass."""

    @staticmethod
    def forward(ctx, q, k, v, q_blk, kv_blk, tau, causal, forced_prefix_tokens, scale, assign,
                sim_threshold):
        B, Hq, N, d = q.shape
        p = make_params(B, Hq, k.shape[1], N, d, q_blk, kv_blk, tau, causal,
                        forced_prefix_tokens, scale, q.dtype, assign, sim_threshold)
        q, k, v = q.contiguous(), k.contiguous(), v.contiguous()
        ws = new_workspace(p, q.device)
        O = torch.empty_like(q)
        lse = torch.empty((B, Hq, N), dtype=torch.float32, device=q.device)
        lm = torch.empty(map_shape(p), dtype=torch.int8, device=q.device)
        forward(p, q, k, v, O, ws, lse, lm)
        ctx.save_for_backward(q, k, v, O, lse, lm)
        ctx.p = p
        return O

    @staticmethod
    def backward(ctx, dO):
        q, k, v, O, lse, lm = ctx.saved_tensors
        p = ctx.p
        ws = new_workspace(p, q.device)
        bws = new_backward_workspace(p, q.device)
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        backward(p, q, k, v, O, lse, dO.contiguous(), ws, bws, dq, dk, dv, level_map=lm)
        return dq, dk, dv, None, None, None, None, None, None, None, None


def psa_attention(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, q_blk: int = 128,
                  kv_blk: int = 64, tau: Sequence[float] = (0.6, 0.8, 0.9, 0.97),
                  causal: bool = False, forced_prefix_tokens: int = 0, scale: float = 0.0,
                  assign: int = ASSIGN_THRESHOLD, sim_threshold: float = -1.0) -> torch.Tensor:
    """PSA attention O [B, Hq, N, d] of CUDA tensors q [B, Hq, N, d], k/v
    [B, Hkv, N, d] (bf16 or fp32), differentiable: the backward pass runs
    psa_backward on the level map the forward pass chose."""
    return _PSAFunction.apply(q, k, v, q_blk, kv_blk, tuple(float(t) for t in tau), causal,
                              forced_prefix_tokens, scale, assign, sim_threshold)


def head_shard(Hq: int, Hkv: int, rank: int, world: int) -> Tuple[int, int, int, int]:
    """The heads rank `rank` of `world` takes of one problem: query heads
    [q0, q1) and the KV heads [kv0, kv1) they read (query head h reads KV
    head h // (Hq / Hkv)).  Every (batch, head) of the forward pass is
    independent, so the shards need no exchange.  With at least as many KV
    heads as ranks, ranks take whole groups of query heads sharing a KV head
    (as even a split of the KV heads as possible); with fewer, each KV head's
    group is split among world / Hkv ranks, so a shard never straddles two
    groups.  Either way the shard's own grouping matches the global one.
    Returns (q0, q1, kv0, kv1); raises ValueError for a split it cannot make."""
    if Hq <= 0 or Hkv <= 0 or Hq % Hkv or not 0 <= rank < world:
        raise ValueError("bad head counts or rank")
    G = Hq // Hkv
    if Hkv >= world:
        kv0, kv1 = rank * Hkv // world, (rank + 1) * Hkv // world
        return kv0 * G, kv1 * G, kv0, kv1
    if world % Hkv:
        raise ValueError(f"{world} ranks cannot split {Hkv} KV heads' groups evenly")
    per = world // Hkv                       # ranks per KV head
    if per > G:
        raise ValueError(f"{per} ranks per KV head exceed its {G} query heads")
    kv = rank // per
    i = rank % per
    q0, q1 = kv * G + i * G // per, kv * G + (i + 1) * G // per
    return q0, q1, kv, kv + 1


def psa_forward_heads(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, out: torch.Tensor,
                      lse: Optional[torch.Tensor], p: Params, rank: int, world: int,
                      workspace: Optional[torch.Tensor] = None, stream=None) -> Params:
    """This rank's share of one forward pass: the heads of head_shard for
    every batch element, written into the matching heads of `out` (and
    `lse`).  q, k, v, out: [B, H, N, d] contiguous device tensors of the full
    problem described by `p`; every rank may hold them whole (they are read
    and written only at its heads).  One psa_forward call per batch element on
    the contiguous head slices.  Returns the per-call params."""
    q0, q1, kv0, kv1 = head_shard(p.Hq, p.Hkv, rank, world)
    sp = Params.from_buffer_copy(p)
    sp.B, sp.Hq, sp.Hkv = 1, q1 - q0, kv1 - kv0
    if sp.Hq == 0:
        return sp
    ws = workspace if workspace is not None else new_workspace(sp, q.device)
    for b in range(p.B):
        forward(sp, q[b, q0:q1], k[b, kv0:kv1], v[b, kv0:kv1], out[b, q0:q1], ws,
                None if lse is None else lse[b, q0:q1], None, stream)
    return sp


def workspace_layout(p: Params) -> dict:
    """Byte offsets of the workspace regions (mirrors the library's layout),
    for inspecting intermediate results."""
    a256 = lambda x: (x + 255) & ~255
    es = 2 if p.dtype == BF16 else 4
    Nq, Nk = -(-p.N // p.q_blk), -(-p.N // p.kv_blk)
    rows = [-(-p.N // (1 << l)) for l in range(4)]
    off, L = 256, {"err": 0, "rows": rows, "Nq": Nq, "Nk": Nk, "kp": [0] * 4, "vp": [0] * 4}
    for l in range(1, 4):
        n = a256(p.B * p.Hkv * rows[l] * p.d * es)
        L["kp"][l], off = off, off + n
        L["vp"][l], off = off, off + n
    # fp32 GEMM operands as tf32 head + exact tail pairs
    k3 = a256(p.B * p.Hkv * rows[3] * p.d * 4)
    L["k3h"], off = off, off + k3
    L["k3l"], off = off, off + k3
    rq = p.B * p.Hq * Nq
    L["qmh"], off = off, off + a256(rq * p.d * 4)
    L["qml"], off = off, off + a256(rq * p.d * 4)
    L["zlog"], off = off, off + a256(rq * Nk * 4)
    L["map"], off = off, off + a256(rq * Nk)
    L["maxlev"], off = off, off + a256(p.B * p.Hkv * Nk)
    L["counts"], off = off, off + a256(rq * 16)
    L["list"], off = off, off + a256(rq * Nk * 4)
    L["total"] = off
    return L


def workspace_view(ws: torch.Tensor, offset: int, shape, dtype: torch.dtype) -> torch.Tensor:
    n = 1
    for s in shape:
        n *= s
    nbytes = n * torch.tensor([], dtype=dtype).element_size()
    return ws[offset:offset + nbytes].view(dtype).view(*shape)
