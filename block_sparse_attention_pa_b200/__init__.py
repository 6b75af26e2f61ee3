"""Python binding of libpa.so: ProxyAttn-style block-sparse prefill attention
on B200 (sm_100a).

Argument marshalling only: every step of the path runs in the CUDA kernels of
``libpa.so`` behind its C ABI (``include/pa.h``).  PyTorch provides device
memory and the current stream.  There is no CPU fallback: if the library is
missing or a tensor is not on a CUDA device, the call raises.

Functions mirror the C entry points:
  pool_heads, block_scores, build_mask, block_sparse_attn, prefill,
  workspace_size, device_status.
Tensors use the [B, N, heads, d] layout (any strides with d contiguous).
"""
from __future__ import annotations

import ctypes
import math
import os
from dataclasses import dataclass

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libpa.so")

DYNAMIC, FIXED_FRACTION, ALL = 0, 1, 2

STATUS = {0: "PA_OK", 1: "PA_ERR_INVALID_ARG", 2: "PA_ERR_UNSUPPORTED", 3: "PA_ERR_WORKSPACE",
          4: "PA_ERR_CUDA", 5: "PA_ERR_TIMEOUT", 6: "PA_ERR_DEVICE_BOUNDS", 7: "PA_ERR_DEVICE_NONFINITE"}

# Every entry point declared in include/pa.h.
ENTRY_POINTS = ("pa_workspace_size", "pa_pool_heads", "pa_block_scores", "pa_build_mask",
                "pa_block_sparse_attn", "pa_prefill", "pa_get_device_status", "pa_status_string",
                "pa_last_error", "pa_abi_version", "pa_build_mask_noalloc", "pa_selftest_wait_timeout",
                "pa_pool_heads_strided", "pa_block_scores_strided", "pa_block_sparse_attn_skip", "pa_xattn_workspace_size", "pa_xattn_mask",
                "pa_workspace_size_varlen", "pa_prefill_varlen")

XATTN_STRIDES = (4, 8, 16)
SCORE_STRIDES = (1, 2, 4, 8)


class PaError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"{STATUS.get(code, code)}: {msg}")
        self.code = code


class Shape(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("seqlen", ctypes.c_int32), ("num_q_heads", ctypes.c_int32),
                ("num_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32), ("block", ctypes.c_int32),
                ("num_groups", ctypes.c_int32), ("non_causal", ctypes.c_int32)]


class Strides(ctypes.Structure):
    _fields_ = [("b", ctypes.c_int64), ("s", ctypes.c_int64), ("h", ctypes.c_int64)]


class Budget(ctypes.Structure):
    _fields_ = [("mode", ctypes.c_int32), ("gamma", ctypes.c_float), ("frac_permille", ctypes.c_int32),
                ("score_stride", ctypes.c_int32), ("skip_threshold", ctypes.c_float)]


class MaskBufs(ctypes.Structure):
    _fields_ = [("rank", ctypes.c_void_p), ("cnt", ctypes.c_void_p), ("budget", ctypes.c_void_p),
                ("mass", ctypes.c_void_p)]


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded libpa.so; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m block_sparse_attention_pa_b200.build` (nvcc, sm_100a)")
        L = ctypes.CDLL(LIB_PATH)
        vp, P = ctypes.c_void_p, ctypes.POINTER
        st = Strides
        L.pa_workspace_size.restype = ctypes.c_size_t
        L.pa_workspace_size.argtypes = [P(Shape), P(Budget)]
        L.pa_pool_heads.argtypes = [P(Shape), vp, st, vp, st, vp, vp, vp]
        L.pa_block_scores.argtypes = [P(Shape), vp, vp, vp, vp]
        L.pa_pool_heads_strided.argtypes = [P(Shape), ctypes.c_int32, vp, st, vp, st, vp, vp, vp]
        L.pa_block_scores_strided.argtypes = [P(Shape), ctypes.c_int32, vp, vp, vp, vp]
        L.pa_build_mask.argtypes = [P(Shape), P(Budget), vp, vp, st, vp, st, P(MaskBufs), vp, ctypes.c_size_t, vp]
        L.pa_block_sparse_attn.argtypes = [P(Shape), vp, st, vp, st, vp, st, vp, vp, ctypes.c_float, vp, st, vp, vp]
        L.pa_block_sparse_attn_skip.argtypes = [P(Shape), vp, st, vp, st, vp, st, vp, vp, ctypes.c_float,
                                                ctypes.c_float, vp, st, vp, vp, vp]
        L.pa_prefill.argtypes = [P(Shape), P(Budget), vp, st, vp, st, vp, st, vp, st, P(MaskBufs), vp,
                                 ctypes.c_size_t, vp]
        L.pa_get_device_status.argtypes = [vp, ctypes.c_int]
        L.pa_workspace_size_varlen.restype = ctypes.c_size_t
        L.pa_workspace_size_varlen.argtypes = [P(Shape), P(Budget), ctypes.c_int32, vp]
        L.pa_prefill_varlen.argtypes = [P(Shape), P(Budget), ctypes.c_int32, vp, vp, st, vp, st, vp, st, vp, st,
                                        P(MaskBufs), vp, ctypes.c_size_t, vp]
        L.pa_xattn_workspace_size.restype = ctypes.c_size_t
        L.pa_xattn_workspace_size.argtypes = [P(Shape), ctypes.c_int32]
        L.pa_xattn_mask.argtypes = [P(Shape), ctypes.c_int32, ctypes.c_float, vp, st, vp, st, vp, vp, vp, vp,
                                    ctypes.c_size_t, vp]
        L.pa_build_mask_noalloc.argtypes = [P(Shape), P(Budget), vp, vp, st, vp, st, P(MaskBufs), vp]
        L.pa_selftest_wait_timeout.argtypes = [ctypes.c_uint32, vp]
        L.pa_status_string.restype = ctypes.c_char_p
        L.pa_status_string.argtypes = [ctypes.c_int]
        L.pa_last_error.restype = ctypes.c_char_p
        L.pa_abi_version.restype = ctypes.c_int32
        for name in ("pa_pool_heads", "pa_block_scores", "pa_build_mask", "pa_block_sparse_attn", "pa_prefill",
                     "pa_get_device_status", "pa_selftest_wait_timeout", "pa_pool_heads_strided",
                     "pa_block_scores_strided", "pa_block_sparse_attn_skip", "pa_xattn_mask", "pa_prefill_varlen",
                     "pa_build_mask_noalloc"):
            getattr(L, name).restype = ctypes.c_int
        _lib = L
    return _lib


def _check(code: int):
    if code != 0:
        msg = lib().pa_last_error().decode() or lib().pa_status_string(code).decode()
        raise PaError(code, msg)


def _stream(device) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _strides(t: torch.Tensor) -> Strides:
    return Strides(t.stride(0), t.stride(1), t.stride(2))


def _cuda_bf16(t: torch.Tensor, name: str):
    if not (isinstance(t, torch.Tensor) and t.is_cuda):
        raise ValueError(f"{name} must be a CUDA tensor (there is no CPU path)")
    if t.dtype != torch.bfloat16 or t.dim() != 4 or t.stride(3) != 1:
        raise ValueError(f"{name} must be bf16 [B, N, heads, d] with a contiguous last dimension")


def make_shape(q: torch.Tensor, k: torch.Tensor, num_groups: int, causal: bool = True) -> Shape:
    B, N, H, d = q.shape
    return Shape(B, N, H, k.shape[2], d, 128, num_groups, 0 if causal else 1)


def rows_total(nb: int, causal: bool = True) -> int:
    """Entries of one (b, g) set of block scores or ranked lists."""
    return nb * (nb + 1) // 2 if causal else nb * nb


def make_budget(mode: int = DYNAMIC, gamma: float = 0.95, frac_permille: int = 0, score_stride: int = 1,
                skip_threshold: float = 0.0) -> Budget:
    return Budget(mode, gamma, frac_permille, score_stride, skip_threshold)


def workspace_size(shape: Shape, budget: Budget) -> int:
    return int(lib().pa_workspace_size(ctypes.byref(shape), ctypes.byref(budget)))


@dataclass
class Mask:
    """Device mask buffers (see pa_mask in include/pa.h)."""
    rank: torch.Tensor     # int32 [B, G, T]
    cnt: torch.Tensor      # int32 [B, H, nb]
    budget: torch.Tensor   # int32 [B, H]
    mass: torch.Tensor | None  # float32 [B, H, nb] (dynamic mode)

    @staticmethod
    def empty(shape: Shape, device, with_mass: bool) -> "Mask":
        nb = shape.seqlen // 128
        T = rows_total(nb, not shape.non_causal)
        i32 = dict(device=device, dtype=torch.int32)
        return Mask(torch.empty(shape.batch, shape.num_groups, T, **i32),
                    torch.empty(shape.batch, shape.num_q_heads, nb, **i32),
                    torch.empty(shape.batch, shape.num_q_heads, **i32),
                    torch.empty(shape.batch, shape.num_q_heads, nb, device=device, dtype=torch.float32)
                    if with_mass else None)

    def bufs(self) -> MaskBufs:
        return MaskBufs(self.rank.data_ptr(), self.cnt.data_ptr(), self.budget.data_ptr(),
                        self.mass.data_ptr() if self.mass is not None else None)


def pool_heads(q: torch.Tensor, k: torch.Tensor, num_groups: int, score_stride: int = 1, causal: bool = True):
    """pa_pool_heads (score_stride 1) or pa_pool_heads_strided -> (q_proxy,
    k_proxy): q_proxy bf16 [B, G, N/score_stride, d], k_proxy [B, G, N, d]."""
    _cuda_bf16(q, "q")
    _cuda_bf16(k, "k")
    shape = make_shape(q, k, num_groups, causal)
    B, N, H, d = q.shape
    r = int(score_stride)
    qp = torch.empty(B, num_groups, N // r if r in SCORE_STRIDES else N, d, device=q.device, dtype=torch.bfloat16)
    kp = torch.empty(B, num_groups, N, d, device=q.device, dtype=torch.bfloat16)
    if r == 1:
        _check(lib().pa_pool_heads(ctypes.byref(shape), q.data_ptr(), _strides(q), k.data_ptr(), _strides(k),
                                   qp.data_ptr(), kp.data_ptr(), _stream(q.device)))
    else:
        _check(lib().pa_pool_heads_strided(ctypes.byref(shape), r, q.data_ptr(), _strides(q), k.data_ptr(),
                                           _strides(k), qp.data_ptr(), kp.data_ptr(), _stream(q.device)))
    return qp, kp


def block_scores(q_proxy: torch.Tensor, k_proxy: torch.Tensor, num_q_heads: int = 1, num_kv_heads: int = 1,
                 score_stride: int = 1, causal: bool = True):
    """pa_block_scores (score_stride 1) or pa_block_scores_strided -> fp32
    [B, G, T].  k_proxy is [B, G, N, d]; q_proxy [B, G, N/score_stride, d]."""
    for t, n in ((q_proxy, "q_proxy"), (k_proxy, "k_proxy")):
        if not (t.is_cuda and t.dtype == torch.bfloat16 and t.is_contiguous() and t.dim() == 4):
            raise ValueError(f"{n} must be a contiguous bf16 CUDA tensor [B, G, N, d]")
    B, G, N, d = k_proxy.shape
    r = int(score_stride)
    if tuple(q_proxy.shape) != (B, G, N // max(r, 1), d):
        raise ValueError(f"q_proxy must be [B, G, N/{r}, d] = {(B, G, N // max(r, 1), d)}, got {tuple(q_proxy.shape)}")
    H = max(num_q_heads, G)
    shape = Shape(B, N, H, min(num_kv_heads, H), d, 128, G, 0 if causal else 1)
    nb = N // 128
    scores = torch.empty(B, G, rows_total(nb, causal), device=q_proxy.device, dtype=torch.float32)
    if r == 1:
        _check(lib().pa_block_scores(ctypes.byref(shape), q_proxy.data_ptr(), k_proxy.data_ptr(), scores.data_ptr(),
                                     _stream(q_proxy.device)))
    else:
        _check(lib().pa_block_scores_strided(ctypes.byref(shape), r, q_proxy.data_ptr(), k_proxy.data_ptr(),
                                             scores.data_ptr(), _stream(q_proxy.device)))
    return scores


def build_mask(scores: torch.Tensor, q: torch.Tensor, k: torch.Tensor, num_groups: int, mode: int = DYNAMIC,
               gamma: float = 0.95, frac_permille: int = 0, workspace: torch.Tensor | None = None,
               causal: bool = True) -> Mask:
    """pa_build_mask -> Mask."""
    _cuda_bf16(q, "q")
    _cuda_bf16(k, "k")
    shape = make_shape(q, k, num_groups, causal)
    budget = make_budget(mode, gamma, frac_permille)
    mask = Mask.empty(shape, q.device, mode == DYNAMIC)
    if workspace is None:
        workspace = torch.empty(max(workspace_size(shape, budget), 256), device=q.device, dtype=torch.uint8)
    bufs = mask.bufs()
    _check(lib().pa_build_mask(ctypes.byref(shape), ctypes.byref(budget), scores.data_ptr(), q.data_ptr(),
                               _strides(q), k.data_ptr(), _strides(k), ctypes.byref(bufs), workspace.data_ptr(),
                               workspace.numel(), _stream(q.device)))
    return mask


def xattn_mask(q: torch.Tensor, k: torch.Tensor, stride: int = 8, tau: float = 0.9,
               workspace: torch.Tensor | None = None, causal: bool = True):
    """pa_xattn_mask -> (rank int32 [B, H, T], cnt int32 [B, H, nb], mass fp32
    [B, H, T]); feed rank/cnt to block_sparse_attn with num_groups = H."""
    _cuda_bf16(q, "q")
    _cuda_bf16(k, "k")
    B, N, H, d = q.shape
    shape = make_shape(q, k, H, causal)
    nb = N // 128
    T = rows_total(nb, causal)
    i32 = dict(device=q.device, dtype=torch.int32)
    rank = torch.empty(B, H, T, **i32)
    cnt = torch.empty(B, H, nb, **i32)
    mass = torch.empty(B, H, T, device=q.device, dtype=torch.float32)
    if workspace is None:
        need = int(lib().pa_xattn_workspace_size(ctypes.byref(shape), int(stride)))
        workspace = torch.empty(max(need, 256), device=q.device, dtype=torch.uint8)
    _check(lib().pa_xattn_mask(ctypes.byref(shape), int(stride), float(tau), q.data_ptr(), _strides(q), k.data_ptr(),
                               _strides(k), rank.data_ptr(), cnt.data_ptr(), mass.data_ptr(), workspace.data_ptr(),
                               workspace.numel(), _stream(q.device)))
    return rank, cnt, mass


def block_sparse_attn(q, k, v, rank, cnt, num_groups: int, softmax_scale: float | None = None,
                      out: torch.Tensor | None = None, return_lse: bool = False, skip_threshold: float = 0.0,
                      return_skipped: bool = False, causal: bool = True):
    """pa_block_sparse_attn (skip_threshold 0) or pa_block_sparse_attn_skip ->
    o (bf16 [B, N, H, d]) [, lse fp32 [B, H, N]] [, skipped uint8 [B, H, T]]."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _cuda_bf16(t, n)
    shape = make_shape(q, k, num_groups, causal)
    B, N, H, d = q.shape
    nb = N // 128
    scale = 1.0 / math.sqrt(d) if softmax_scale is None else softmax_scale
    o = torch.empty_like(q, memory_format=torch.contiguous_format) if out is None else out
    lse = torch.empty(B, H, N, device=q.device, dtype=torch.float32) if return_lse else None
    skipped = torch.zeros(B, H, rows_total(nb, causal), device=q.device, dtype=torch.uint8) if return_skipped else None
    lse_p = lse.data_ptr() if lse is not None else None
    if skip_threshold == 0.0 and not return_skipped:
        _check(lib().pa_block_sparse_attn(ctypes.byref(shape), q.data_ptr(), _strides(q), k.data_ptr(), _strides(k),
                                          v.data_ptr(), _strides(v), rank.data_ptr(), cnt.data_ptr(), scale,
                                          o.data_ptr(), _strides(o), lse_p, _stream(q.device)))
    else:
        _check(lib().pa_block_sparse_attn_skip(ctypes.byref(shape), q.data_ptr(), _strides(q), k.data_ptr(),
                                               _strides(k), v.data_ptr(), _strides(v), rank.data_ptr(),
                                               cnt.data_ptr(), scale, skip_threshold, o.data_ptr(), _strides(o),
                                               lse_p, skipped.data_ptr() if skipped is not None else None,
                                               _stream(q.device)))
    res = (o,) + ((lse,) if return_lse else ()) + ((skipped,) if return_skipped else ())
    return res if len(res) > 1 else o


class Prefill:
    """A reusable pa_prefill call: workspace and mask buffers allocated once."""

    def __init__(self, q, k, v, num_groups: int, mode: int = DYNAMIC, gamma: float = 0.95, frac_permille: int = 0,
                 score_stride: int = 1, skip_threshold: float = 0.0, causal: bool = True):
        for t, n in ((q, "q"), (k, "k"), (v, "v")):
            _cuda_bf16(t, n)
        self.shape = make_shape(q, k, num_groups, causal)
        self.budget = make_budget(mode, gamma, frac_permille, score_stride, skip_threshold)
        self.mask = Mask.empty(self.shape, q.device, mode == DYNAMIC)
        self.ws = torch.empty(workspace_size(self.shape, self.budget), device=q.device, dtype=torch.uint8)
        self._bufs = self.mask.bufs()

    def __call__(self, q, k, v, out):
        _check(lib().pa_prefill(ctypes.byref(self.shape), ctypes.byref(self.budget), q.data_ptr(), _strides(q),
                                k.data_ptr(), _strides(k), v.data_ptr(), _strides(v), out.data_ptr(),
                                _strides(out), ctypes.byref(self._bufs), self.ws.data_ptr(), self.ws.numel(),
                                _stream(q.device)))
        return out


def prefill(q, k, v, num_groups: int, mode: int = DYNAMIC, gamma: float = 0.95, frac_permille: int = 0,
            score_stride: int = 1, skip_threshold: float = 0.0, causal: bool = True):
    """pa_prefill -> (o, Mask)."""
    call = Prefill(q, k, v, num_groups, mode, gamma, frac_permille, score_stride, skip_threshold, causal)
    o = torch.empty_like(q, memory_format=torch.contiguous_format)
    call(q, k, v, o)
    return o, call.mask


def device_status(clear: bool = True, device=None) -> int:
    """pa_get_device_status: syncs the current stream; 0 if no kernel recorded a problem."""
    return int(lib().pa_get_device_status(_stream(device), 1 if clear else 0))


def selftest_wait_timeout(timeout_us: int = 1000, device=None) -> None:
    """pa_selftest_wait_timeout: a bounded device wait that is made to run out."""
    _check(lib().pa_selftest_wait_timeout(int(timeout_us), _stream(device)))


@dataclass
class VarlenMask:
    """Packed mask buffers of pa_prefill_varlen and each sequence's views."""
    rank: torch.Tensor     # int32, sequences' [G, T_s] blocks back to back
    cnt: torch.Tensor      # int32, sequences' [H, nb_s] blocks back to back
    budget: torch.Tensor   # int32 [num_seqs, H]
    mass: torch.Tensor | None
    views: list            # per sequence: Mask of views into the packed buffers


def prefill_varlen(q, k, v, cu_seqlens, num_groups: int, mode: int = DYNAMIC, gamma: float = 0.95,
                   frac_permille: int = 0, score_stride: int = 1, skip_threshold: float = 0.0, causal: bool = True):
    """pa_prefill_varlen: q, k, v are [1, total, heads, d]; cu_seqlens a list of
    num_seqs+1 token offsets -> (o, VarlenMask)."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _cuda_bf16(t, n)
    cu = [int(x) for x in cu_seqlens]
    nseq = len(cu) - 1
    shape = make_shape(q, k, num_groups, causal)
    budget = make_budget(mode, gamma, frac_permille, score_stride, skip_threshold)
    H, G = shape.num_q_heads, num_groups
    nbs = [(cu[s + 1] - cu[s]) // 128 for s in range(nseq)]
    Ts = [rows_total(nb, causal) for nb in nbs]
    dev = q.device
    i32 = dict(device=dev, dtype=torch.int32)
    rank = torch.empty(G * sum(Ts), **i32)
    cnt = torch.empty(H * sum(nbs), **i32)
    bud = torch.empty(nseq, H, **i32)
    mass = torch.empty(H * sum(nbs), device=dev, dtype=torch.float32) if mode == DYNAMIC else None
    cu_arr = (ctypes.c_int32 * len(cu))(*cu)
    need = int(lib().pa_workspace_size_varlen(ctypes.byref(shape), ctypes.byref(budget), nseq, cu_arr))
    ws = torch.empty(max(need, 256), device=dev, dtype=torch.uint8)
    o = torch.empty_like(q, memory_format=torch.contiguous_format)
    bufs = MaskBufs(rank.data_ptr(), cnt.data_ptr(), bud.data_ptr(), mass.data_ptr() if mass is not None else None)
    _check(lib().pa_prefill_varlen(ctypes.byref(shape), ctypes.byref(budget), nseq, cu_arr, q.data_ptr(),
                                   _strides(q), k.data_ptr(), _strides(k), v.data_ptr(), _strides(v), o.data_ptr(),
                                   _strides(o), ctypes.byref(bufs), ws.data_ptr(), ws.numel(), _stream(dev)))
    views, ro, bo = [], 0, 0
    for s in range(nseq):
        views.append(Mask(rank[G * ro: G * (ro + Ts[s])].view(1, G, Ts[s]),
                          cnt[H * bo: H * (bo + nbs[s])].view(1, H, nbs[s]),
                          bud[s].view(1, H),
                          mass[H * bo: H * (bo + nbs[s])].view(1, H, nbs[s]) if mass is not None else None))
        ro += Ts[s]
        bo += nbs[s]
    return o, VarlenMask(rank, cnt, bud, mass, views)
