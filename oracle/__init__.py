"""CPU oracle for ProxyAttn-style block-sparse prefill attention (fp64).

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py``.  The product path never imports it.

This module is argument marshalling around ``pa_oracle.c`` (plain C, fp64,
OpenMP); every step of the method lives in that file, which cites the page
passage each function follows.  Inputs are bf16 torch tensors on the CPU with a
contiguous last dimension; they are read as raw bf16 bits and upcast exactly.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "pa_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

DYNAMIC, FIXED_FRACTION, ALL = 0, 1, 2
BLK = 128


def build(force: bool = False) -> str:
    """Compile pa_oracle.c into liboracle.so next to it (gcc, OpenMP, IEEE fp64)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
                               "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        _lib.pa_oracle_f64_to_bf16.restype = ctypes.c_uint16
        _lib.pa_oracle_f64_to_bf16.argtypes = [ctypes.c_double]
        _lib.pa_oracle_num_threads.restype = ctypes.c_int
    return _lib


_i = ctypes.c_int
_i64 = ctypes.c_int64
_d = ctypes.c_double


def _p(a: np.ndarray):
    return ctypes.c_void_p(a.ctypes.data)


def _bits(t: torch.Tensor):
    """(uint16 numpy view sharing storage, (sb, ss, sh) element strides) of a
    bf16 [B, N, heads, d] CPU tensor."""
    assert t.dtype == torch.bfloat16 and t.device.type == "cpu" and t.dim() == 4
    assert t.stride(3) == 1, "last dimension must be contiguous"
    base = t.as_strided((t.untyped_storage().nbytes() // 2,), (1,), 0)
    arr = base.view(torch.int16).numpy().view(np.uint16)
    off = t.storage_offset()
    return arr[off:], (t.stride(0), t.stride(1), t.stride(2))


def f64_to_bf16_bits(x: float) -> int:
    return int(lib().pa_oracle_f64_to_bf16(float(x)))


def num_threads() -> int:
    return int(lib().pa_oracle_num_threads())


def pool(q: torch.Tensor, k: torch.Tensor, G: int):
    """o1: returns (qp_f64, kp_f64, qp_bf16, kp_bf16); shapes [B, G, N, d];
    the bf16 ones as torch.bfloat16 tensors."""
    B, N, H, d = q.shape
    Hkv = k.shape[2]
    qa, qs = _bits(q)
    ka, ks = _bits(k)
    qp = np.empty((B, G, N, d), np.float64)
    kp = np.empty((B, G, N, d), np.float64)
    qpb = np.empty((B, G, N, d), np.uint16)
    kpb = np.empty((B, G, N, d), np.uint16)
    lib().pa_oracle_pool(_i(B), _i(N), _i(H), _i(Hkv), _i(d), _i(G),
                         _p(qa), _i64(qs[0]), _i64(qs[1]), _i64(qs[2]),
                         _p(ka), _i64(ks[0]), _i64(ks[1]), _i64(ks[2]),
                         _p(qp), _p(kp), _p(qpb), _p(kpb))
    to_bf = lambda a: torch.from_numpy(a.view(np.int16)).view(torch.bfloat16)
    return qp, kp, to_bf(qpb), to_bf(kpb)


def _proxy_bits(t: torch.Tensor) -> np.ndarray:
    assert t.dtype == torch.bfloat16 and t.is_contiguous() and t.device.type == "cpu"
    return t.view(torch.int16).numpy().view(np.uint16)


def rows_total(nb: int, causal: bool = True) -> int:
    """Entries of one (b, g) row set of scores or lists: T = nb(nb+1)/2
    causal (row qb at qb(qb+1)/2), nb*nb non-causal (row qb at qb*nb)."""
    return nb * (nb + 1) // 2 if causal else nb * nb


def row_at(nb: int, qb: int, causal: bool = True) -> int:
    return qb * (qb + 1) // 2 if causal else qb * nb


def block_scores(qp_bf16: torch.Tensor, kp_bf16: torch.Tensor, scale: float | None = None,
                 stride: int = 1, causal: bool = True) -> np.ndarray:
    """o2: scores [B, G, T] fp64 from the bf16 proxies [B, G, N, d]; with
    stride r only the query rows i = r-1 (mod r) are scored."""
    B, G, N, d = qp_bf16.shape
    nb = N // BLK
    scale = 1.0 / np.sqrt(d) if scale is None else scale
    assert stride >= 1 and BLK % stride == 0
    out = np.empty((B, G, rows_total(nb, causal)), np.float64)
    lib().pa_oracle_block_scores(_i(B), _i(N), _i(G), _i(d), _p(_proxy_bits(qp_bf16)),
                                 _p(_proxy_bits(kp_bf16)), _d(scale), _i(stride), _i(int(causal)), _p(out))
    return out


def block_score_tiles(qp_bf16: torch.Tensor, kp_bf16: torch.Tensor, tiles, scale: float | None = None,
                      stride: int = 1, causal: bool = True) -> np.ndarray:
    """o2 on a sample: tiles is an int array [n, 4] of (b, g, qb, kb)."""
    B, G, N, d = qp_bf16.shape
    scale = 1.0 / np.sqrt(d) if scale is None else scale
    assert stride >= 1 and BLK % stride == 0
    tiles = np.ascontiguousarray(np.asarray(tiles, np.int32).reshape(-1, 4))
    out = np.empty(len(tiles), np.float64)
    lib().pa_oracle_block_score_tiles(_i(N), _i(G), _i(d), _p(_proxy_bits(qp_bf16)),
                                      _p(_proxy_bits(kp_bf16)), _d(scale), _i(stride), _i(int(causal)),
                                      _i(len(tiles)),
                                      _p(tiles), _p(out))
    return out


def head_mass(q: torch.Tensor, k: torch.Tensor, scale: float | None = None, with_rowsum=False,
              causal: bool = True):
    """o3: mass [B, H, nb] fp64 (and, optionally, max |row sum - 1| per (b, h))."""
    B, N, H, d = q.shape
    Hkv = k.shape[2]
    nb = N // BLK
    scale = 1.0 / np.sqrt(d) if scale is None else scale
    qa, qs = _bits(q)
    ka, ks = _bits(k)
    mass = np.empty((B, H, nb), np.float64)
    dev = np.empty((B, H), np.float64)
    lib().pa_oracle_head_mass(_i(B), _i(N), _i(H), _i(Hkv), _i(d),
                              _p(qa), _i64(qs[0]), _i64(qs[1]), _i64(qs[2]),
                              _p(ka), _i64(ks[0]), _i64(ks[1]), _i64(ks[2]),
                              _d(scale), _i(int(causal)), _p(mass), _p(dev))
    return (mass, dev) if with_rowsum else mass


def rank(scores: np.ndarray, nb: int, causal: bool = True) -> np.ndarray:
    """o4a: ranked lists [B, G, T] int32 from block scores [B, G, T] (any float dtype;
    converted exactly to fp64)."""
    s = np.ascontiguousarray(np.asarray(scores, dtype=np.float64))
    B, G, T = s.shape
    assert T == rows_total(nb, causal)
    out = np.empty((B, G, T), np.int32)
    lib().pa_oracle_rank(_i(B), _i(G), _i(nb), _p(s), _i(int(causal)), _p(out))
    return out


def budget(rank_lists: np.ndarray, mass, H: int, G: int, nb: int, mode: int = DYNAMIC,
           gamma: float = 0.95, frac_permille: int = 0, causal: bool = True):
    """o4b: (budget [B, H] int32, cnt [B, H, nb] int32)."""
    r = np.ascontiguousarray(np.asarray(rank_lists, np.int32))
    B = r.shape[0]
    if mass is None:
        m = np.zeros((B, H, nb), np.float64)
    else:
        m = np.ascontiguousarray(np.asarray(mass, np.float64))
    bud = np.empty((B, H), np.int32)
    cnt = np.empty((B, H, nb), np.int32)
    lib().pa_oracle_budget(_i(B), _i(H), _i(G), _i(nb), _i(mode), _d(gamma), _i(frac_permille),
                           _p(r), _p(m), _i(int(causal)), _p(bud), _p(cnt))
    return bud, cnt


def sparse_attn(q, k, v, rank_lists, cnt, G: int, items, scale: float | None = None, causal: bool = True):
    """o5: for items [n, 3] of (b, h, qb) returns (O [n, 128, d], lse [n, 128]) fp64."""
    B, N, H, d = q.shape
    Hkv = k.shape[2]
    scale = 1.0 / np.sqrt(d) if scale is None else scale
    qa, qs = _bits(q)
    ka, ks = _bits(k)
    va, vs = _bits(v)
    items = np.ascontiguousarray(np.asarray(items, np.int32).reshape(-1, 3))
    r = np.ascontiguousarray(np.asarray(rank_lists, np.int32))
    c = np.ascontiguousarray(np.asarray(cnt, np.int32))
    out = np.empty((len(items), BLK, d), np.float64)
    lse = np.empty((len(items), BLK), np.float64)
    lib().pa_oracle_sparse_attn(_i(N), _i(H), _i(Hkv), _i(d), _i(G),
                                _p(qa), _i64(qs[0]), _i64(qs[1]), _i64(qs[2]),
                                _p(ka), _i64(ks[0]), _i64(ks[1]), _i64(ks[2]),
                                _p(va), _i64(vs[0]), _i64(vs[1]), _i64(vs[2]),
                                _p(r), _p(c), _d(scale), _i(int(causal)), _i(len(items)), _p(items), _p(out),
                                _p(lse))
    return out, lse


def sparse_attn_skip(q, k, v, rank_lists, cnt, G: int, items, lam: float, skip_in=None,
                     scale: float | None = None, causal: bool = True):
    """o7: o5 with the running-max block skip at threshold lam.  Returns
    (O [n, 128, d], lse [n, 128], skip [B, H, T] uint8, gap [B, H, T] fp64):
    skip and gap hold the oracle's own decision and its margin (log2 units)
    for every visited block of the items (gap NaN elsewhere, +inf for each
    item's first block).  skip_in ([B, H, T], nonzero = skipped) replaces the
    oracle's decisions in the output."""
    B, N, H, d = q.shape
    Hkv = k.shape[2]
    nb = N // BLK
    T = rows_total(nb, causal)
    scale = 1.0 / np.sqrt(d) if scale is None else scale
    qa, qs = _bits(q)
    ka, ks = _bits(k)
    va, vs = _bits(v)
    items = np.ascontiguousarray(np.asarray(items, np.int32).reshape(-1, 3))
    r = np.ascontiguousarray(np.asarray(rank_lists, np.int32))
    c = np.ascontiguousarray(np.asarray(cnt, np.int32))
    out = np.empty((len(items), BLK, d), np.float64)
    lse = np.empty((len(items), BLK), np.float64)
    skip = np.zeros((B, H, T), np.uint8)
    gap = np.full((B, H, T), np.nan, np.float64)
    sin = None if skip_in is None else np.ascontiguousarray(np.asarray(skip_in, np.uint8).reshape(B, H, T))
    lib().pa_oracle_sparse_attn_skip(_i(N), _i(H), _i(Hkv), _i(d), _i(G),
                                     _p(qa), _i64(qs[0]), _i64(qs[1]), _i64(qs[2]),
                                     _p(ka), _i64(ks[0]), _i64(ks[1]), _i64(ks[2]),
                                     _p(va), _i64(vs[0]), _i64(vs[1]), _i64(vs[2]),
                                     _p(r), _p(c), _d(scale), _d(lam), _i(int(causal)), _i(len(items)), _p(items),
                                     _p(sin) if sin is not None else None, _p(skip), _p(gap), _p(out), _p(lse))
    return out, lse, skip, gap


def xattn_mass(q, k, S: int, causal: bool = True) -> np.ndarray:
    """o8: XAttention antidiagonal block estimates [B, H, T] at stride S."""
    B, N, H, d = q.shape
    Hkv = k.shape[2]
    nb = N // BLK
    assert BLK % S == 0
    qa, qs = _bits(q)
    ka, ks = _bits(k)
    out = np.empty((B, H, rows_total(nb, causal)), np.float64)
    lib().pa_oracle_xattn_mass(_i(B), _i(N), _i(H), _i(Hkv), _i(d), _i(S),
                               _p(qa), _i64(qs[0]), _i64(qs[1]), _i64(qs[2]),
                               _p(ka), _i64(ks[0]), _i64(ks[1]), _i64(ks[2]), _i(int(causal)), _p(out))
    return out


def find_blocks(mass, nb: int, tau: float, causal: bool = True):
    """o8 selection: (rank [B, H, T] int32, cnt [B, H, nb] int32) from block
    estimates [B, H, T] (any float type; compared as float64)."""
    m = np.ascontiguousarray(np.asarray(mass, np.float64))
    B, H, T = m.shape
    assert T == rows_total(nb, causal)
    rank = np.empty((B, H, T), np.int32)
    cnt = np.empty((B, H, nb), np.int32)
    lib().pa_oracle_find_blocks(_i(B), _i(H), _i(nb), _p(m), _d(tau), _i(int(causal)), _p(rank), _p(cnt))
    return rank, cnt


def dense_attn(q, k, v, rows, scale: float | None = None, causal: bool = True):
    """o6: for rows [n, 3] of (b, h, i) returns (O [n, d], lse [n]) fp64."""
    B, N, H, d = q.shape
    Hkv = k.shape[2]
    scale = 1.0 / np.sqrt(d) if scale is None else scale
    qa, qs = _bits(q)
    ka, ks = _bits(k)
    va, vs = _bits(v)
    rows = np.ascontiguousarray(np.asarray(rows, np.int32).reshape(-1, 3))
    out = np.empty((len(rows), d), np.float64)
    lse = np.empty(len(rows), np.float64)
    lib().pa_oracle_dense_attn(_i(N), _i(H), _i(Hkv), _i(d),
                               _p(qa), _i64(qs[0]), _i64(qs[1]), _i64(qs[2]),
                               _p(ka), _i64(ks[0]), _i64(ks[1]), _i64(ks[2]),
                               _p(va), _i64(vs[0]), _i64(vs[1]), _i64(vs[2]),
                               _d(scale), _i(int(causal)), _i(len(rows)), _p(rows), _p(out), _p(lse))
    return out, lse


def prefill_masks(q, k, G: int, mode=DYNAMIC, gamma=0.95, frac_permille=0, stride=1, causal=True):
    """o1-o4 end to end on the oracle's own fp64 scores and masses:
    dict(qp, kp, scores, mass, rank, budget, cnt)."""
    B, N, H, d = q.shape
    nb = N // BLK
    _, _, qpb, kpb = pool(q, k, G)
    scores = block_scores(qpb, kpb, stride=stride, causal=causal)
    mass = head_mass(q, k, causal=causal) if mode == DYNAMIC else None
    r = rank(scores, nb, causal)
    bud, cnt = budget(r, mass, H, G, nb, mode, gamma, frac_permille, causal)
    return dict(qp=qpb, kp=kpb, scores=scores, mass=mass, rank=r, budget=bud, cnt=cnt)
