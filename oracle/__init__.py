"""Python (ctypes + numpy) front of the CPU fp64 oracle.

TEST INFRASTRUCTURE ONLY. The tests, the smoke check and the benchmark's
CPU-baseline leg are the only callers; the product package never imports
this module. Inputs are numpy arrays on the host: bf16 logits are passed as
their uint16 bit patterns, fp32 logits as float32.
"""
import ctypes
import os

import numpy as np

from .build import build_oracle

F32, BF16 = 0, 1
FLAG_TOKEN_RANGE, FLAG_NONFINITE, FLAG_VERIFY_LEN, FLAG_SCORES = 1, 2, 4, 8

_lib = None


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build_oracle())
        P, I, I64, D = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_double
        lib.oracle_softmax_T.argtypes = [P, I, I64, I64, I64, D, P, P, P]
        lib.oracle_verify.argtypes = [P, P, P, I, P, P, P, P, P, I, I, I, I64, D, D, I, P, P, P]
        lib.oracle_dvl_allocate.argtypes = [P, I, I, I, P, P, P, P]
        lib.oracle_pack.argtypes = [P, I, I, I, I64, P, P, P]
        for f in (lib.oracle_softmax_T, lib.oracle_verify, lib.oracle_dvl_allocate, lib.oracle_pack):
            f.restype = ctypes.c_int
        _lib = lib
    return _lib


class _Diag(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in (
        "lp", "lq", "rho", "accept_margin", "terminal_row", "terminal_kind",
        "argmax_gap", "argmax_kappa", "terminal_dist", "nucleus_margin")]


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _logits(a):
    """Return (contiguous array, dtype code) for fp32 or bf16-bit (uint16) logits."""
    a = np.ascontiguousarray(a)
    if a.dtype == np.float32:
        return a, F32
    if a.dtype == np.uint16:
        return a, BF16
    raise TypeError("logits must be float32 or bf16 bits as uint16, got %s" % a.dtype)


def softmax_T(x, T, probs=False):
    """Row statistics of z = x / T for x of shape [rows, V].

    Returns (row_max, row_lse) or (row_max, row_lse, probs) as float64."""
    x, dt = _logits(x)
    rows, V = x.shape
    rmax = np.empty(rows, np.float64)
    rlse = np.empty(rows, np.float64)
    p = np.empty((rows, V), np.float64) if probs else None
    st = _load().oracle_softmax_T(_ptr(x), dt, rows, V, V, float(T), _ptr(rmax), _ptr(rlse), _ptr(p))
    if st < 0:
        raise ValueError("oracle_softmax_T rejected its arguments (%d)" % st)
    return (rmax, rlse, p) if probs else (rmax, rlse)


def verify(target, draft, tokens, u, g, T, *, mix_w=None, verify_len=None, target_row_off=None,
           n_threads=1, diag=False, top_p=1.0):
    """Speculative verification of B drafted blocks (see oracle.h).

    target: [B, L+1, V] dense, or packed [S, V] with target_row_off [B].
    draft:  [B, L, V] (independent) or [B, K, L, V] (latent mixture, with mix_w [B, K]).
    top_p:  nucleus filter of every target and draft row (1 = none; see oracle.h).
    Returns dict(accept_len, out_tokens, flags[, diagnostics...])."""
    target, dt = _logits(target)
    draft, dt2 = _logits(draft)
    if dt != dt2:
        raise TypeError("target and draft logits must share a dtype")
    tokens = np.ascontiguousarray(tokens, np.int32)
    B, L = tokens.shape
    V = target.shape[-1]
    if draft.ndim == 3:
        K = 1
    else:
        K = draft.shape[1]
    u = np.ascontiguousarray(u, np.float32)
    g = np.ascontiguousarray(g, np.float32)
    if g.shape != (B, L + 1, V):
        raise ValueError("g must be [B, L+1, V]")
    w = None if mix_w is None else np.ascontiguousarray(mix_w, np.float32)
    vl = None if verify_len is None else np.ascontiguousarray(verify_len, np.int32)
    off = None if target_row_off is None else np.ascontiguousarray(target_row_off, np.int32)
    acc = np.empty(B, np.int32)
    out = np.empty((B, L + 1), np.int32)
    res = {}
    dptr = None
    if diag:
        res = dict(lp=np.empty((B, L)), lq=np.empty((B, L)), rho=np.empty((B, L)),
                   accept_margin=np.empty((B, L)), terminal_row=np.empty(B, np.int32),
                   terminal_kind=np.empty(B, np.int32), argmax_gap=np.empty(B),
                   argmax_kappa=np.empty(B), terminal_dist=np.empty((B, V)), nucleus_margin=np.empty(B))
        dptr = ctypes.byref(_Diag(*[_ptr(res[f[0]]) for f in _Diag._fields_]))
    st = _load().oracle_verify(_ptr(target), _ptr(off), _ptr(draft), dt, _ptr(tokens), _ptr(vl),
                               _ptr(u), _ptr(g), _ptr(w), K, B, L, V, float(T), float(top_p), int(n_threads),
                               _ptr(acc), _ptr(out), dptr)
    if st < 0:
        raise ValueError("oracle_verify rejected its arguments (%d)" % st)
    res.update(accept_len=acc, out_tokens=out, flags=st)
    return res


def dvl_allocate(scores, budget):
    """Greedy global top-k verify-length allocation. Returns dict(verify_len,
    offsets, slot_map, prefix, flags)."""
    s = np.ascontiguousarray(scores, np.float32)
    B, L = s.shape
    vl = np.empty(B, np.int32)
    off = np.empty(B + 1, np.int32)
    sm = np.empty(max(int(budget), 0), np.int32)
    pre = np.empty((B, L), np.float64)
    st = _load().oracle_dvl_allocate(_ptr(s), B, L, int(budget), _ptr(vl), _ptr(off), _ptr(sm), _ptr(pre))
    if st < 0:
        raise ValueError("oracle_dvl_allocate rejected its arguments (%d)" % st)
    return dict(verify_len=vl, offsets=off, slot_map=sm, prefix=pre, flags=st)


def pack(dense, verify_len, offsets, budget):
    """packed[offsets[b] + i] = dense[b, i] for i <= verify_len[b]; other rows are zero."""
    dense, dt = _logits(dense)
    B, L1, V = dense.shape
    packed = np.zeros((int(budget), V), dense.dtype)
    vl = np.ascontiguousarray(verify_len, np.int32)
    off = np.ascontiguousarray(offsets, np.int32)
    st = _load().oracle_pack(_ptr(dense), dt, B, L1 - 1, V, _ptr(vl), _ptr(off), _ptr(packed))
    if st < 0:
        raise ValueError("oracle_pack rejected its arguments (%d)" % st)
    return packed


def n_cores():
    return len(os.sched_getaffinity(0))
