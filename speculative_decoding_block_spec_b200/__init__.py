"""specv — batched verification and acceptance of block-diffusion speculative
drafts on NVIDIA B200 (sm_100a).

This module is a thin ctypes binding over libspecv.so, whose C ABI is
declared in include/specv.h. It only marshals torch CUDA tensors into
pointers and sizes; every step of the computation runs in the library's CUDA
kernels. There is no CPU fallback: if the library is not built, or a tensor
is not on a CUDA device, the call raises.

Entry points (same names as the C ABI):
  softmax_T(logits, T, probs=False)             temperature softmax statistics
  spec_softmax_T(logits, T, row_max, row_lse, probs=None, workspace=None)
  spec_softmax_T_noalloc(logits, T, row_max, row_lse, probs=None)
  spec_verify_block(target, draft, tokens, u, g, T, ...)
  spec_verify_mixture(target, draft, mix_w, tokens, u, g, T, ...)
  spec_verify_block_top_p(target, draft, tokens, u, g, T, top_p, ...)     rows filtered to their nuclei
  spec_verify_mixture_top_p(target, draft, mix_w, tokens, u, g, T, top_p, ...)
  spec_verify_window_stats(...), spec_verify_accept(...)   the two verify stages
  dvl_allocate_pack(scores, budget, dense_target=None, packed_target=None)
Workspaces: Workspace(nbytes, device), with verify/softmax/dvl size helpers;
Workspace.status() reads the sticky device flags (DEV_*).
"""
import ctypes
import os

import torch

__all__ = ["SpecError", "Workspace", "lib", "softmax_T", "spec_softmax_T", "spec_softmax_T_noalloc", "NOALLOC_MAX_ROWS", "spec_verify_block",
           "spec_verify_mixture", "spec_verify_block_top_p", "spec_verify_mixture_top_p",
           "verify_top_p_workspace_size", "spec_verify_window_stats", "spec_verify_accept", "dvl_allocate_pack", "verify_workspace_size", "softmax_workspace_size",
           "dvl_workspace_size", "check_verify_args", "LIB_PATH", "EXPORTS", "DEV_TOKEN_RANGE", "DEV_NONFINITE", "DEV_VERIFY_LEN",
           "DEV_SCORES"]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "_lib", "libspecv.so")

DEV_TOKEN_RANGE, DEV_NONFINITE, DEV_VERIFY_LEN, DEV_SCORES = 1, 2, 4, 8
NOALLOC_MAX_ROWS = 4096  # SPEC_NOALLOC_MAX_ROWS
_F32, _BF16 = 0, 1

_P, _I, _I64, _F, _SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t
_SIGS = {
    "spec_status_string": ([_I], ctypes.c_char_p),
    "spec_softmax_workspace_size": ([_I64], _SZ),
    "spec_verify_workspace_size": ([_I, _I, _I, _I64], _SZ),
    "spec_verify_top_p_workspace_size": ([_I, _I, _I, _I64], _SZ),
    "spec_dvl_workspace_size": ([_I], _SZ),
    "spec_workspace_init": ([_P, _SZ, _P], _I),
    "spec_softmax_T": ([_P, _I, _I64, _I64, _I64, _F, _P, _P, _P, _P, _SZ, _P], _I),
    "spec_softmax_T_noalloc": ([_P, _I, _I64, _I64, _I64, _F, _P, _P, _P, _P], _I),
    "spec_verify_block": ([_P, _P, _P, _I, _P, _P, _P, _P, _I, _I, _I64, _F, _P, _P, _P, _SZ, _P], _I),
    "spec_verify_mixture": ([_P, _P, _P, _P, _I, _I, _P, _P, _P, _P, _I, _I, _I64, _F, _P, _P, _P, _SZ, _P], _I),
    "spec_verify_block_top_p": ([_P, _P, _P, _I, _P, _P, _P, _P, _I, _I, _I64, _F, _F, _P, _P, _P, _SZ, _P], _I),
    "spec_verify_mixture_top_p": ([_P, _P, _P, _P, _I, _I, _P, _P, _P, _P, _I, _I, _I64, _F, _F, _P, _P, _P, _SZ, _P],
                                  _I),
    "spec_verify_window_stats": ([_P, _P, _P, _I, _I, _P, _P, _I, _I, _I64, _F, _P, _SZ, _P], _I),
    "spec_verify_accept": ([_P, _P, _P, _P, _I, _I, _P, _P, _P, _P, _I, _I, _I64, _F, _P, _P, _P, _SZ, _P], _I),
    "dvl_allocate_pack": ([_P, _I, _I, _I, _P, _P, _P, _P, _P, _I, _I64, _P, _SZ, _P], _I),
}
EXPORTS = tuple(_SIGS)

_lib = None


class SpecError(RuntimeError):
    """A specv call was rejected (negative spec_status)."""

    def __init__(self, fn, status):
        super().__init__("%s: %s" % (fn, lib().spec_status_string(status).decode()))
        self.status = status


def lib():
    """Load libspecv.so (built in-tree by `python -m speculative_decoding_block_spec_b200.build`)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError("libspecv.so is not built (%s); run "
                               "`python -m speculative_decoding_block_spec_b200.build`" % LIB_PATH)
        h = ctypes.CDLL(LIB_PATH)
        for name, (args, res) in _SIGS.items():
            fn = getattr(h, name)
            fn.argtypes = args
            fn.restype = res
        _lib = h
    return _lib


def _call(name, *args):
    st = getattr(lib(), name)(*args)
    if st != 0:
        raise SpecError(name, st)


def softmax_workspace_size(rows):
    return int(lib().spec_softmax_workspace_size(rows))


def verify_workspace_size(B, L, K=1, V=151936):
    return int(lib().spec_verify_workspace_size(B, L, K, V))


def verify_top_p_workspace_size(B, L, K=1, V=151936):
    return int(lib().spec_verify_top_p_workspace_size(B, L, K, V))


def dvl_workspace_size(B):
    return int(lib().spec_dvl_workspace_size(B))


class Workspace:
    """A caller-owned, fixed-address device workspace, zeroed once at creation."""

    def __init__(self, nbytes, device=None):
        if nbytes <= 0:
            raise ValueError("workspace size must be positive (shape outside the supported limits?)")
        self.buf = torch.empty(int(nbytes), dtype=torch.uint8, device=device or "cuda")
        self.init()

    @property
    def nbytes(self):
        return self.buf.numel()

    def ptr(self):
        return self.buf.data_ptr()

    def init(self):
        _call("spec_workspace_init", self.ptr(), self.nbytes, _stream(self.buf))

    def status(self):
        """Sticky device status (OR of DEV_* flags); synchronises the current stream."""
        return int(self.buf[:4].view(torch.int32).item())


def _stream(t):
    return torch.cuda.current_stream(t.device).cuda_stream


def _dtype_code(t):
    if t.dtype == torch.float32:
        return _F32
    if t.dtype == torch.bfloat16:
        return _BF16
    raise TypeError("logits must be float32 or bfloat16, got %s" % t.dtype)


def _dev(t, name, dtype=None):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError("%s must be a CUDA tensor" % name)
    if dtype is not None and t.dtype != dtype:
        raise TypeError("%s must be %s, got %s" % (name, dtype, t.dtype))
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)
    return t.data_ptr()


def _opt(t, name, dtype):
    return None if t is None else _dev(t, name, dtype)


def _softmax_shapes(logits, row_max, row_lse, probs):
    _shape(logits, "logits", (None, None))
    rows, V = logits.shape
    _shape(row_max, "row_max", (rows,))
    _shape(row_lse, "row_lse", (rows,))
    if probs is not None:
        _shape(probs, "probs", (rows, V))
    return rows, V


def spec_softmax_T(logits, T, row_max, row_lse, probs=None, workspace=None):
    """C-ABI spec_softmax_T on preallocated outputs. logits [rows, V] (row stride V)."""
    rows, V = _softmax_shapes(logits, row_max, row_lse, probs)
    ws = workspace or Workspace(softmax_workspace_size(rows), logits.device)
    _call("spec_softmax_T", _dev(logits, "logits"), _dtype_code(logits), rows, V, V, float(T),
          _dev(row_max, "row_max", torch.float32), _dev(row_lse, "row_lse", torch.float32),
          _opt(probs, "probs", torch.float32), ws.ptr(), ws.nbytes, _stream(logits))
    return ws


def spec_softmax_T_noalloc(logits, T, row_max, row_lse, probs=None):
    """C-ABI spec_softmax_T_noalloc on preallocated outputs: spec_softmax_T with
    the library's fixed scratch instead of a workspace (rows <= NOALLOC_MAX_ROWS;
    calls on one device must not overlap on the GPU)."""
    rows, V = _softmax_shapes(logits, row_max, row_lse, probs)
    if rows > NOALLOC_MAX_ROWS:
        raise ValueError("spec_softmax_T_noalloc: %d rows exceed the fixed scratch limit of %d rows"
                         % (rows, NOALLOC_MAX_ROWS))
    _call("spec_softmax_T_noalloc", _dev(logits, "logits"), _dtype_code(logits), rows, V, V, float(T),
          _dev(row_max, "row_max", torch.float32), _dev(row_lse, "row_lse", torch.float32),
          _opt(probs, "probs", torch.float32), _stream(logits))


def softmax_T(logits, T, probs=False, workspace=None):
    """Temperature softmax of each row of logits [rows, V]: returns (row_max,
    row_lse) of z = logits / T, plus fp32 probabilities if probs=True."""
    rows, V = logits.shape
    rmax = torch.empty(rows, dtype=torch.float32, device=logits.device)
    rlse = torch.empty_like(rmax)
    p = torch.empty((rows, V), dtype=torch.float32, device=logits.device) if probs else None
    spec_softmax_T(logits, T, rmax, rlse, p, workspace)
    return (rmax, rlse, p) if probs else (rmax, rlse)


def _shape(t, name, shape):
    """Raises unless tensor t has exactly `shape` (entries of None match any size)."""
    if not isinstance(t, torch.Tensor):
        raise TypeError("%s must be a tensor" % name)
    if t.dim() != len(shape) or any(want is not None and got != want for got, want in zip(t.shape, shape)):
        raise ValueError("%s has shape %s, expected %s" % (name, tuple(t.shape),
                                                            tuple("*" if w is None else w for w in shape)))


def check_verify_args(target, draft, tokens, u, g, *, mix_w=None, verify_len=None, target_row_off=None,
                      out=None, mixture=None):
    """Host-side shape and device checks of a verify call, done before any
    pointer reaches the library (the C ABI sees raw pointers and cannot tell a
    short tensor from a long one). Returns (B, L, K, V). mixture=None infers
    the draft layout from its rank: [B, L, V] (K = 1) or [B, K, L, V]."""
    _shape(tokens, "tokens", (None, None))
    B, L = tokens.shape
    if mixture is None:
        mixture = draft.dim() == 4
    if mixture:
        _shape(draft, "draft", (B, None, L, None))
        K = draft.shape[1]
    else:
        _shape(draft, "draft", (B, L, None))
        K = 1
    V = draft.shape[-1]
    if target_row_off is None:
        _shape(target, "target", (B, L + 1, V))
    else:
        _shape(target, "target", (None, V))
        if target.shape[0] < L + 1:
            raise ValueError("packed target has %d rows, fewer than one request's L+1 = %d" % (target.shape[0], L + 1))
        if target_row_off.dim() != 1 or target_row_off.numel() < B:
            raise ValueError("target_row_off must be 1-D with at least B = %d entries" % B)
    _shape(u, "u", (B, L))
    _shape(g, "g", (B, L + 1, V))
    if mix_w is not None:
        _shape(mix_w, "mix_w", (B, K))
    if verify_len is not None and (verify_len.dim() != 1 or verify_len.numel() < B):
        raise ValueError("verify_len must be 1-D with at least B = %d entries" % B)
    if out is not None:
        _shape(out[0], "accept_len", (B,))
        _shape(out[1], "out_tokens", (B, L + 1))
    tensors = [target, draft, tokens, u, g, mix_w, verify_len, target_row_off] + list(out or [])
    devs = {t.device for t in tensors if t is not None}
    if len(devs) > 1:
        raise ValueError("all tensors of a verify call must be on one device, got %s" % sorted(map(str, devs)))
    return B, L, K, V


def _outputs(B, L, device, out):
    if out is None:
        return (torch.empty(B, dtype=torch.int32, device=device),
                torch.empty((B, L + 1), dtype=torch.int32, device=device))
    return out


def spec_verify_block(target, draft, tokens, u, g, T, *, verify_len=None, target_row_off=None, workspace=None,
                      out=None):
    """Verify B independently drafted blocks. target [B, L+1, V] (or packed rows
    [S, V] with target_row_off [B]), draft [B, L, V], tokens [B, L] int32,
    u [B, L] fp32, g [B, L+1, V] fp32. Returns (accept_len [B], out_tokens [B, L+1])."""
    B, L, _, V = check_verify_args(target, draft, tokens, u, g, verify_len=verify_len,
                                   target_row_off=target_row_off, out=out, mixture=False)
    ws = workspace or Workspace(verify_workspace_size(B, L, 1, V), draft.device)
    acc, outt = _outputs(B, L, draft.device, out)
    if _dtype_code(target) != _dtype_code(draft):
        raise TypeError("target and draft logits must share a dtype")
    _call("spec_verify_block", _dev(target, "target"), _opt(target_row_off, "target_row_off", torch.int32),
          _dev(draft, "draft"), _dtype_code(draft), _dev(tokens, "tokens", torch.int32),
          _opt(verify_len, "verify_len", torch.int32), _dev(u, "u", torch.float32), _dev(g, "g", torch.float32),
          B, L, V, float(T), _dev(acc, "accept_len", torch.int32), _dev(outt, "out_tokens", torch.int32),
          ws.ptr(), ws.nbytes, _stream(draft))
    return acc, outt


def spec_verify_mixture(target, draft, mix_w, tokens, u, g, T, *, verify_len=None, target_row_off=None,
                        workspace=None, out=None):
    """Verify B latent-mixture drafts: draft [B, K, L, V], mix_w [B, K] fp32
    (category probabilities q(z|y)); other arguments as spec_verify_block."""
    B, L, K, V = check_verify_args(target, draft, tokens, u, g, mix_w=mix_w, verify_len=verify_len,
                                   target_row_off=target_row_off, out=out, mixture=True)
    ws = workspace or Workspace(verify_workspace_size(B, L, K, V), draft.device)
    acc, outt = _outputs(B, L, draft.device, out)
    if _dtype_code(target) != _dtype_code(draft):
        raise TypeError("target and draft logits must share a dtype")
    _call("spec_verify_mixture", _dev(target, "target"), _opt(target_row_off, "target_row_off", torch.int32),
          _dev(draft, "draft"), _dev(mix_w, "mix_w", torch.float32), K, _dtype_code(draft),
          _dev(tokens, "tokens", torch.int32), _opt(verify_len, "verify_len", torch.int32),
          _dev(u, "u", torch.float32), _dev(g, "g", torch.float32), B, L, V, float(T),
          _dev(acc, "accept_len", torch.int32), _dev(outt, "out_tokens", torch.int32), ws.ptr(), ws.nbytes,
          _stream(draft))
    return acc, outt


def spec_verify_block_top_p(target, draft, tokens, u, g, T, top_p, *, verify_len=None, target_row_off=None,
                            workspace=None, out=None):
    """spec_verify_block with every target and draft row filtered to its top-p
    nucleus (0 < top_p <= 1). The workspace is verify_top_p_workspace_size."""
    B, L, _, V = check_verify_args(target, draft, tokens, u, g, verify_len=verify_len,
                                   target_row_off=target_row_off, out=out, mixture=False)
    ws = workspace or Workspace(verify_top_p_workspace_size(B, L, 1, V), draft.device)
    acc, outt = _outputs(B, L, draft.device, out)
    if _dtype_code(target) != _dtype_code(draft):
        raise TypeError("target and draft logits must share a dtype")
    _call("spec_verify_block_top_p", _dev(target, "target"), _opt(target_row_off, "target_row_off", torch.int32),
          _dev(draft, "draft"), _dtype_code(draft), _dev(tokens, "tokens", torch.int32),
          _opt(verify_len, "verify_len", torch.int32), _dev(u, "u", torch.float32), _dev(g, "g", torch.float32),
          B, L, V, float(T), float(top_p), _dev(acc, "accept_len", torch.int32),
          _dev(outt, "out_tokens", torch.int32), ws.ptr(), ws.nbytes, _stream(draft))
    return acc, outt


def spec_verify_mixture_top_p(target, draft, mix_w, tokens, u, g, T, top_p, *, verify_len=None,
                              target_row_off=None, workspace=None, out=None):
    """spec_verify_mixture with every target and draft row filtered to its
    top-p nucleus (0 < top_p <= 1)."""
    B, L, K, V = check_verify_args(target, draft, tokens, u, g, mix_w=mix_w, verify_len=verify_len,
                                   target_row_off=target_row_off, out=out, mixture=True)
    ws = workspace or Workspace(verify_top_p_workspace_size(B, L, K, V), draft.device)
    acc, outt = _outputs(B, L, draft.device, out)
    if _dtype_code(target) != _dtype_code(draft):
        raise TypeError("target and draft logits must share a dtype")
    _call("spec_verify_mixture_top_p", _dev(target, "target"), _opt(target_row_off, "target_row_off", torch.int32),
          _dev(draft, "draft"), _dev(mix_w, "mix_w", torch.float32), K, _dtype_code(draft),
          _dev(tokens, "tokens", torch.int32), _opt(verify_len, "verify_len", torch.int32),
          _dev(u, "u", torch.float32), _dev(g, "g", torch.float32), B, L, V, float(T), float(top_p),
          _dev(acc, "accept_len", torch.int32), _dev(outt, "out_tokens", torch.int32), ws.ptr(), ws.nbytes,
          _stream(draft))
    return acc, outt


def spec_verify_window_stats(target, draft, tokens, T, workspace, *, verify_len=None, target_row_off=None):
    """Stage 1 of verification: temperature-softmax statistics of the verify
    window, and each row's logit at the drafted token, into `workspace`
    (draft [B, L, V] for K == 1, else [B, K, L, V]; tokens [B, L] int32)."""
    _shape(tokens, "tokens", (None, None))
    B, L = tokens.shape
    _shape(draft, "draft", (B, L, None) if draft.dim() == 3 else (B, None, L, None))
    K = 1 if draft.dim() == 3 else draft.shape[1]
    V = draft.shape[-1]
    if target_row_off is None:
        _shape(target, "target", (B, L + 1, V))
    else:
        _shape(target, "target", (None, V))
    _call("spec_verify_window_stats", _dev(target, "target"), _opt(target_row_off, "target_row_off", torch.int32),
          _dev(draft, "draft"), K, _dtype_code(draft), _dev(tokens, "tokens", torch.int32),
          _opt(verify_len, "verify_len", torch.int32), B, L, V, float(T), workspace.ptr(), workspace.nbytes,
          _stream(draft))


def spec_verify_accept(target, draft, tokens, u, g, T, workspace, *, mix_w=None, verify_len=None,
                       target_row_off=None, out=None):
    """Stage 2 of verification (after spec_verify_window_stats on the same
    workspace): accept tests, first rejection and the terminal draw."""
    B, L, K, V = check_verify_args(target, draft, tokens, u, g, mix_w=mix_w, verify_len=verify_len,
                                   target_row_off=target_row_off, out=out)
    acc, outt = _outputs(B, L, draft.device, out)
    _call("spec_verify_accept", _dev(target, "target"), _opt(target_row_off, "target_row_off", torch.int32),
          _dev(draft, "draft"), _opt(mix_w, "mix_w", torch.float32), K, _dtype_code(draft),
          _dev(tokens, "tokens", torch.int32), _opt(verify_len, "verify_len", torch.int32),
          _dev(u, "u", torch.float32), _dev(g, "g", torch.float32), B, L, V, float(T),
          _dev(acc, "accept_len", torch.int32), _dev(outt, "out_tokens", torch.int32), workspace.ptr(),
          workspace.nbytes, _stream(draft))
    return acc, outt


def dvl_allocate_pack(scores, budget, *, dense_target=None, packed_target=None, workspace=None, out=None):
    """DVL allocation from survival scores [B, L] fp32 under `budget` slots.
    Returns (verify_len [B], offsets [B+1], slot_map [budget]) int32; if
    dense_target [B, L+1, V] and packed_target [budget, V] are given, the
    selected rows are copied into packed_target."""
    _shape(scores, "scores", (None, None))
    B, L = scores.shape
    dev = scores.device
    if out is not None:
        _shape(out[0], "verify_len", (B,))
        _shape(out[1], "offsets", (B + 1,))
        if out[2] is not None and (out[2].dim() != 1 or out[2].numel() < int(budget)):
            raise ValueError("slot_map must be 1-D with at least budget = %d entries" % int(budget))
    if dense_target is not None:
        _shape(dense_target, "dense_target", (B, L + 1, None))
    if packed_target is not None:
        _shape(packed_target, "packed_target", (None, None if dense_target is None else dense_target.shape[-1]))
        if packed_target.shape[0] < int(budget):
            raise ValueError("packed_target has %d rows, fewer than budget = %d" % (packed_target.shape[0], int(budget)))
    ws = workspace or Workspace(dvl_workspace_size(B), dev)
    if out is None:
        out = (torch.empty(B, dtype=torch.int32, device=dev), torch.empty(B + 1, dtype=torch.int32, device=dev),
               torch.empty(max(int(budget), 0), dtype=torch.int32, device=dev))
    vl, off, sm = out
    dptr = pptr = None
    dt, V = 0, 1
    if dense_target is not None or packed_target is not None:
        if dense_target is None or packed_target is None:
            raise ValueError("dense_target and packed_target go together")
        dt, V = _dtype_code(dense_target), dense_target.shape[-1]
        dptr, pptr = _dev(dense_target, "dense_target"), _dev(packed_target, "packed_target", dense_target.dtype)
    _call("dvl_allocate_pack", _dev(scores, "scores", torch.float32), B, L, int(budget),
          _dev(vl, "verify_len", torch.int32), _dev(off, "offsets", torch.int32),
          _opt(sm, "slot_map", torch.int32), dptr, pptr, dt, V, ws.ptr(), ws.nbytes, _stream(scores))
    return vl, off, sm
