"""Python binding of ``libsplitkv.so`` (the C ABI declared in include/splitkv.h).

Argument marshalling only: shapes are read off the tensors, device pointers
and the current CUDA stream are passed through ctypes, and every step of the
computation runs in the library's sm_100a kernels.  PyTorch supplies device
memory (outputs and workspace are allocated with ``torch.empty`` when the
caller does not pass them) and streams.  There is no fallback: if the shared
library is missing or a call fails, an exception is raised.

Entry points (same names as the C ABI):

* ``attn_fwd_lse``        prefill / varlen attention, O and per-row log2 LSE
* ``attn_fwd_lse_chunks`` the partials of several KV chunks in one launch (for merge_state)
* ``attn_splitkv_decode`` split-KV decode (stable per-split online softmax)
* ``merge_state``         merge partial (O, LSE) pairs of disjoint KV ranges
* ``attn_splitkv_plan``, ``attn_splitkv_workspace``, ``attn_splitkv_workspace_init``, ``attn_fwd_lse_workspace``,
  ``attn_varlen_plan``     host-side planning / sizing queries
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence, Tuple

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libsplitkv.so")

SKV_OK, SKV_ERR_INVALID_ARG, SKV_ERR_UNSUPPORTED, SKV_ERR_WORKSPACE_TOO_SMALL, SKV_ERR_CUDA = range(5)
DTYPES = {"bf16": 0, "fp16": 1, "fp32": 2}
LAYOUTS = {"HND": 0, "NHD": 1, "TND": 2}

# (name, restype, argtypes) of every exported symbol
_c_int, _c_float, _c_size, _c_i64, _vp = ctypes.c_int, ctypes.c_float, ctypes.c_size_t, ctypes.c_int64, ctypes.c_void_p
SIGNATURES = {
    "attn_fwd_lse": (_c_int, [_vp, _vp, _vp, _vp, _vp, _c_int, _c_int, _c_int, _c_int, _c_int, _c_int, _c_float,
                              _c_int, _c_int, _vp, _vp, _c_int, _c_int, _c_int, _vp, _c_size, _vp]),
    "attn_fwd_lse_causal": (_c_int, [_vp, _vp, _vp, _vp, _vp, _c_int, _c_int, _c_int, _c_int, _c_int, _c_int,
                                     _c_float, _c_int, _c_int, _vp, _vp, _c_int, _c_int, _c_int, _vp, _c_size, _vp]),
    "attn_fwd_lse_chunks": (_c_int, [_vp, _vp, _vp, _vp, _vp, _c_int, _c_int, _c_int, _c_int, _c_int, _c_int,
                                     _c_float, _c_int, _c_int, _c_int, _vp, _c_int, _vp, _c_size, _vp]),
    "attn_fwd_lse_chunks_workspace": (_c_size, [_c_int, _c_int, _c_int, _c_int, _c_int, _c_int, _c_int, _c_int,
                                                _c_int]),
    "attn_fwd_lse_int8": (_c_int, [_vp, _vp, _vp, _vp, _vp, _c_int, _c_int, _c_int, _c_int, _c_int, _c_int, _c_float,
                                   _c_int, _c_int, _vp, _c_size, _vp]),
    "attn_fwd_lse_int8_workspace": (_c_size, [_c_int, _c_int, _c_int, _c_int, _c_int, _c_int]),
    "attn_fwd_lse_workspace": (_c_size, [_c_int, _c_int, _c_int, _c_int, _c_int, _c_int, _c_int, _c_int]),
    "attn_varlen_plan": (_c_int, [_vp, _vp, _c_int, _c_int, _c_int, _vp, _vp]),
    "attn_splitkv_decode": (_c_int, [_vp, _vp, _vp, _vp, _vp, _c_int, _c_int, _c_int, _c_int, _c_int, _c_int,
                                     _c_float, _c_int, _vp, _c_int, _vp, _c_size, _vp]),
    "attn_splitkv_decode_static": (_c_int, [_vp, _vp, _vp, _vp, _vp, _c_int, _c_int, _c_int, _c_int, _c_int, _c_int,
                                            _c_float, _c_int, _vp, _c_int, _vp]),
    "attn_splitkv_plan": (_c_int, [_c_int, _c_int, _c_int, _c_int, _c_int, _c_int, _c_int, _c_int, _vp, _vp]),
    "attn_splitkv_workspace": (_c_size, [_c_int, _c_int, _c_int, _c_int, _c_int]),
    "attn_splitkv_decode_causal": (_c_int, [_vp, _vp, _vp, _vp, _vp, _c_int, _c_int, _c_int, _c_int, _c_int, _c_int,
                                            _c_float, _c_int, _vp, _c_int, _vp, _c_size, _vp]),
    "attn_splitkv_decode_fused": (_c_int, [_vp, _vp, _vp, _vp, _vp, _c_int, _c_int, _c_int, _c_int, _c_int, _c_int,
                                           _c_float, _c_int, _vp, _c_int, _vp, _c_size, _vp]),
    "attn_splitkv_workspace_init": (_c_int, [_vp, _c_size, _vp]),
    "merge_state": (_c_int, [_vp, _vp, _vp, _vp, _c_int, _c_int, _c_int, _c_int, _c_int, _c_int, _c_int, _c_int,
                             _c_i64, _c_i64, _vp]),
    "skv_status_string": (ctypes.c_char_p, [_c_int]),
    "skv_last_cuda_error": (_c_int, []),
    "skv_device_error": (_c_int, [_vp]),
    "skv_version": (ctypes.c_char_p, []),
    "skv_launch_count": (ctypes.c_uint64, []),
    "skv_exp2_fma": (_c_int, [_vp, _vp, _c_i64, _vp]),
}

_lib = None


class SkvError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        msg = f"{what}: {status_string(status)}"
        if status == SKV_ERR_CUDA:
            msg += f" (cudaError {lib().skv_last_cuda_error()})"
        super().__init__(msg)


def lib() -> ctypes.CDLL:
    """The loaded shared library (loaded once, on first use)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m split_kv_merge_attn_b200._build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().skv_status_string(int(status)).decode()


def _check(status: int, what: str) -> None:
    if status != SKV_OK:
        raise SkvError(status, what)


# ------------------------------------------------------------------ helpers

def _torch():
    import torch
    return torch


def _dtype_code(t) -> int:
    torch = _torch()
    m = {torch.bfloat16: 0, torch.float16: 1, torch.float32: 2}
    if t.dtype not in m:
        raise TypeError(f"unsupported dtype {t.dtype}")
    return m[t.dtype]


def _ptr(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(stream, device) -> Optional[int]:
    torch = _torch()
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return stream.cuda_stream


def _need_cuda(*ts):
    for t in ts:
        if t is not None:
            if not t.is_cuda:
                raise ValueError("tensors must be on a CUDA device")
            if not t.is_contiguous():
                raise ValueError("tensors must be contiguous")


def _expect(cond: bool, msg: str) -> None:
    if not cond:
        raise ValueError(msg)


def _consistent(q, named, *, same_dtype=(), fp32=(), int32=()):
    """Shape-independent consistency of the tensors of one call, checked before
    anything reaches the library (which sees only q's dtype and the sizes read
    off q and k): every tensor on q's device, the named 16-bit operands in q's
    dtype, LSE buffers fp32, index arrays int32.  `named` maps names to
    tensors (None entries are skipped)."""
    torch = _torch()
    for name, t in named.items():
        if t is None:
            continue
        _expect(t.device == q.device, f"{name} is on {t.device}, q on {q.device}")
        if name in same_dtype:
            _expect(t.dtype == q.dtype, f"{name} has dtype {t.dtype}, q has {q.dtype}")
        if name in fp32:
            _expect(t.dtype == torch.float32, f"{name} must be float32, got {t.dtype}")
        if name in int32:
            _expect(t.dtype == torch.int32, f"{name} must be int32, got {t.dtype}")


def _shape(t, shape, name: str) -> None:
    if t is not None:
        _expect(tuple(t.shape) == tuple(shape), f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")


def _workspace(nbytes: int, device, workspace):
    torch = _torch()
    if nbytes == 0:
        return workspace, (workspace.numel() * workspace.element_size() if workspace is not None else 0)
    if workspace is None:
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=device)
    return workspace, workspace.numel() * workspace.element_size()


# ------------------------------------------------------------------ queries

def attn_splitkv_plan(B: int, Hq: int, Hkv: int, Lq: int, n: int, D: int = 128, num_sms: int = 148,
                      requested_splits: int = 0) -> Tuple[int, list]:
    """Host split plan: (num_splits, bounds[num_splits + 1])."""
    ns = ctypes.c_int(0)
    _check(lib().attn_splitkv_plan(B, Hq, Hkv, Lq, n, D, num_sms, requested_splits, ctypes.byref(ns), None),
           "attn_splitkv_plan")
    bounds = (ctypes.c_int32 * (ns.value + 1))()
    _check(lib().attn_splitkv_plan(B, Hq, Hkv, Lq, n, D, num_sms, requested_splits, ctypes.byref(ns), bounds),
           "attn_splitkv_plan")
    return ns.value, list(bounds)


def attn_splitkv_workspace(B: int, Hq: int, Lq: int, D: int, num_splits: int) -> int:
    return int(lib().attn_splitkv_workspace(B, Hq, Lq, D, num_splits))


def attn_fwd_lse_workspace(B: int, Hq: int, Hkv: int, Sk: int, D: int, dtype: str = "bf16",
                           layout: str = "HND", smooth_k: int = 0) -> int:
    return int(lib().attn_fwd_lse_workspace(B, Hq, Hkv, Sk, D, DTYPES[dtype], LAYOUTS[layout], int(smooth_k)))


def attn_varlen_plan(cu_seqlens_q: Sequence[int], cu_seqlens_k: Sequence[int], Hq: int,
                     D: int = 128) -> Tuple[list, list]:
    """Host restatement of the device varlen work order: (order[B], offsets[B+1])
    for head dimension D (256 query rows per CTA for D <= 128, 128 for D = 256)."""
    B = len(cu_seqlens_q) - 1
    cq = (ctypes.c_int32 * (B + 1))(*[int(x) for x in cu_seqlens_q])
    ck = (ctypes.c_int32 * (B + 1))(*[int(x) for x in cu_seqlens_k])
    order = (ctypes.c_int32 * max(B, 1))()
    offsets = (ctypes.c_int32 * (B + 1))()
    _check(lib().attn_varlen_plan(cq, ck, B, Hq, D, order, offsets), "attn_varlen_plan")
    return list(order)[:B], list(offsets)


def launch_count() -> int:
    """Kernels launched by the library in this process so far."""
    return int(lib().skv_launch_count())


def exp2_fma(x, stream=None):
    """The prefill softmax's FMA-pipe exp2, elementwise on a float32 CUDA tensor (diagnostics)."""
    torch = _torch()
    _need_cuda(x)
    _expect(x.dtype == torch.float32, "x must be float32")
    y = torch.empty_like(x)
    _check(lib().skv_exp2_fma(_ptr(x), _ptr(y), x.numel(), _stream(stream, x.device)), "skv_exp2_fma")
    return y


def device_error() -> int:
    """Reads and clears the device error word (synchronises the device)."""
    code = ctypes.c_int(0)
    _check(lib().skv_device_error(ctypes.byref(code)), "skv_device_error")
    return code.value


# ------------------------------------------------------------------ operations

def attn_fwd_lse(q, k, v, scale: Optional[float] = None, layout: str = "HND", cu_seqlens_q=None,
                 cu_seqlens_k=None, max_seqlen_q: Optional[int] = None, max_seqlen_k: Optional[int] = None,
                 smooth_k: int = 0, out=None, lse=None, return_lse: bool = True, workspace=None, stream=None,
                 causal: bool = False):
    """Attention forward with one log2 LSE per query row.

    Dense: q [B,Hq,Sq,D] (HND) or [B,Sq,Hq,D] (NHD), k/v likewise with Hkv, Sk.
    Varlen (layout "TND"): q [total_q,Hq,D], k/v [total_k,Hkv,D], int32 device
    cu_seqlens_q/k of B+1 entries.  Returns (out, lse) with lse [B,Hq,Sq]
    (dense) or [Hq,total_q] (varlen), or (out, None) if return_lse is False.
    smooth_k: 0 off; 1 mean-shift applied to the fp32 logits; 2 K' = K - mean
    materialised in the input type.  Both return the LSE of the original logits.
    causal: attn_fwd_lse_causal (query row i sees keys j <= i + len_k - len_q).
    """
    torch = _torch()
    _consistent(q, {"k": k, "v": v, "out": out, "lse": lse, "cu_seqlens_q": cu_seqlens_q,
                    "cu_seqlens_k": cu_seqlens_k}, same_dtype=("k", "v", "out"), fp32=("lse",),
                int32=("cu_seqlens_q", "cu_seqlens_k"))
    if layout == "TND":
        if cu_seqlens_q is None or cu_seqlens_k is None:
            raise ValueError("TND layout needs cu_seqlens_q and cu_seqlens_k")
        _expect(q.dim() == 3 and k.dim() == 3, "TND tensors are [tokens, heads, D]")
        Tq, Hq, D = q.shape
        Tk, Hkv, _ = k.shape
        B = cu_seqlens_q.numel() - 1
        _expect(cu_seqlens_k.numel() == B + 1, "cu_seqlens_q and cu_seqlens_k must have the same length")
        Sq, Sk = Tq, Tk
        if max_seqlen_q is None or max_seqlen_k is None:
            raise ValueError("TND layout needs max_seqlen_q and max_seqlen_k")
        lse_shape = (Hq, Tq)
        k_shape = (Tk, Hkv, D)
    else:
        _expect(q.dim() == 4 and k.dim() == 4, f"{layout} tensors are 4-D")
        if layout == "HND":
            B, Hq, Sq, D = q.shape
            _, Hkv, Sk, _ = k.shape
            k_shape = (B, Hkv, Sk, D)
        elif layout == "NHD":
            B, Sq, Hq, D = q.shape
            _, Sk, Hkv, _ = k.shape
            k_shape = (B, Sk, Hkv, D)
        else:
            raise ValueError(layout)
        max_seqlen_q = max_seqlen_q or 0
        max_seqlen_k = max_seqlen_k or 0
        lse_shape = (B, Hq, Sq)
    _shape(k, k_shape, "k")
    _shape(v, k_shape, "v")
    _shape(out, q.shape, "out")
    _shape(lse, lse_shape, "lse")
    _need_cuda(q, k, v, out, lse, cu_seqlens_q, cu_seqlens_k)
    if scale is None:
        scale = D ** -0.5
    if out is None:
        out = torch.empty_like(q)
    if return_lse and lse is None:
        lse = torch.empty(lse_shape, dtype=torch.float32, device=q.device)
    if not return_lse:
        lse = None
    nbytes = attn_fwd_lse_workspace(B, Hq, Hkv, Sk, D, {0: "bf16", 1: "fp16", 2: "fp32"}[_dtype_code(q)],
                                    layout, smooth_k)
    workspace, wbytes = _workspace(nbytes, q.device, workspace)
    fn = lib().attn_fwd_lse_causal if causal else lib().attn_fwd_lse
    st = fn(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, Hq, Hkv, Sq, Sk, D, float(scale), _dtype_code(q),
            LAYOUTS[layout], _ptr(cu_seqlens_q), _ptr(cu_seqlens_k), int(max_seqlen_q), int(max_seqlen_k),
            int(smooth_k), _ptr(workspace), wbytes, _stream(stream, q.device))
    _check(st, "attn_fwd_lse_causal" if causal else "attn_fwd_lse")
    return out, lse


def attn_fwd_lse_chunks_workspace(B: int, Hq: int, Hkv: int, Sk: int, D: int, num_chunks: int, dtype: str = "bf16",
                                  layout: str = "HND", smooth_k: int = 0) -> int:
    return int(lib().attn_fwd_lse_chunks_workspace(B, Hq, Hkv, Sk, D, DTYPES[dtype], LAYOUTS[layout], num_chunks,
                                                   int(smooth_k)))


def attn_fwd_lse_chunks(q, k, v, chunk_bounds: Sequence[int], scale: Optional[float] = None, layout: str = "HND",
                        smooth_k: int = 0, out=None, lse=None, return_lse: bool = True, workspace=None, stream=None):
    """Partial (O, LSE) of q over each KV chunk [chunk_bounds[c], chunk_bounds[c+1])
    in one launch (dense HND / NHD, non-causal).  Returns (out [C, *q.shape],
    lse [C, B, Hq, Sq]); merge_state of the C parts gives attention over all keys.
    With smooth_k each chunk is smoothed by its own mean (LSE of the original logits)."""
    torch = _torch()
    _consistent(q, {"k": k, "v": v, "out": out, "lse": lse}, same_dtype=("k", "v", "out"), fp32=("lse",))
    _expect(q.dim() == 4 and k.dim() == 4, f"{layout} tensors are 4-D")
    if layout == "HND":
        B, Hq, Sq, D = q.shape
        _, Hkv, Sk, _ = k.shape
        k_shape = (B, Hkv, Sk, D)
    elif layout == "NHD":
        B, Sq, Hq, D = q.shape
        _, Sk, Hkv, _ = k.shape
        k_shape = (B, Sk, Hkv, D)
    else:
        raise ValueError(f"attn_fwd_lse_chunks takes HND or NHD, not {layout}")
    C = len(chunk_bounds) - 1
    _expect(C >= 1, "chunk_bounds needs at least two entries")
    _shape(k, k_shape, "k")
    _shape(v, k_shape, "v")
    _shape(out, (C,) + tuple(q.shape), "out")
    _shape(lse, (C, B, Hq, Sq), "lse")
    _need_cuda(q, k, v, out, lse)
    if scale is None:
        scale = D ** -0.5
    if out is None:
        out = torch.empty((C,) + tuple(q.shape), dtype=q.dtype, device=q.device)
    if return_lse and lse is None:
        lse = torch.empty((C, B, Hq, Sq), dtype=torch.float32, device=q.device)
    if not return_lse:
        lse = None
    nbytes = attn_fwd_lse_chunks_workspace(B, Hq, Hkv, Sk, D, C, {0: "bf16", 1: "fp16", 2: "fp32"}[_dtype_code(q)],
                                           layout, smooth_k)
    workspace, wbytes = _workspace(nbytes, q.device, workspace)
    bounds = (ctypes.c_int32 * (C + 1))(*[int(x) for x in chunk_bounds])
    st = lib().attn_fwd_lse_chunks(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, Hq, Hkv, Sq, Sk, D,
                                   float(scale), _dtype_code(q), LAYOUTS[layout], C, bounds, int(smooth_k),
                                   _ptr(workspace), wbytes, _stream(stream, q.device))
    _check(st, "attn_fwd_lse_chunks")
    return out, lse


def attn_fwd_lse_int8_workspace(B: int, Hq: int, Hkv: int, Sq: int, Sk: int, D: int = 128) -> int:
    return int(lib().attn_fwd_lse_int8_workspace(B, Hq, Hkv, Sq, Sk, D))


def attn_fwd_lse_int8(q, k, v, scale: Optional[float] = None, causal: bool = False, out=None, lse=None,
                      return_lse: bool = True, workspace=None, stream=None):
    """Attention with Q K'^T from INT8 codes of Q and of the smoothed K
    (dense HND, D = 128).  Returns (out, lse [B,Hq,Sq])."""
    torch = _torch()
    _consistent(q, {"k": k, "v": v, "out": out, "lse": lse}, same_dtype=("k", "v", "out"), fp32=("lse",))
    _expect(q.dim() == 4 and k.dim() == 4, "HND tensors are 4-D")
    B, Hq, Sq, D = q.shape
    _, Hkv, Sk, _ = k.shape
    _shape(k, (B, Hkv, Sk, D), "k")
    _shape(v, (B, Hkv, Sk, D), "v")
    _shape(out, q.shape, "out")
    _shape(lse, (B, Hq, Sq), "lse")
    _need_cuda(q, k, v, out, lse)
    if scale is None:
        scale = D ** -0.5
    if out is None:
        out = torch.empty_like(q)
    if return_lse and lse is None:
        lse = torch.empty((B, Hq, Sq), dtype=torch.float32, device=q.device)
    if not return_lse:
        lse = None
    workspace, wbytes = _workspace(attn_fwd_lse_int8_workspace(B, Hq, Hkv, Sq, Sk, D), q.device, workspace)
    st = lib().attn_fwd_lse_int8(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, Hq, Hkv, Sq, Sk, D,
                                 float(scale), _dtype_code(q), int(bool(causal)), _ptr(workspace), wbytes,
                                 _stream(stream, q.device))
    _check(st, "attn_fwd_lse_int8")
    return out, lse


def attn_splitkv_workspace_init(workspace, stream=None):
    """Zeroes a decode workspace (uint8 device tensor) on `stream`: needed once
    before its first use by attn_splitkv_decode(..., fused=True)."""
    nbytes = workspace.numel() * workspace.element_size()
    _check(lib().attn_splitkv_workspace_init(_ptr(workspace), nbytes, _stream(stream, workspace.device)),
           "attn_splitkv_workspace_init")
    return workspace


def attn_splitkv_decode(q, k, v, scale: Optional[float] = None, kv_len=None, num_splits: int = 0, out=None,
                        lse=None, return_lse: bool = True, workspace=None, stream=None, fused: bool = False,
                        causal: bool = False):
    """Split-KV decode: q [B,Hq,Lq,D], k/v [B,Hkv,Lkv,D] (HND).  kv_len: optional
    int32 device tensor [B].  num_splits 0 = automatic.  Returns (out, lse).
    fused=True: one kernel launch, the splits merged by the last CTA of each
    group (attn_splitkv_decode_fused); a workspace passed in must have been
    zeroed once (attn_splitkv_workspace_init), one allocated here is zeroed.
    causal=True: attn_splitkv_decode_causal (row i of Lq sees the first
    kv_len - Lq + 1 + i keys); not combined with fused."""
    if fused and causal:
        raise ValueError("the single-launch decode has no causal variant")
    torch = _torch()
    _consistent(q, {"k": k, "v": v, "out": out, "lse": lse, "kv_len": kv_len}, same_dtype=("k", "v", "out"),
                fp32=("lse",), int32=("kv_len",))
    _expect(q.dim() == 4 and k.dim() == 4, "decode tensors are [B, H, L, D]")
    B, Hq, Lq, D = q.shape
    _, Hkv, Lkv, _ = k.shape
    _shape(k, (B, Hkv, Lkv, D), "k")
    _shape(v, (B, Hkv, Lkv, D), "v")
    _shape(out, q.shape, "out")
    _shape(lse, (B, Hq, Lq), "lse")
    _shape(kv_len, (B,), "kv_len")
    _need_cuda(q, k, v, out, lse, kv_len)
    if scale is None:
        scale = D ** -0.5
    if out is None:
        out = torch.empty_like(q)
    if return_lse and lse is None:
        lse = torch.empty((B, Hq, Lq), dtype=torch.float32, device=q.device)
    if not return_lse:
        lse = None
    splits = num_splits
    if splits == 0:
        sms = torch.cuda.get_device_properties(q.device).multi_processor_count
        splits, _ = attn_splitkv_plan(B, Hq, Hkv, Lq, Lkv, D, sms, 0)
    nbytes = attn_splitkv_workspace(B, Hq, Lq, D, splits)
    fresh = workspace is None and nbytes > 0
    workspace, wbytes = _workspace(nbytes, q.device, workspace)
    if fused and fresh:
        attn_splitkv_workspace_init(workspace, stream)
    fn = lib().attn_splitkv_decode_fused if fused else (
        lib().attn_splitkv_decode_causal if causal else lib().attn_splitkv_decode)
    st = fn(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, Hq, Hkv, Lq, Lkv, D, float(scale), _dtype_code(q),
            _ptr(kv_len), int(splits), _ptr(workspace), wbytes, _stream(stream, q.device))
    _check(st, "attn_splitkv_decode_fused" if fused else (
        "attn_splitkv_decode_causal" if causal else "attn_splitkv_decode"))
    return out, lse


def attn_splitkv_decode_static(q, k, v, scale: Optional[float] = None, kv_len=None, num_splits: int = 0,
                               out=None, lse=None, return_lse: bool = True, stream=None):
    """attn_splitkv_decode for callers that cannot allocate device memory: the
    per-split partials live in the library's fixed 8 MiB device array (no
    workspace).  This wrapper allocates out/lse only if they are not given.

    The array is looked up on the device of q (made current for the call) the
    first time a device is used: make that first call before any stream
    capture.  Every call on a device shares the one array, so calls that
    overlap on the GPU (several streams or host threads) race on it and must
    be serialised by the caller.  Problems whose partials need more than
    8 MiB raise with SKV_ERR_WORKSPACE_TOO_SMALL."""
    torch = _torch()
    _consistent(q, {"k": k, "v": v, "out": out, "lse": lse, "kv_len": kv_len}, same_dtype=("k", "v", "out"),
                fp32=("lse",), int32=("kv_len",))
    _expect(q.dim() == 4 and k.dim() == 4, "decode tensors are [B, H, L, D]")
    B, Hq, Lq, D = q.shape
    _, Hkv, Lkv, _ = k.shape
    _shape(k, (B, Hkv, Lkv, D), "k")
    _shape(v, (B, Hkv, Lkv, D), "v")
    _shape(out, q.shape, "out")
    _shape(lse, (B, Hq, Lq), "lse")
    _shape(kv_len, (B,), "kv_len")
    _need_cuda(q, k, v, out, lse, kv_len)
    if scale is None:
        scale = D ** -0.5
    if out is None:
        out = torch.empty_like(q)
    if return_lse and lse is None:
        lse = torch.empty((B, Hq, Lq), dtype=torch.float32, device=q.device)
    if not return_lse:
        lse = None
    with torch.cuda.device(q.device):  # the scratch array is looked up on the current device
        st = lib().attn_splitkv_decode_static(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, Hq, Hkv, Lq, Lkv,
                                              D, float(scale), _dtype_code(q), _ptr(kv_len), int(num_splits),
                                              _stream(stream, q.device))
    _check(st, "attn_splitkv_decode_static")
    return out, lse


def merge_state(o_parts, lse_parts, layout: str = "HND", out=None, lse=None, out_dtype=None,
                return_lse: bool = True, stream=None):
    """Merge P partial results.  o_parts [P,B,H,S,D] (HND), [P,B,S,H,D] (NHD)
    or [P,T,H,D] (TND); lse_parts [P,B,H,S] or [P,H,T] (fp32).  Returns (out, lse)."""
    torch = _torch()
    _consistent(o_parts, {"lse_parts": lse_parts, "out": out, "lse": lse}, fp32=("lse_parts", "lse"))
    P = o_parts.shape[0]
    if layout == "HND":
        _expect(o_parts.dim() == 5, "HND o_parts is [P, B, H, S, D]")
        _, B, H, S, D = o_parts.shape
        lse_shape = (P, B, H, S)
    elif layout == "NHD":
        _expect(o_parts.dim() == 5, "NHD o_parts is [P, B, S, H, D]")
        _, B, S, H, D = o_parts.shape
        lse_shape = (P, B, H, S)
    elif layout == "TND":
        _expect(o_parts.dim() == 4, "TND o_parts is [P, T, H, D]")
        _, S, H, D = o_parts.shape
        B = 1
        lse_shape = (P, H, S)
    else:
        raise ValueError(layout)
    _shape(lse_parts, lse_shape, "lse_parts")
    _shape(out, o_parts.shape[1:], "out")
    _shape(lse, lse_shape[1:], "lse")
    _need_cuda(o_parts, lse_parts, out, lse)
    if out is None:
        out = torch.empty(o_parts.shape[1:], dtype=out_dtype or o_parts.dtype, device=o_parts.device)
    if return_lse and lse is None:
        lse = torch.empty(lse_parts.shape[1:], dtype=torch.float32, device=o_parts.device)
    if not return_lse:
        lse = None
    st = lib().merge_state(_ptr(o_parts), _ptr(lse_parts), _ptr(out), _ptr(lse), P, B, H, S, D, LAYOUTS[layout],
                           _dtype_code(o_parts), _dtype_code(out), 0, 0, _stream(stream, o_parts.device))
    _check(st, "merge_state")
    return out, lse


__all__ = ["attn_fwd_lse", "attn_fwd_lse_chunks", "attn_fwd_lse_chunks_workspace", "attn_fwd_lse_int8", "attn_splitkv_decode", "attn_splitkv_decode_static", "merge_state",
           "attn_splitkv_plan", "attn_splitkv_workspace", "attn_splitkv_workspace_init", "attn_fwd_lse_workspace",
           "attn_fwd_lse_int8_workspace", "attn_varlen_plan", "device_error", "launch_count", "lib", "SkvError",
           "status_string", "LIB_PATH", "SIGNATURES"]
