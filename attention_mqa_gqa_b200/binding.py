"""ctypes binding of ``libattn_b200.so`` (declared in ``include/attn_b200.h``).

Argument marshalling only: every step of the attention runs in the CUDA
library.  Torch tensors supply device pointers, strides and the stream; the
library must be built (``python -m attention_mqa_gqa_b200.build``) and a
missing library is an error, never a fallback.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libattn_b200.so")

(ATTN_OK, ATTN_EINVAL, ATTN_EUNSUPPORTED, ATTN_EWORKSPACE, ATTN_ECUDA, ATTN_ETIMEOUT,
 ATTN_EOVERFLOW, ATTN_EINDEX) = range(8)
ATTN_BF16, ATTN_FP16 = 0, 1


class Strides(ctypes.Structure):
    _fields_ = [("b", ctypes.c_int64), ("h", ctypes.c_int64), ("s", ctypes.c_int64)]


class Plan(ctypes.Structure):
    _fields_ = [("path", ctypes.c_int), ("heads_per_cta", ctypes.c_int),
                ("head_blocks", ctypes.c_int), ("kv_ranges", ctypes.c_int),
                ("partials", ctypes.c_int64), ("dv_parts", ctypes.c_int),
                ("grid_ctas", ctypes.c_int64), ("workspace_bytes", ctypes.c_size_t)]

    def as_dict(self) -> dict:
        return {f: getattr(self, f) for f, _ in self._fields_}


class AttnError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = status
        super().__init__(f"{what}: {status_str(status)} ({status})" if what else status_str(status))


# Every symbol include/attn_b200.h declares (checked by the CPU test suite).
EXPORTS = ("attn_plan", "attn_workspace_bytes", "attn_fwd", "attn_decode_partial",
           "attn_decode_combine", "attn_fwd_noalloc", "attn_last_device_error", "attn_status_str",
           "attn_version", "attn_set_wait_timeout_ns", "attn_cache_append",
           "attn_gather_rows", "attn_topk_fwd")
NOALLOC_SCRATCH_BYTES = 32 << 20  # ATTN_NOALLOC_SCRATCH_BYTES in the header

_lib = None


def load(path: str | None = None):
    """Load the library (once).  Raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    path = path or LIB_PATH
    if not os.path.exists(path):
        raise RuntimeError(f"CUDA library not built: {path} is missing "
                           "(run python -m attention_mqa_gqa_b200.build)")
    lib = ctypes.CDLL(path)
    i32, i64, sz, vp = ctypes.c_int, ctypes.c_int64, ctypes.c_size_t, ctypes.c_void_p
    lib.attn_plan.restype = i32
    lib.attn_plan.argtypes = [i32, i32, i32, i32, i32, i32, i32, i32, i32, ctypes.POINTER(Plan)]
    lib.attn_workspace_bytes.restype = sz
    lib.attn_workspace_bytes.argtypes = [i32] * 7
    for fn in (lib.attn_fwd, lib.attn_decode_partial, lib.attn_decode_combine):
        fn.restype = i32
        fn.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, vp, i32, i32, i32,
                       ctypes.c_float, i32, i32, Strides, Strides, Strides, Strides, vp, sz, vp]
    lib.attn_fwd_noalloc.restype = i32
    lib.attn_fwd_noalloc.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, vp, i32, i32, i32,
                                     ctypes.c_float, i32, i32, Strides, Strides, Strides,
                                     Strides, vp]
    lib.attn_cache_append.restype = i32
    lib.attn_cache_append.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, Strides,
                                      Strides, Strides, Strides, vp]
    lib.attn_gather_rows.restype = i32
    lib.attn_gather_rows.argtypes = [vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, Strides,
                                     Strides, i64, vp]
    lib.attn_topk_fwd.restype = i32
    lib.attn_topk_fwd.argtypes = [vp, vp, vp, vp, i32, i32, vp, i64, vp, vp, i32, i32, i32, i32,
                                  ctypes.c_float, i32, Strides, Strides, Strides, vp, sz, vp]
    lib.attn_set_wait_timeout_ns.restype = ctypes.c_uint64
    lib.attn_set_wait_timeout_ns.argtypes = [ctypes.c_uint64]
    lib.attn_last_device_error.restype = i32
    lib.attn_last_device_error.argtypes = [vp]
    lib.attn_status_str.restype = ctypes.c_char_p
    lib.attn_status_str.argtypes = [i32]
    lib.attn_version.restype = ctypes.c_char_p
    lib.attn_version.argtypes = []
    _lib = lib
    return lib


def status_str(status: int) -> str:
    return load().attn_status_str(int(status)).decode()


def version() -> str:
    return load().attn_version().decode()


def dtype_code(dt: torch.dtype) -> int:
    if dt == torch.bfloat16:
        return ATTN_BF16
    if dt == torch.float16:
        return ATTN_FP16
    raise TypeError(f"unsupported element type {dt}")


def plan(B, Hq, Hkv, Sq, max_skv, d_k, d_v, dtype=torch.bfloat16, num_sms: int = 0) -> dict:
    pl = Plan()
    code = dtype_code(dtype) if isinstance(dtype, torch.dtype) else int(dtype)
    rc = load().attn_plan(B, Hq, Hkv, Sq, max_skv, d_k, d_v, code, num_sms, ctypes.byref(pl))
    if rc != ATTN_OK:
        raise AttnError(rc, "attn_plan")
    return pl.as_dict()


def workspace_bytes(B, Hq, Hkv, Sq, max_skv, d_k, d_v) -> int:
    return int(load().attn_workspace_bytes(B, Hq, Hkv, Sq, max_skv, d_k, d_v))


def _on_one_gpu(*tensors) -> None:
    """Every tensor handed to the library is CUDA memory of one device (a
    host pointer reaching a kernel would be an illegal access)."""
    ts = [t for t in tensors if t is not None]
    for t in ts:
        if not t.is_cuda:
            raise ValueError("all tensors must be CUDA tensors")
    if len({t.device for t in ts}) > 1:
        raise ValueError("all tensors must be on the same CUDA device")


def _strides4(t: torch.Tensor) -> Strides:
    if t.dim() != 4 or t.stride(-1) != 1:
        raise ValueError("expected a [B, H, S, d] tensor with a contiguous last dimension")
    return Strides(t.stride(0), t.stride(1), t.stride(2))


def fwd_raw(q, k, v, out, lse, B, Hq, Hkv, Sq, skv_ptr, max_skv, d_k, d_v, scale, causal,
            dtype_code_, sq: Strides, sk: Strides, sv: Strides, so: Strides,
            workspace_ptr, workspace_nbytes, stream_ptr, entry: str = "attn_fwd") -> int:
    """Direct call with raw pointers (ints); returns the status code.
    ``entry`` selects attn_fwd, attn_decode_partial or attn_decode_combine."""
    fn = getattr(load(), entry)
    return fn(q, k, v, out, lse, B, Hq, Hkv, Sq, skv_ptr, max_skv, d_k, d_v, float(scale),
              int(causal), dtype_code_, sq, sk, sv, so, workspace_ptr, workspace_nbytes,
              stream_ptr)


def topk_raw(*args) -> int:
    """attn_topk_fwd with raw pointers (ints), in the header's argument
    order; returns the status code."""
    return load().attn_topk_fwd(*args)


def attn_fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, out: torch.Tensor,
             skv: torch.Tensor, max_skv: int, scale: float, causal: bool = True,
             lse: torch.Tensor | None = None, workspace: torch.Tensor | None = None,
             stream: torch.cuda.Stream | None = None) -> None:
    """Enqueue the forward on ``stream`` (default: torch's current stream).

    q [B,Hq,Sq,d_k], k [B,Hkv,S,d_k], v [B,Hkv,S,d_v], out [B,Hq,Sq,d_v]
    (device tensors, last dim contiguous, any 16-byte-aligned strides);
    skv int32 [B] device; lse fp32 [B,Hq,Sq] contiguous or None; workspace a
    device byte tensor of at least ``workspace_bytes(...)`` bytes."""
    B, Hq, Sq, d_k = q.shape
    Hkv, d_v = k.shape[1], v.shape[-1]
    if skv.dtype != torch.int32:
        raise TypeError("skv must be int32")
    if lse is not None and (lse.dtype != torch.float32 or not lse.is_contiguous()):
        raise TypeError("lse must be a contiguous float32 tensor")
    _on_one_gpu(q, k, v, out, skv, lse, workspace)
    st = stream if stream is not None else torch.cuda.current_stream(q.device)
    ws_ptr = workspace.data_ptr() if workspace is not None else None
    ws_n = workspace.numel() * workspace.element_size() if workspace is not None else 0
    with torch.cuda.device(q.device):  # the launch plan is made for the current device
        rc = fwd_raw(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                     lse.data_ptr() if lse is not None else None,
                     B, Hq, Hkv, Sq, skv.data_ptr(), int(max_skv), d_k, d_v, scale, causal,
                     dtype_code(q.dtype), _strides4(q), _strides4(k), _strides4(v),
                     _strides4(out), ws_ptr, ws_n, st.cuda_stream)
    if rc != ATTN_OK:
        raise AttnError(rc, "attn_fwd")


def attn_fwd_noalloc(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, out: torch.Tensor,
                     skv: torch.Tensor, max_skv: int, scale: float, causal: bool = True,
                     lse: torch.Tensor | None = None,
                     stream: torch.cuda.Stream | None = None) -> None:
    """Like :func:`attn_fwd` but without a workspace: the library's built-in
    scratch buffer is used (for callers that cannot allocate device memory;
    see the header).  Calls sharing the buffer must not overlap on the GPU."""
    B, Hq, Sq, d_k = q.shape
    Hkv, d_v = k.shape[1], v.shape[-1]
    if skv.dtype != torch.int32:
        raise TypeError("skv must be int32")
    if lse is not None and (lse.dtype != torch.float32 or not lse.is_contiguous()):
        raise TypeError("lse must be a contiguous float32 tensor")
    _on_one_gpu(q, k, v, out, skv, lse)
    st = stream if stream is not None else torch.cuda.current_stream(q.device)
    with torch.cuda.device(q.device):  # the library takes its scratch from the current device
        rc = load().attn_fwd_noalloc(
            q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
            lse.data_ptr() if lse is not None else None, B, Hq, Hkv, Sq, skv.data_ptr(),
            int(max_skv), d_k, d_v, float(scale), int(causal), dtype_code(q.dtype),
            _strides4(q), _strides4(k), _strides4(v), _strides4(out), st.cuda_stream)
    if rc != ATTN_OK:
        raise AttnError(rc, "attn_fwd_noalloc")


def last_device_error(stream: torch.cuda.Stream | None = None) -> int:
    st = stream if stream is not None else torch.cuda.current_stream()
    return int(load().attn_last_device_error(st.cuda_stream))


def cache_append(k_cache: torch.Tensor, v_cache: torch.Tensor | None, k_new: torch.Tensor,
                 v_new: torch.Tensor | None, skv: torch.Tensor,
                 stream: torch.cuda.Stream | None = None) -> None:
    """attn_cache_append: write k_new[b, h] (and v_new[b, h]) at position
    skv[b] of the caches and advance skv (device-side).  k_cache/v_cache are
    [B, Hkv, max_skv, d] (views allowed); for an MLA latent cache pass the
    same tensor (or None) as v_cache.  k_new/v_new are [B, Hkv, 1, d]."""
    B, Hkv, max_skv, d_k = k_cache.shape
    if skv.dtype != torch.int32:
        raise TypeError("skv must be int32")
    _on_one_gpu(k_cache, v_cache, k_new, v_new, skv)
    latent = v_cache is None or v_cache.data_ptr() == k_cache.data_ptr()
    d_v = 0 if latent else v_cache.shape[-1]
    st = stream if stream is not None else torch.cuda.current_stream(k_cache.device)
    zero = Strides(0, 0, 0)
    rc = load().attn_cache_append(k_cache.data_ptr(), None if latent else v_cache.data_ptr(),
                                  k_new.data_ptr(), None if latent else v_new.data_ptr(),
                                  skv.data_ptr(), B, Hkv, max_skv, d_k, d_v,
                                  dtype_code(k_cache.dtype), _strides4(k_cache),
                                  zero if latent else _strides4(v_cache), _strides4(k_new),
                                  zero if latent else _strides4(v_new), st.cuda_stream)
    if rc != ATTN_OK:
        raise AttnError(rc, "attn_cache_append")


def gather_rows(src: torch.Tensor, dst: torch.Tensor, idx: torch.Tensor, n_sel: torch.Tensor,
                skv: torch.Tensor, dst_len: torch.Tensor,
                stream: torch.cuda.Stream | None = None) -> None:
    """attn_gather_rows: dst[b, h, t] = src[b, h, idx[b, t]] for t < n_sel[b],
    dst_len[b] = n_sel[b] (device-side).  src [B, H, S, d] and dst
    [B, H, topk, d] (views allowed, last dim contiguous); idx int32
    [B, >= topk] (last dim contiguous); n_sel, skv, dst_len int32 [B]."""
    B, H, topk, d = dst.shape
    for t in (idx, n_sel, skv, dst_len):
        if t.dtype != torch.int32:
            raise TypeError("idx, n_sel, skv and dst_len must be int32")
    if idx.dim() != 2 or idx.stride(1) != 1 or not n_sel.is_contiguous() \
            or not skv.is_contiguous() or not dst_len.is_contiguous():
        raise ValueError("idx rows and n_sel/skv/dst_len must be contiguous")
    if src.dtype != dst.dtype:
        raise TypeError("src and dst must have the same element type")
    _on_one_gpu(src, dst, idx, n_sel, skv, dst_len)
    st = stream if stream is not None else torch.cuda.current_stream(dst.device)
    rc = load().attn_gather_rows(src.data_ptr(), dst.data_ptr(), idx.data_ptr(), n_sel.data_ptr(),
                                 skv.data_ptr(), dst_len.data_ptr(), B, H, topk, d,
                                 dtype_code(dst.dtype), _strides4(src), _strides4(dst),
                                 idx.stride(0), st.cuda_stream)
    if rc != ATTN_OK:
        raise AttnError(rc, "attn_gather_rows")


def topk_fwd(q: torch.Tensor, cache: torch.Tensor, out: torch.Tensor, idx: torch.Tensor,
             n_sel: torch.Tensor, skv: torch.Tensor, scale: float, lse: torch.Tensor | None,
             workspace: torch.Tensor, stream: torch.cuda.Stream | None = None) -> None:
    """attn_topk_fwd: absorbed-MLA decode over the cache rows at idx[b, t],
    t < n_sel[b], gathered inside the kernel.  q [B, Hq, 1, 576], cache
    [B, 1, S, 576], out [B, Hq, 1, 512] (views allowed, last dim contiguous);
    idx int32 [B, >= topk] with topk = idx.shape[1]; n_sel, skv int32 [B]."""
    B, Hq, _, d_k = q.shape
    topk = idx.shape[1]
    for t in (idx, n_sel, skv):
        if t.dtype != torch.int32:
            raise TypeError("idx, n_sel and skv must be int32")
    if idx.dim() != 2 or idx.stride(1) != 1 or not n_sel.is_contiguous() or not skv.is_contiguous():
        raise ValueError("idx rows and n_sel/skv must be contiguous")
    if lse is not None and (lse.dtype != torch.float32 or not lse.is_contiguous()):
        raise TypeError("lse must be a contiguous float32 tensor")
    _on_one_gpu(q, cache, out, idx, n_sel, skv, lse, workspace)
    st = stream if stream is not None else torch.cuda.current_stream(q.device)
    rc = load().attn_topk_fwd(q.data_ptr(), cache.data_ptr(), out.data_ptr(),
                              lse.data_ptr() if lse is not None else None, B, Hq, idx.data_ptr(),
                              idx.stride(0), n_sel.data_ptr(), skv.data_ptr(), topk,
                              cache.shape[2], d_k, out.shape[-1], float(scale),
                              dtype_code(q.dtype), _strides4(q), _strides4(cache), _strides4(out),
                              workspace.data_ptr(), workspace.numel(), st.cuda_stream)
    if rc != ATTN_OK:
        raise AttnError(rc, "attn_topk_fwd")


def set_wait_timeout_ns(ns: int) -> int:
    """Bound every device-side wait of later launches (0 = default 2 s);
    returns the previous bound.  Diagnostic only (see the header)."""
    return int(load().attn_set_wait_timeout_ns(int(ns)))


def attention(q, k, v, skv, max_skv, scale, causal=True, with_lse=True, workspace=None,
              stream=None):
    """Allocate out (and lse, workspace) with torch and run :func:`attn_fwd`."""
    B, Hq, Sq, _ = q.shape
    d_v = v.shape[-1]
    out = torch.empty(B, Hq, Sq, d_v, dtype=q.dtype, device=q.device)
    lse = torch.empty(B, Hq, Sq, dtype=torch.float32, device=q.device) if with_lse else None
    if workspace is None:
        n = workspace_bytes(B, Hq, k.shape[1], Sq, int(max_skv), q.shape[-1], d_v)
        workspace = torch.empty(max(n, 16), dtype=torch.uint8, device=q.device)
    attn_fwd(q, k, v, out, skv, max_skv, scale, causal, lse, workspace, stream)
    return out, lse


def topk_attention(q, k_cache, v_cache, idx, n_sel, skv, scale, d_v=None, with_lse=True,
                   scratch=None, stream=None, fused=True):
    """Sparse (top-k) decode over topk = idx.shape[1] selections per sequence.
    k_cache/v_cache [B, Hkv, S, d]; for an absorbed-MLA latent cache pass
    v_cache=None and d_v (the value rows are the first d_v columns of the
    selected rows).  An absorbed-MLA decode (latent d 576 / 512, one query)
    runs in one pass, attn_topk_fwd, unless ``fused`` is False; otherwise
    attn_gather_rows copies the selected rows into scratch caches and
    attn_fwd attends over them, both on one stream.  ``scratch`` is an
    optional dict the scratch tensors (keys k, v, len, ws) are kept in
    between calls; they are reallocated when the problem's shapes change.
    Returns (out, lse)."""
    B, Hkv, _, d_k = k_cache.shape
    topk = idx.shape[1]
    latent = v_cache is None
    if latent and d_v is None:
        raise ValueError("d_v is required for a latent (MLA) cache")
    d_v = d_v if latent else v_cache.shape[-1]
    sc = scratch if scratch is not None else {}
    if fused and latent and d_k == 576 and d_v == 512 and Hkv == 1 and q.shape[2] == 1:
        key = ("fused", B, topk, q.shape[1], k_cache.device)
        if sc.get("key") != key:
            sc.clear()
            sc["key"] = key
            n = workspace_bytes(B, q.shape[1], 1, 1, topk, d_k, d_v)
            sc["ws"] = torch.empty(max(n, 16), dtype=torch.uint8, device=k_cache.device)
        out = torch.empty(B, q.shape[1], 1, d_v, dtype=q.dtype, device=q.device)
        lse = (torch.empty(B, q.shape[1], 1, dtype=torch.float32, device=q.device)
               if with_lse else None)
        topk_fwd(q, k_cache, out, idx, n_sel, skv, scale, lse, sc["ws"], stream)
        return out, lse
    key = (B, Hkv, topk, d_k, d_v, latent, k_cache.dtype, k_cache.device, q.shape[1], q.shape[2])
    if sc.get("key") != key:  # (re)allocate for this problem's shapes
        sc.clear()
        sc["key"] = key
        sc["k"] = torch.empty(B, Hkv, topk, d_k, dtype=k_cache.dtype, device=k_cache.device)
        sc["v"] = None if latent else torch.empty(B, Hkv, topk, d_v, dtype=k_cache.dtype,
                                                  device=k_cache.device)
        sc["len"] = torch.empty(B, dtype=torch.int32, device=k_cache.device)
        n = workspace_bytes(B, q.shape[1], Hkv, q.shape[2], topk, d_k, d_v)
        sc["ws"] = torch.empty(max(n, 16), dtype=torch.uint8, device=k_cache.device)
    gather_rows(k_cache, sc["k"], idx, n_sel, skv, sc["len"], stream)
    if not latent:
        gather_rows(v_cache, sc["v"], idx, n_sel, skv, sc["len"], stream)
    v = sc["k"][..., :d_v] if latent else sc["v"]
    out = torch.empty(B, q.shape[1], q.shape[2], d_v, dtype=q.dtype, device=q.device)
    lse = (torch.empty(B, q.shape[1], q.shape[2], dtype=torch.float32, device=q.device)
           if with_lse else None)
    attn_fwd(q, sc["k"], v, out, sc["len"], topk, scale, True, lse, sc["ws"], stream)
    return out, lse
