"""ctypes binding of the C ABI in ``include/gqa.h``: argument marshalling only.

Every step of the computation runs in the CUDA library ``libgqa_b200.so``; this module checks
tensor shapes and dtypes, allocates outputs with PyTorch (device memory is plumbing), passes raw
device pointers and the current CUDA stream, and turns status codes into exceptions.  There is no
fallback: if the library is missing, importing this module raises.
"""

from __future__ import annotations

import ctypes
import os
import threading

import torch

_PKG_DIR = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG_DIR, "libgqa_b200.so")

GQA_OK = 0
STATUS_NAMES = {
    0: "GQA_OK",
    1: "GQA_ERR_INVALID_ARG",
    2: "GQA_ERR_UNSUPPORTED",
    3: "GQA_ERR_CUDA",
    4: "GQA_ERR_DEVICE",
    5: "GQA_ERR_WORKSPACE",
}
GQA_BF16, GQA_FP32 = 0, 1
DEVERR_NAMES = {0: "none", 1: "kv_len out of range", 2: "position out of range",
                3: "query with no visible key", 4: "pipeline wait timed out",
                5: "block-table entry out of range"}

# name -> (restype, argtypes), mirroring include/gqa.h
_P, _I, _F, _Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
SIGNATURES = {
    "gqa_prefill": (_I, [_P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _I, _I, _I, _P]),
    "gqa_decode_workspace_size": (_Z, [_I, _I, _I, _I, _I, _I, _I]),
    "gqa_decode": (_I, [_P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _F, _I, _I, _P, _Z, _I, _P]),
    "gqa_decode_noalloc": (_I, [_P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _F, _I, _I, _I, _P]),
    "kv_append": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _P]),
    "gqa_decode_paged": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _F, _I,
                              _I, _P, _Z, _I, _P]),
    "kv_append_paged": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _P]),
    "gqa_prefill_backward_workspace_size": (_Z, [_I, _I, _I]),
    "gqa_mla_decode_workspace_size": (_Z, [_I, _I, _I, _I, _I, _I]),
    "gqa_mla_decode": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _F, _I, _P, _Z, _I, _P]),
    "gqa_prefill_backward": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I,
                                  _F, _I, _I, _I, _P, _Z, _P]),
    "gqa_get_device_error": (_I, [ctypes.POINTER(_I), _P]),
    "gqa_status_string": (ctypes.c_char_p, [_I]),
    "gqa_version": (ctypes.c_char_p, []),
    "gqa_debug_expire_waits": (_I, [_I]),
}


class GQAError(RuntimeError):
    """A non-OK status returned by the library."""

    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn} returned {STATUS_NAMES.get(status, status)}")


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    if not os.path.exists(path):
        raise ImportError(
            f"{path} is missing: build it with `python -c 'import __graft_entry__ as g; g.build()'` "
            "(or `python kv_cache_attention_gqa_b200/build.py`). There is no fallback implementation."
        )
    lib = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


_lib = load_library()


def _check(fn: str, status: int) -> None:
    if status != GQA_OK:
        raise GQAError(fn, status)


def version() -> str:
    return _lib.gqa_version().decode()


def status_string(status: int) -> str:
    return _lib.gqa_status_string(status).decode()


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return GQA_BF16
    if t.dtype == torch.float32:
        return GQA_FP32
    raise TypeError(f"unsupported dtype {t.dtype}: bf16 (tensor-core path) or fp32 (check mode)")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _need_cuda(*ts):
    """Every tensor given is a contiguous CUDA tensor on the current device (the library launches on
    the current device and its current stream)."""
    dev = None
    for t in ts:
        if t is None:
            continue
        if not t.is_cuda:
            raise ValueError("tensors must live on a CUDA device")
        if not t.is_contiguous():
            raise ValueError("tensors must be contiguous (row-major)")
        if dev is None:
            dev = torch.cuda.current_device()
        if t.device.index != dev:
            raise ValueError(f"tensors must live on the current CUDA device (cuda:{dev}), not {t.device}")


def _int_vec(x, B: int, device, name: str):
    """Device int32[B] from None / int / sequence / tensor (None stays None = library default)."""
    if x is None:
        return None
    if (isinstance(x, torch.Tensor) and x.is_cuda and x.device == torch.device(device)
            and x.dtype == torch.int32 and x.is_contiguous()):
        if x.numel() != B:
            raise ValueError(f"{name} must have {B} entries")
        return x
    if isinstance(x, int):
        x = [x] * B
    t = torch.as_tensor(x, dtype=torch.int32, device=device).contiguous()
    if t.numel() != B:
        raise ValueError(f"{name} must have {B} entries")
    return t


def _out(out, shape, dtype, device):
    """The output tensor: a new one, or the caller's after checking its shape and dtype (the kernels
    write every element of ``shape``; a smaller buffer would be overrun)."""
    if out is None:
        return torch.empty(shape, dtype=dtype, device=device)
    if tuple(out.shape) != tuple(shape) or out.dtype != dtype:
        raise ValueError(f"out must be {dtype} of shape {tuple(shape)}, not {out.dtype} {tuple(out.shape)}")
    return out


def _ws_bytes(ws) -> int:
    """Byte size of a caller workspace, which must be a contiguous tensor on the current device."""
    _need_cuda(ws)
    return ws.numel() * ws.element_size()


def _scale(scale) -> float:
    """None -> 0.0, which the C ABI reads as its default 1/sqrt(d_h) (MLA: 1/sqrt(d_qk))."""
    return 0.0 if scale is None else float(scale)


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def debug_expire_waits(enable: bool) -> None:
    """Failure-detection test hook (gqa_debug_expire_waits): while enabled, bf16 prefill and
    contiguous bf16 decode make one bounded wait run out, so the call reports a timeout."""
    _check("gqa_debug_expire_waits", _lib.gqa_debug_expire_waits(1 if enable else 0))


def get_device_error() -> int:
    """Synchronise the current stream, read and clear the sticky device error word."""
    code = ctypes.c_int(0)
    st = _lib.gqa_get_device_error(ctypes.byref(code), _stream())
    if st not in (GQA_OK, 4):
        raise GQAError("gqa_get_device_error", st)
    return code.value


def kv_append(k_cache: torch.Tensor, v_cache: torch.Tensor, k_new: torch.Tensor,
              v_new: torch.Tensor, pos) -> None:
    """cache[b, g, pos[b] + t] = new[b, g, t] for t < S_new (in place, bit-exact)."""
    _need_cuda(k_cache, v_cache, k_new, v_new)
    B, h_kv, T_max, d_h = k_cache.shape
    if v_cache.shape != k_cache.shape or k_new.shape != v_new.shape:
        raise ValueError("shape mismatch")
    if k_new.dim() != 4 or k_new.shape[0] != B or k_new.shape[1] != h_kv or k_new.shape[3] != d_h:
        raise ValueError("k_new must be (B, h_kv, S_new, d_h)")
    dt = _dtype_code(k_cache)
    if any(t.dtype != k_cache.dtype for t in (v_cache, k_new, v_new)):
        raise TypeError("all four tensors must share one dtype")
    pos_t = _int_vec(pos, B, k_cache.device, "pos")
    _check("kv_append", _lib.kv_append(_ptr(k_cache), _ptr(v_cache), _ptr(k_new), _ptr(v_new),
                                       _ptr(pos_t), B, h_kv, k_new.shape[2], T_max, d_h, dt, _stream()))


def prefill(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor, *, q_start=None,
            kv_len=None, scale: float | None = None, causal: bool = True, window: int = 0,
            out=None, return_lse: bool = False):
    """Grouped-query attention of q (B, h_q, S_q, d_h) over the cache (B, h_kv, T_max, d_h).
    ``window`` > 0: sliding window, row at position p sees keys p - window < j <= p."""
    _need_cuda(q, k_cache, v_cache, out)
    B, h_q, S_q, d_h = q.shape
    Bk, h_kv, T_max, dk = k_cache.shape
    if (Bk, dk) != (B, d_h) or v_cache.shape != k_cache.shape:
        raise ValueError("q / k_cache / v_cache shapes disagree")
    dt = _dtype_code(q)
    if k_cache.dtype != q.dtype or v_cache.dtype != q.dtype:
        raise TypeError("q, k_cache and v_cache must share one dtype")
    out = _out(out, q.shape, q.dtype, q.device)
    lse = torch.empty((B, h_q, S_q), dtype=torch.float32, device=q.device) if return_lse else None
    qs = _int_vec(q_start, B, q.device, "q_start")
    kl = _int_vec(kv_len, B, q.device, "kv_len")
    scale = _scale(scale)
    _check("gqa_prefill", _lib.gqa_prefill(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(out), _ptr(lse),
                                           _ptr(qs), _ptr(kl), B, h_q, h_kv, S_q, T_max, d_h, scale,
                                           1 if causal else 0, int(window), dt, _stream()))
    return (out, lse) if return_lse else out


def decode_workspace_size(B: int, h_q: int, h_kv: int, T_max: int, d_h: int, dtype=torch.bfloat16,
                          num_splits: int = 0) -> int:
    dt = GQA_BF16 if dtype == torch.bfloat16 else GQA_FP32
    n = _lib.gqa_decode_workspace_size(B, h_q, h_kv, T_max, d_h, dt, num_splits)
    if n == 0:
        raise GQAError("gqa_decode_workspace_size", 1)
    return n


_ws_lock = threading.Lock()
_ws_cache: dict = {}
_ws_sizes: dict = {}


def workspace(nbytes: int, device) -> torch.Tensor:
    """A zero-filled, 256-byte aligned device workspace of at least ``nbytes``, cached per device
    and stream (every completed decode leaves its counter region at zero again)."""
    dev = torch.device(device)
    key = (dev.index, torch.cuda.current_stream(dev).cuda_stream)
    with _ws_lock:
        buf = _ws_cache.get(key)
        if buf is None or buf.numel() < nbytes:
            buf = torch.zeros(max(nbytes, 1 << 20), dtype=torch.uint8, device=dev)
            _ws_cache[key] = buf
    return buf


def decode(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor, *, kv_len=None,
           q_pos=None, scale: float | None = None, window: int = 0, num_splits: int = 0, out=None,
           return_lse: bool = False, ws: torch.Tensor | None = None):
    """Split-KV decode of q (B, h_q, d_h) over the cache (B, h_kv, T_max, d_h).
    ``window`` > 0: sliding window, the query at q_pos sees keys q_pos - window < j <= q_pos."""
    _need_cuda(q, k_cache, v_cache, out)
    B, h_q, d_h = q.shape
    Bk, h_kv, T_max, dk = k_cache.shape
    if (Bk, dk) != (B, d_h) or v_cache.shape != k_cache.shape:
        raise ValueError("q / k_cache / v_cache shapes disagree")
    dt = _dtype_code(q)
    if k_cache.dtype != q.dtype or v_cache.dtype != q.dtype:
        raise TypeError("q, k_cache and v_cache must share one dtype")
    out = _out(out, q.shape, q.dtype, q.device)
    lse = torch.empty((B, h_q), dtype=torch.float32, device=q.device) if return_lse else None
    kl = _int_vec(kv_len, B, q.device, "kv_len")
    qp = _int_vec(q_pos, B, q.device, "q_pos")
    scale = _scale(scale)
    key = (B, h_q, h_kv, T_max, d_h, dt, num_splits, q.device.index)
    need = _ws_sizes.get(key)
    if need is None:
        need = _ws_sizes[key] = decode_workspace_size(B, h_q, h_kv, T_max, d_h, q.dtype, num_splits)
    if ws is None:
        ws = workspace(need, q.device)
    _check("gqa_decode", _lib.gqa_decode(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(out), _ptr(lse),
                                         _ptr(kl), _ptr(qp), B, h_q, h_kv, T_max, d_h, scale,
                                         int(window), dt, _ptr(ws), _ws_bytes(ws), num_splits, _stream()))
    return (out, lse) if return_lse else out


def decode_noalloc(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor, *, kv_len=None,
                   q_pos=None, scale: float | None = None, window: int = 0, num_splits: int = 0,
                   out=None, return_lse: bool = False):
    """gqa_decode_noalloc: the decode with the library's fixed device scratch array instead of a
    caller workspace, for callers that cannot allocate device memory (the output buffer may be
    passed in as ``out``). Overlapping calls on different streams race on that array."""
    _need_cuda(q, k_cache, v_cache, out)
    B, h_q, d_h = q.shape
    Bk, h_kv, T_max, dk = k_cache.shape
    if (Bk, dk) != (B, d_h) or v_cache.shape != k_cache.shape:
        raise ValueError("q / k_cache / v_cache shapes disagree")
    dt = _dtype_code(q)
    if k_cache.dtype != q.dtype or v_cache.dtype != q.dtype:
        raise TypeError("q, k_cache and v_cache must share one dtype")
    out = _out(out, q.shape, q.dtype, q.device)
    lse = torch.empty((B, h_q), dtype=torch.float32, device=q.device) if return_lse else None
    kl = _int_vec(kv_len, B, q.device, "kv_len")
    qp = _int_vec(q_pos, B, q.device, "q_pos")
    scale = _scale(scale)
    _check("gqa_decode_noalloc", _lib.gqa_decode_noalloc(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(out),
                                                         _ptr(lse), _ptr(kl), _ptr(qp), B, h_q, h_kv, T_max,
                                                         d_h, scale, int(window), dt, num_splits, _stream()))
    return (out, lse) if return_lse else out


def _block_table(block_table, B: int, device) -> torch.Tensor:
    t = block_table
    if not (isinstance(t, torch.Tensor) and t.is_cuda and t.device == torch.device(device)
            and t.dtype == torch.int32 and t.is_contiguous()):
        t = torch.as_tensor(block_table, dtype=torch.int32, device=device).contiguous()
    if t.dim() != 2 or t.shape[0] != B:
        raise ValueError("block_table must be (B, max_pages)")
    return t


def _pool_shape(k_pages: torch.Tensor, v_pages: torch.Tensor):
    if k_pages.dim() != 4 or v_pages.shape != k_pages.shape:
        raise ValueError("k_pages / v_pages must both be (num_pages, h_kv, page_size, d_h)")
    return k_pages.shape


def decode_paged(q: torch.Tensor, k_pages: torch.Tensor, v_pages: torch.Tensor, block_table, *,
                 kv_len=None, q_pos=None, scale: float | None = None, window: int = 0,
                 num_splits: int = 0, out=None, return_lse: bool = False,
                 ws: torch.Tensor | None = None):
    """Split-KV decode of q (B, h_q, d_h) over a paged cache: pools (num_pages, h_kv, page_size,
    d_h) and block_table (B, max_pages) int32; position t of sequence b is row t % page_size of
    page block_table[b, t // page_size]."""
    _need_cuda(q, k_pages, v_pages, out)
    B, h_q, d_h = q.shape
    num_pages, h_kv, page_size, dk = _pool_shape(k_pages, v_pages)
    if dk != d_h:
        raise ValueError("q and the page pools disagree on d_h")
    dt = _dtype_code(q)
    if k_pages.dtype != q.dtype or v_pages.dtype != q.dtype:
        raise TypeError("q, k_pages and v_pages must share one dtype")
    bt = _block_table(block_table, B, q.device)
    max_pages = bt.shape[1]
    out = _out(out, q.shape, q.dtype, q.device)
    lse = torch.empty((B, h_q), dtype=torch.float32, device=q.device) if return_lse else None
    kl = _int_vec(kv_len, B, q.device, "kv_len")
    qp = _int_vec(q_pos, B, q.device, "q_pos")
    scale = _scale(scale)
    T_max = max_pages * page_size
    key = (B, h_q, h_kv, T_max, d_h, dt, num_splits, q.device.index)
    need = _ws_sizes.get(key)
    if need is None:
        need = _ws_sizes[key] = decode_workspace_size(B, h_q, h_kv, T_max, d_h, q.dtype, num_splits)
    if ws is None:
        ws = workspace(need, q.device)
    _check("gqa_decode_paged", _lib.gqa_decode_paged(
        _ptr(q), _ptr(k_pages), _ptr(v_pages), _ptr(out), _ptr(lse), _ptr(kl), _ptr(qp), _ptr(bt),
        B, h_q, h_kv, num_pages, page_size, max_pages, d_h, scale, int(window), dt, _ptr(ws), _ws_bytes(ws),
        num_splits, _stream()))
    return (out, lse) if return_lse else out


def kv_append_paged(k_pages: torch.Tensor, v_pages: torch.Tensor, k_new: torch.Tensor,
                    v_new: torch.Tensor, pos, block_table) -> None:
    """Write new[b, g, t] at logical position pos[b] + t of a paged cache (in place, bit-exact)."""
    _need_cuda(k_pages, v_pages, k_new, v_new)
    num_pages, h_kv, page_size, d_h = _pool_shape(k_pages, v_pages)
    if k_new.dim() != 4 or k_new.shape != v_new.shape or k_new.shape[1] != h_kv or k_new.shape[3] != d_h:
        raise ValueError("k_new / v_new must be (B, h_kv, S_new, d_h)")
    B = k_new.shape[0]
    dt = _dtype_code(k_pages)
    if any(t.dtype != k_pages.dtype for t in (v_pages, k_new, v_new)):
        raise TypeError("all four tensors must share one dtype")
    bt = _block_table(block_table, B, k_pages.device)
    pos_t = _int_vec(pos, B, k_pages.device, "pos")
    _check("kv_append_paged", _lib.kv_append_paged(
        _ptr(k_pages), _ptr(v_pages), _ptr(k_new), _ptr(v_new), _ptr(pos_t), _ptr(bt), B, h_kv,
        k_new.shape[2], num_pages, page_size, bt.shape[1], d_h, dt, _stream()))


def prefill_backward(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor, o: torch.Tensor,
                     d_o: torch.Tensor, lse: torch.Tensor, *, q_start=None, kv_len=None,
                     scale: float | None = None, causal: bool = True, window: int = 0,
                     ws: torch.Tensor | None = None):
    """Gradients (dq, dk, dv) of ``prefill`` for the upstream gradient ``d_o``; ``o`` and ``lse``
    are the forward's outputs (``prefill(..., return_lse=True)``). dk, dv have the cache's shape,
    zero past each kv_len."""
    _need_cuda(q, k_cache, v_cache, o, d_o, lse)
    B, h_q, S_q, d_h = q.shape
    Bk, h_kv, T_max, dk_ = k_cache.shape
    if (Bk, dk_) != (B, d_h) or v_cache.shape != k_cache.shape or o.shape != q.shape or d_o.shape != q.shape:
        raise ValueError("q / k_cache / v_cache / o / d_o shapes disagree")
    if lse.shape != (B, h_q, S_q) or lse.dtype != torch.float32:
        raise ValueError("lse must be fp32 (B, h_q, S_q)")
    dt = _dtype_code(q)
    if any(t.dtype != q.dtype for t in (k_cache, v_cache, o, d_o)):
        raise TypeError("q, k_cache, v_cache, o and d_o must share one dtype")
    dq = torch.empty_like(q)
    dk = torch.empty_like(k_cache)
    dv = torch.empty_like(v_cache)
    qs = _int_vec(q_start, B, q.device, "q_start")
    kl = _int_vec(kv_len, B, q.device, "kv_len")
    scale = _scale(scale)
    need = _lib.gqa_prefill_backward_workspace_size(B, h_q, S_q)
    if ws is None or _ws_bytes(ws) < need:
        ws = torch.empty(need, dtype=torch.uint8, device=q.device)
    _check("gqa_prefill_backward", _lib.gqa_prefill_backward(
        _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(o), _ptr(d_o), _ptr(lse), _ptr(dq), _ptr(dk),
        _ptr(dv), _ptr(qs), _ptr(kl), B, h_q, h_kv, S_q, T_max, d_h, scale, 1 if causal else 0,
        int(window), dt, _ptr(ws), _ws_bytes(ws), _stream()))
    return dq, dk, dv


def mla_decode(q: torch.Tensor, cache: torch.Tensor, d_v: int = 512, *, kv_len=None, q_pos=None,
               scale: float | None = None, num_splits: int = 0, out=None, return_lse: bool = False,
               ws: torch.Tensor | None = None):
    """MLA decode over a latent cache: q (B, h_q, d_qk) = [absorbed latent query | rotary part],
    cache (B, T_max, d_qk) = [latent | rotary key]; returns the latent output (B, h_q, d_v) (the
    value rows are cache[..., :d_v]). ``scale`` should be the model's softmax scale."""
    _need_cuda(q, cache, out)
    B, h_q, d_qk = q.shape
    Bc, T_max, dc = cache.shape
    if (Bc, dc) != (B, d_qk):
        raise ValueError("q and cache shapes disagree")
    dt = _dtype_code(q)
    if cache.dtype != q.dtype:
        raise TypeError("q and cache must share one dtype")
    out = _out(out, (B, h_q, d_v), q.dtype, q.device)
    lse = torch.empty((B, h_q), dtype=torch.float32, device=q.device) if return_lse else None
    kl = _int_vec(kv_len, B, q.device, "kv_len")
    qp = _int_vec(q_pos, B, q.device, "q_pos")
    scale = _scale(scale)
    key = ("mla", B, h_q, T_max, d_v, dt, num_splits, q.device.index)
    need = _ws_sizes.get(key)
    if need is None:
        need = _lib.gqa_mla_decode_workspace_size(B, h_q, T_max, d_v, dt, num_splits)
        if need == 0:
            raise GQAError("gqa_mla_decode_workspace_size", 1)
        _ws_sizes[key] = need
    if ws is None:
        ws = workspace(need, q.device)
    _check("gqa_mla_decode", _lib.gqa_mla_decode(
        _ptr(q), _ptr(cache), _ptr(out), _ptr(lse), _ptr(kl), _ptr(qp), B, h_q, T_max, d_qk, d_v,
        scale, dt, _ptr(ws), _ws_bytes(ws), num_splits, _stream()))
    return (out, lse) if return_lse else out
