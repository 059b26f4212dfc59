"""ctypes binding of libgqa (include/gqa.h).

Argument marshalling only: shape/dtype/device checks, output allocation with torch,
the current torch stream, and the C call.  Every step of the computation runs in the
CUDA kernels of libgqa.so; there is no fallback path.  If the library is missing, the
first call raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libgqa.so")

GQA_OK = 0
DEVERR_SEQLEN = 1
DEVERR_TIMEOUT = 2
DEVERR_PAGE = 4

_lib = None


class GQAError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        super().__init__(f"{what} failed with code {code}: {strerror(code)}")


def load() -> ctypes.CDLL:
    """Load libgqa.so (built by grouped_query_attention_gqa_b200.build); raise if absent."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                           f"`python -m grouped_query_attention_gqa_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i, f = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    lib.gqa_prefill.argtypes = [vp, vp, vp, vp, i, i, i, i, i, f]
    lib.gqa_prefill.restype = i
    lib.gqa_decode.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, f]
    lib.gqa_decode.restype = i
    lib.gqa_decode_paged.argtypes = [vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, i, f]
    lib.gqa_decode_paged.restype = i
    lib.gqa_qkv_rope.argtypes = [vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, f]
    lib.gqa_qkv_rope.restype = i
    lib.gqa_qkv_append.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, i, i, f]
    lib.gqa_qkv_append.restype = i
    lib.gqa_set_decode_self_in_cache.argtypes = [i]
    lib.gqa_set_decode_self_in_cache.restype = i
    lib.gqa_set_decode_cache_rotated.argtypes = [i]
    lib.gqa_set_decode_cache_rotated.restype = i
    lib.gqa_prefill_rotated.argtypes = [vp, vp, vp, vp, i, i, i, i, i]
    lib.gqa_prefill_rotated.restype = i
    lib.gqa_out_proj.argtypes = [vp, vp, vp, vp, i, i, i]
    lib.gqa_out_proj.restype = i
    lib.gqa_set_rope_scaling.argtypes = [f, i]
    lib.gqa_set_rope_scaling.restype = i
    lib.gqa_set_timing_events.argtypes = [vp, vp]
    lib.gqa_set_timing_events.restype = i
    lib.gqa_set_stream.argtypes = [vp]
    lib.gqa_set_stream.restype = i
    lib.gqa_last_error.argtypes = []
    lib.gqa_last_error.restype = i
    lib.gqa_release.argtypes = []
    lib.gqa_release.restype = None
    lib.gqa_strerror.argtypes = [i]
    lib.gqa_strerror.restype = ctypes.c_char_p
    lib.gqa_abi_version.argtypes = []
    lib.gqa_abi_version.restype = i
    ip = ctypes.POINTER(ctypes.c_int)
    lib.gqa_prefill_schedule.argtypes = [i, i, i, i, i, ip, ip, i, ip]
    lib.gqa_prefill_schedule.restype = i
    _lib = lib
    return lib


def strerror(code: int) -> str:
    return load().gqa_strerror(int(code)).decode()


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _check(t, name, shape, dtype=torch.bfloat16):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")


def _stream(device) -> None:
    load().gqa_set_stream(ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream))


def prefill(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, theta: float = 1.0e6,
            out: torch.Tensor | None = None) -> torch.Tensor:
    """Causal GQA prefill.  q [B,L,h_q,d], k/v [B,L,h_kv,d] bf16 CUDA -> out [B,L,h_q,d] bf16."""
    if q.dim() != 4 or k.dim() != 4:
        raise ValueError("q and k must be 4-D [B, L, heads, d]")
    B, L, h_q, d = q.shape
    h_kv = k.shape[2]
    _check(q, "q", None)
    _check(k, "k", (B, L, h_kv, d))
    _check(v, "v", (B, L, h_kv, d))
    if out is None:
        out = torch.empty_like(q)
    _check(out, "out", (B, L, h_q, d))
    with torch.cuda.device(q.device):
        _stream(q.device)
        rc = load().gqa_prefill(_ptr(q), _ptr(k), _ptr(v), _ptr(out), B, L, h_q, h_kv, d, float(theta))
    if rc != GQA_OK:
        raise GQAError(rc, "gqa_prefill")
    return out


def decode(q: torch.Tensor, kcache: torch.Tensor, vcache: torch.Tensor, seqlens: torch.Tensor,
           theta: float = 1.0e6, out: torch.Tensor | None = None) -> torch.Tensor:
    """One decode step.  q [B,h_q,d]; caches packed [sum(seqlens),h_kv,d]; seqlens int32 [B] (device)."""
    if q.dim() != 3 or kcache.dim() != 3:
        raise ValueError("q must be [B, h_q, d] and kcache [rows, h_kv, d]")
    B, h_q, d = q.shape
    h_kv = kcache.shape[1]
    _check(q, "q", None)
    _check(kcache, "kcache", (kcache.shape[0], h_kv, d))
    _check(vcache, "vcache", tuple(kcache.shape))
    _check(seqlens, "seqlens", (B,), dtype=torch.int32)
    if out is None:
        out = torch.empty_like(q)
    _check(out, "out", (B, h_q, d))
    with torch.cuda.device(q.device):
        _stream(q.device)
        rc = load().gqa_decode(_ptr(q), _ptr(kcache), _ptr(vcache), _ptr(seqlens), _ptr(out),
                               B, h_q, h_kv, d, float(theta))
    if rc != GQA_OK:
        raise GQAError(rc, "gqa_decode")
    return out


def decode_paged(q: torch.Tensor, kpages: torch.Tensor, vpages: torch.Tensor, block_table: torch.Tensor,
                 seqlens: torch.Tensor, theta: float = 1.0e6, out: torch.Tensor | None = None) -> torch.Tensor:
    """One decode step over a paged cache.

    q [B, h_q, d]; kpages / vpages [num_pages, page_size, h_kv, d]; block_table int32 [B, max_pages]
    (device): position j of sequence b is slot j % page_size of page block_table[b, j // page_size];
    seqlens int32 [B] (device).
    """
    if q.dim() != 3 or kpages.dim() != 4:
        raise ValueError("q must be [B, h_q, d] and kpages [num_pages, page_size, h_kv, d]")
    B, h_q, d = q.shape
    num_pages, page_size, h_kv = kpages.shape[:3]
    _check(q, "q", None)
    _check(kpages, "kpages", (num_pages, page_size, h_kv, d))
    _check(vpages, "vpages", tuple(kpages.shape))
    _check(seqlens, "seqlens", (B,), dtype=torch.int32)
    if block_table.dim() != 2 or block_table.shape[0] != B:
        raise ValueError(f"block_table must be [B={B}, max_pages], got {tuple(block_table.shape)}")
    _check(block_table, "block_table", None, dtype=torch.int32)
    if out is None:
        out = torch.empty_like(q)
    _check(out, "out", (B, h_q, d))
    with torch.cuda.device(q.device):
        _stream(q.device)
        rc = load().gqa_decode_paged(_ptr(q), _ptr(kpages), _ptr(vpages), _ptr(block_table), _ptr(seqlens),
                                     _ptr(out), B, h_q, h_kv, d, page_size, num_pages, block_table.shape[1],
                                     float(theta))
    if rc != GQA_OK:
        raise GQAError(rc, "gqa_decode_paged")
    return out


def qkv_rope(x: torch.Tensor, w_qkv: torch.Tensor, b_qkv: torch.Tensor | None, h_q: int, h_kv: int,
             theta: float = 1.0e6, out=None):
    """Fused QKV projection + bias + RoPE.  x [B, L, d_model]; w_qkv [(h_q + 2 h_kv) d, d_model] (nn.Linear
    layout); b_qkv [(h_q + 2 h_kv) d] or None.  Returns (qr [B,h_q,L,d], kr [B,h_kv,L,d] rotated,
    k [B,L,h_kv,d] raw, v [B,L,h_kv,d]); `out` may give those four tensors (e.g. k, v inside a cache)."""
    if x.dim() != 3 or w_qkv.dim() != 2:
        raise ValueError("x must be [B, L, d_model] and w_qkv [(h_q + 2 h_kv) d, d_model]")
    B, L, dm = x.shape
    n = w_qkv.shape[0]
    if n % (h_q + 2 * h_kv) != 0:
        raise ValueError(f"w_qkv has {n} rows, not a multiple of h_q + 2 h_kv = {h_q + 2 * h_kv}")
    d = n // (h_q + 2 * h_kv)
    _check(x, "x", None)
    _check(w_qkv, "w_qkv", (n, dm))
    if b_qkv is not None:
        _check(b_qkv, "b_qkv", (n,))
    if out is None:
        out = (x.new_empty(B, h_q, L, d), x.new_empty(B, h_kv, L, d), x.new_empty(B, L, h_kv, d),
               x.new_empty(B, L, h_kv, d))
    qr, kr, k, v = out
    _check(qr, "qr", (B, h_q, L, d))
    _check(kr, "kr", (B, h_kv, L, d))
    _check(k, "k", (B, L, h_kv, d))
    _check(v, "v", (B, L, h_kv, d))
    with torch.cuda.device(x.device):
        _stream(x.device)
        rc = load().gqa_qkv_rope(_ptr(x), _ptr(w_qkv), _ptr(b_qkv), _ptr(qr), _ptr(kr), _ptr(k), _ptr(v),
                                 B, L, dm, h_q, h_kv, d, float(theta))
    if rc != GQA_OK:
        raise GQAError(rc, "gqa_qkv_rope")
    return qr, kr, k, v


def qkv_append(x: torch.Tensor, w_qkv: torch.Tensor, b_qkv: torch.Tensor | None, h_q: int, h_kv: int,
               seqlens: torch.Tensor, kpages: torch.Tensor, vpages: torch.Tensor, block_table: torch.Tensor,
               q: torch.Tensor | None = None, theta: float = 1.0e6) -> torch.Tensor:
    """One decode step's projection and cache append.  x [B, d_model] (the new token of each sequence);
    w_qkv, b_qkv as for qkv_rope; seqlens int32 [B] (device): each new token's position (the cache length
    before the append).  Writes the tokens' K (un-rotated, or rotated at its position with base `theta`
    while set_decode_cache_rotated(True) is in effect) and V into kpages / vpages [num_pages, page_size,
    h_kv, d] at those positions through block_table int32 [B, max_pages]; returns q [B, h_q, d] (un-rotated)."""
    if x.dim() != 2 or w_qkv.dim() != 2 or kpages.dim() != 4:
        raise ValueError("x must be [B, d_model], w_qkv [(h_q + 2 h_kv) d, d_model], kpages [P, page, h_kv, d]")
    B, dm = x.shape
    n = w_qkv.shape[0]
    if n % (h_q + 2 * h_kv) != 0:
        raise ValueError(f"w_qkv has {n} rows, not a multiple of h_q + 2 h_kv = {h_q + 2 * h_kv}")
    d = n // (h_q + 2 * h_kv)
    num_pages, page_size = kpages.shape[:2]
    _check(x, "x", None)
    _check(w_qkv, "w_qkv", (n, dm))
    if b_qkv is not None:
        _check(b_qkv, "b_qkv", (n,))
    _check(kpages, "kpages", (num_pages, page_size, h_kv, d))
    _check(vpages, "vpages", tuple(kpages.shape))
    _check(seqlens, "seqlens", (B,), dtype=torch.int32)
    if block_table.dim() != 2 or block_table.shape[0] != B:
        raise ValueError(f"block_table must be [B={B}, max_pages], got {tuple(block_table.shape)}")
    _check(block_table, "block_table", None, dtype=torch.int32)
    if q is None:
        q = x.new_empty(B, h_q, d)
    _check(q, "q", (B, h_q, d))
    with torch.cuda.device(x.device):
        _stream(x.device)
        rc = load().gqa_qkv_append(_ptr(x), _ptr(w_qkv), _ptr(b_qkv), _ptr(seqlens), _ptr(q), _ptr(kpages),
                                   _ptr(vpages), _ptr(block_table), B, dm, h_q, h_kv, d, page_size, num_pages,
                                   block_table.shape[1], float(theta))
    if rc != GQA_OK:
        raise GQAError(rc, "gqa_qkv_append")
    return q


def set_decode_self_in_cache(on: bool) -> None:
    """Later decode calls: False (default) -- the query sits at seqlens[b] and attends to the seqlens[b]
    cached rows; True -- the cache's last row is the query's own, so it sits at seqlens[b] - 1."""
    rc = load().gqa_set_decode_self_in_cache(1 if on else 0)
    if rc != GQA_OK:
        raise GQAError(rc, "gqa_set_decode_self_in_cache")


def set_decode_cache_rotated(on: bool) -> None:
    """Later decode / append / qkv_rope calls: False (default) -- the K cache holds raw keys, rotated by the
    decode on load; True -- it holds keys already rotated at their positions (qkv_append and qkv_rope's k
    output write them so), and the decode rotates only the query."""
    rc = load().gqa_set_decode_cache_rotated(1 if on else 0)
    if rc != GQA_OK:
        raise GQAError(rc, "gqa_set_decode_cache_rotated")


def prefill_rotated(qr: torch.Tensor, kr: torch.Tensor, v: torch.Tensor, out: torch.Tensor | None = None):
    """Causal GQA attention on rotated inputs: qr [B,h_q,L,d], kr [B,h_kv,L,d], v [B,L,h_kv,d] -> [B,L,h_q,d]."""
    if qr.dim() != 4 or kr.dim() != 4 or v.dim() != 4:
        raise ValueError("qr, kr and v must be 4-D")
    B, h_q, L, d = qr.shape
    h_kv = kr.shape[1]
    _check(qr, "qr", None)
    _check(kr, "kr", (B, h_kv, L, d))
    _check(v, "v", (B, L, h_kv, d))
    if out is None:
        out = qr.new_empty(B, L, h_q, d)
    _check(out, "out", (B, L, h_q, d))
    with torch.cuda.device(qr.device):
        _stream(qr.device)
        rc = load().gqa_prefill_rotated(_ptr(qr), _ptr(kr), _ptr(v), _ptr(out), B, L, h_q, h_kv, d)
    if rc != GQA_OK:
        raise GQAError(rc, "gqa_prefill_rotated")
    return out


def out_proj(attn: torch.Tensor, w_o: torch.Tensor, residual: torch.Tensor | None = None,
             out: torch.Tensor | None = None) -> torch.Tensor:
    """out [T, d_model] = attn [T, d_in] @ w_o[d_model, d_in]^T (+ residual [T, d_model]); `out` may be
    `residual` itself.  A [B, L, h_q, d] attention output may be passed as attn (viewed as [B*L, h_q*d])."""
    a = attn.reshape(-1, attn.shape[-2] * attn.shape[-1]) if attn.dim() == 4 else attn
    if a.dim() != 2 or w_o.dim() != 2:
        raise ValueError("attn must be [T, d_in] (or [B, L, h, d]) and w_o [d_model, d_in]")
    T, d_in = a.shape
    dm = w_o.shape[0]
    _check(a, "attn", None)
    _check(w_o, "w_o", (dm, d_in))
    if residual is not None:
        _check(residual, "residual", (T, dm))
    if out is None:
        out = a.new_empty(T, dm)
    _check(out, "out", (T, dm))
    with torch.cuda.device(a.device):
        _stream(a.device)
        rc = load().gqa_out_proj(_ptr(a), _ptr(w_o), _ptr(residual), _ptr(out), T, d_in, dm)
    if rc != GQA_OK:
        raise GQAError(rc, "gqa_out_proj")
    return out


def set_rope_scaling(factor: float = 1.0, original_max_position: int = 0) -> None:
    """YaRN scaling of RoPE (factor s, trained window) for later calls; factor 1 turns it off."""
    rc = load().gqa_set_rope_scaling(float(factor), int(original_max_position))
    if rc != GQA_OK:
        raise GQAError(rc, "gqa_set_rope_scaling")


def last_error(device=None) -> int:
    """Synchronise and return/clear the device error word (GQA_DEVERR_* bits)."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    with torch.cuda.device(dev):
        _stream(dev)
        return int(load().gqa_last_error())


def set_timing_events(start=None, stop=None) -> None:
    """Record torch.cuda.Event `start`/`stop` around the main kernel of later calls (None: off).

    Both events must already exist on the device (record each once before handing it over).
    """
    h = (lambda e: None if e is None else ctypes.c_void_p(e.cuda_event))
    load().gqa_set_timing_events(h(start), h(stop))


def release() -> None:
    load().gqa_release()


def prefill_schedule(B: int, L: int, h_q: int, h_kv: int, grid: int):
    """The attention work schedule gqa_prefill uses for this shape over `grid` CTAs (host only).

    Returns (lists, grouped): lists[c] is CTA c's item list in order; grouped is True where the items are
    dealt plane group by plane group for L2 reuse (many items per CTA), False where they are packed by
    best fit for balance.
    """
    lib = load()
    grouped = ctypes.c_int(0)
    n = lib.gqa_prefill_schedule(B, L, h_q, h_kv, grid, None, None, 0, ctypes.byref(grouped))
    if n < 0:
        raise GQAError(n, "gqa_prefill_schedule")
    g = min(grid, n)
    starts = (ctypes.c_int * (g + 1))()
    items = (ctypes.c_int * max(n, 1))()
    lib.gqa_prefill_schedule(B, L, h_q, h_kv, grid, starts, items, n, ctypes.byref(grouped))
    return [list(items[starts[c]:starts[c + 1]]) for c in range(g)], bool(grouped.value)
