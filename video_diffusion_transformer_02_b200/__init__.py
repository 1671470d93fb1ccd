"""Python binding of libvattn (B200 spatiotemporal attention kernels).

Argument marshalling only: every step of the computation runs in the CUDA
kernels of libvattn.so, called through its C ABI (include/vattn.h) with
ctypes.  Tensors are torch tensors used as device memory; the current torch
CUDA stream is passed to every call.  The module refuses to import when the
shared library is missing: there is no fallback.
"""
from __future__ import annotations

import ctypes
import dataclasses
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libvattn.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        "libvattn.so is not built (run `python -m video_diffusion_transformer_02_b200._build`); "
        "this package has no non-CUDA fallback")

_lib = ctypes.CDLL(LIB_PATH)

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_CUDA, ERR_TIMEOUT = range(5)
FULL, CHUNK_CAUSAL, SLIDING = 0, 1, 2
MODES = {"full": FULL, "chunk_causal": CHUNK_CAUSAL, "sliding": SLIDING}


class VattnError(RuntimeError):
    def __init__(self, status: int, detail: str):
        super().__init__("vattn status %d (%s): %s" % (status, status_string(status), detail))
        self.status = status


class vattn_rope(ctypes.Structure):
    _fields_ = [("Hg", ctypes.c_int), ("Wg", ctypes.c_int), ("pairs_t", ctypes.c_int),
                ("pairs_h", ctypes.c_int), ("pairs_w", ctypes.c_int), ("max_pos", ctypes.c_int),
                ("theta", ctypes.c_double)]


@dataclasses.dataclass(frozen=True)
class Rope:
    """3D-RoPE configuration (mirrors struct vattn_rope)."""
    Hg: int
    Wg: int
    pairs: tuple
    max_pos: int
    theta: float = 10000.0

    def c(self) -> vattn_rope:
        return vattn_rope(self.Hg, self.Wg, self.pairs[0], self.pairs[1], self.pairs[2],
                          self.max_pos, self.theta)


_P, _I, _F, _S = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
_RP = ctypes.POINTER(vattn_rope)


def _sig(name, res, *args):
    f = getattr(_lib, name)
    f.restype = res
    f.argtypes = list(args)
    return f


_status_string = _sig("vattn_status_string", ctypes.c_char_p, _I)
_last_error = _sig("vattn_last_error", ctypes.c_char_p)
_check = _sig("vattn_check", _I, _P)
_table_bytes = _sig("vattn_rope_table_bytes", _S, _RP, _I)
_table_build = _sig("vattn_rope_table_build", _I, _RP, _I, _P, _P)
_rope_qk = _sig("vattn_rope_qk", _I, _P, _P, _P, _P, _I, _I, _I, _I, _I, _RP, _P, _I, _P)
_attention = _sig("vattn_attention", _I, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _I, _I, _I,
                  _I, _I, _I, _I, _RP, _P, _P, _S, _P)
_attn_ws = _sig("vattn_attention_workspace_bytes", _S, _I, _I, _I, _I, _RP)
_attn_ws_ex = _sig("vattn_attention_workspace_bytes_ex", _S, _I, _I, _I, _I, _I, _I, _I, _RP)
_merge = _sig("vattn_attention_merge", _I, _P, _P, _I, _P, _P, _I, _I, _I, _I, _P)
_kv_init = _sig("vattn_kvcache_init", _I, ctypes.POINTER(_P), _P, _P, _P, _I, _I, _I, _I, _I, _P)
_kv_append = _sig("vattn_kvcache_append", _I, _P, _P, _P, _I, _P)
_attention_stream = _sig("vattn_attention_stream", _I, _P, _P, _P, _P, _P, _P, _I, _I, _I, _F, _RP,
                         _P, _P)
_kv_ids = _sig("vattn_kvcache_frame_ids", _I, _P, _P)
_kv_restore = _sig("vattn_kvcache_restore", _I, _P, _P, _P)
_kv_rope = _sig("vattn_kvcache_enable_rope", _I, _P, _P, _RP, _P, _P)
_kv_destroy = _sig("vattn_kvcache_destroy", _I, _P)
_kv_step_ws = _sig("vattn_kvcache_step_workspace_bytes", _S, _P, _I, _I)
_kv_step = _sig("vattn_kvcache_step", _I, _P, _P, _P, _P, _P, _P, _I, _I, _I, _F, _RP, _P, _I, _P, _S, _P)
_hyb_ws = _sig("vattn_hybrid_workspace_bytes", _S, _I, _I, _I, _I, _I)
_hybrid = _sig("vattn_hybrid_chunk", _I, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _F, _P, _S, _P)
_hybrid_delta = _sig("vattn_hybrid_delta", _I, _P, _P, _I, _I, _I, _I, _I, _P, _S, _P)
_hyb_ws_ex = _sig("vattn_hybrid_workspace_bytes_ex", _S, _I, _I, _I, _I, _I, _I)
_hybrid_ex = _sig("vattn_hybrid_chunk_ex", _I, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _I, _P, _P, _S, _P)
FMAP_ELU1, FMAP_POLY3 = 0, 1
_hybrid_scan = _sig("vattn_hybrid_scan", _I, _P, _P, _I, _I, _I, _I, _I, _P, _S, _P)
_hybrid_noalloc = _sig("vattn_hybrid_chunk_noalloc", _I, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _F, _P)
_selftest = _sig("vattn_selftest_umma", _I, _I, _P, _P, _P, _P)
_selftest_timeout = _sig("vattn_selftest_wait_timeout", _I, ctypes.c_uint32, _P)
_selftest_attn_timeout = _sig("vattn_selftest_attention_timeout", _I, _P, _P, _P, _P, _I, _I, _I,
                              ctypes.c_uint32, _P)
_selftest_ex2 = _sig("vattn_selftest_ex2", _I, _I, _P, _P, _I, _P)
HYBRID_NOALLOC_MAX_BYTES = 32 << 20


def status_string(status: int) -> str:
    return _status_string(status).decode()


def last_error() -> str:
    return _last_error().decode()


def _ok(status: int):
    if status != OK:
        raise VattnError(status, last_error())


def _stream(stream=None, device=None) -> int:
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _ptr(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensor must be on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    return t.data_ptr()


def _bf16(t, name):
    if t.dtype != torch.bfloat16:
        raise TypeError("%s must be bfloat16" % name)
    return _ptr(t)


# Argument checks of the wrappers.  They run before any pointer is taken or
# anything is launched: a tensor whose shape or dtype disagrees with the
# call would otherwise be read or written past its end by the kernels, and
# the library runs on the device of the first tensor, so every tensor must
# live there.
def _expect(t, name, shape, dtype):
    if not isinstance(t, torch.Tensor):
        raise TypeError("%s must be a torch tensor" % name)
    if t.dtype != dtype:
        raise TypeError("%s must be %s (got %s)" % (name, dtype, t.dtype))
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError("%s must have shape %s (got %s)" % (name, tuple(shape), tuple(t.shape)))
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)


def _min_bytes(t, name, nbytes):
    if not isinstance(t, torch.Tensor):
        raise TypeError("%s must be a torch tensor" % name)
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)
    have = t.numel() * t.element_size()
    if have < nbytes:
        raise ValueError("%s holds %d bytes, %d needed" % (name, have, nbytes))


def _rank(t, name, n):
    if not isinstance(t, torch.Tensor):
        raise TypeError("%s must be a torch tensor" % name)
    if t.dim() != n:
        raise ValueError("%s must have %d dimensions (got shape %s)" % (name, n, tuple(t.shape)))


def _device(*named):
    """The common CUDA device of the given (name, tensor) pairs (None entries
    are skipped); raises if one is not on CUDA or they differ."""
    dev = None
    for name, t in named:
        if t is None:
            continue
        if not t.is_cuda:
            raise ValueError("%s must be on a CUDA device (got %s)" % (name, t.device))
        if dev is None:
            dev = t.device
        elif t.device != dev:
            raise ValueError("%s is on %s, the other tensors on %s" % (name, t.device, dev))
    return dev


def _rope_c(rope):
    if rope is None:
        return None
    return ctypes.byref(rope.c())


# ------------------------------------------------------------------- RoPE
def vattn_rope_table_bytes(rope: Rope, d: int) -> int:
    return _table_bytes(ctypes.byref(rope.c()), d)


def vattn_rope_table_build(rope: Rope, d: int, table: torch.Tensor, stream=None):
    n = vattn_rope_table_bytes(rope, d)
    if n == 0:
        raise VattnError(ERR_INVALID_ARG, last_error())
    if table.dtype != torch.float32:
        raise TypeError("table must be float32")
    _min_bytes(table, "table", n)
    dev = _device(("table", table))
    with torch.cuda.device(dev):
        _ok(_table_build(ctypes.byref(rope.c()), d, _ptr(table), _stream(stream, dev)))


def rope_table(rope: Rope, d: int, device="cuda") -> torch.Tensor:
    """Allocate (torch) and fill the fp32 cos/sin table of a configuration."""
    n = vattn_rope_table_bytes(rope, d)
    if n == 0:
        raise VattnError(ERR_INVALID_ARG, last_error())
    t = torch.empty(n // 4, dtype=torch.float32, device=device)
    vattn_rope_table_build(rope, d, t)
    return t


def vattn_rope_qk(q, k, q_out, k_out, rope: Rope, table, frame_offset=0, stream=None):
    """3D-RoPE of q [B, L, H, d] into q_out and of k [B, L, Hkv, d] into k_out
    (either pair may be None)."""
    if (q is None) != (q_out is None) or (k is None) != (k_out is None):
        raise ValueError("q/q_out and k/k_out go together")
    ref = q if q is not None else k
    if ref is None:
        raise ValueError("q or k must be given")
    _rank(ref, "q" if q is not None else "k", 4)
    B, L, _, d = ref.shape
    H = q.shape[2] if q is not None else 1
    Hkv = k.shape[2] if k is not None else 1
    if q is not None:
        _expect(q, "q", (B, L, H, d), torch.bfloat16)
        _expect(q_out, "q_out", (B, L, H, d), torch.bfloat16)
    if k is not None:
        _expect(k, "k", (B, L, Hkv, d), torch.bfloat16)
        _expect(k_out, "k_out", (B, L, Hkv, d), torch.bfloat16)
    _expect(table, "table", None, torch.float32)
    dev = _device(("q", q), ("k", k), ("q_out", q_out), ("k_out", k_out), ("table", table))
    with torch.cuda.device(dev):
        _ok(_rope_qk(_ptr(q), _ptr(k), _ptr(q_out), _ptr(k_out), B, L, H, Hkv, d, _rope_c(rope),
                     _ptr(table), frame_offset, _stream(stream, dev)))


# -------------------------------------------------------------- attention
def vattn_attention_workspace_bytes(B, Lk, Hkv, d, rope: Rope | None) -> int:
    return _attn_ws(B, Lk, Hkv, d, _rope_c(rope))


def vattn_attention_workspace_bytes_ex(B, Lq, Lk, H, Hkv, d, mode="full", rope: Rope | None = None,
                                       device=None) -> int:
    """Workspace bytes for the rotated keys plus the tail split of a FULL
    call (zero-fill it before first use); depends on the SM count of `device`
    (the current device when None)."""
    m = MODES[mode] if isinstance(mode, str) else int(mode)
    if device is None:
        return _attn_ws_ex(B, Lq, Lk, H, Hkv, d, m, _rope_c(rope))
    with torch.cuda.device(device):
        return _attn_ws_ex(B, Lq, Lk, H, Hkv, d, m, _rope_c(rope))


def vattn_attention(q, k, v, o, lse=None, scale=None, mode="full", tokens_per_frame=0,
                    chunk_frames=1, window_back=0, window_fwd=0, q_frame_offset=0,
                    k_frame_offset=0, rope: Rope | None = None, table=None, workspace=None,
                    fuse_k_rope=False, stream=None):
    """o = masked softmax attention (see include/vattn.h); q/k/v/o [B, L, H, d] bf16.

    With rope, keys are rotated once into `workspace` (allocated here with
    torch when not given); fuse_k_rope=True passes no workspace, so the kernel
    rotates every K tile in shared memory instead.  A zero-filled uint8
    workspace of vattn_attention_workspace_bytes_ex bytes also enables the
    tail split of FULL calls.
    """
    _rank(q, "q", 4)
    _rank(k, "k", 4)
    B, Lq, H, d = q.shape
    Lk, Hkv = k.shape[1], k.shape[2]
    _expect(q, "q", None, torch.bfloat16)
    _expect(k, "k", (B, Lk, Hkv, d), torch.bfloat16)
    _expect(v, "v", (B, Lk, Hkv, d), torch.bfloat16)
    _expect(o, "o", (B, Lq, H, d), torch.bfloat16)
    if lse is not None:
        _expect(lse, "lse", (B, H, Lq), torch.float32)
    if (rope is None) != (table is None):
        raise ValueError("rope and table go together")
    if table is not None:
        _expect(table, "table", None, torch.float32)
        _min_bytes(table, "table", vattn_rope_table_bytes(rope, d))
    if scale is None:
        scale = d ** -0.5
    m = MODES[mode] if isinstance(mode, str) else int(mode)
    dev = _device(("q", q), ("k", k), ("v", v), ("o", o), ("lse", lse), ("table", table),
                  ("workspace", workspace))
    ws_ptr, ws_bytes = None, 0
    if rope is not None and not fuse_k_rope:
        need = vattn_attention_workspace_bytes(B, Lk, Hkv, d, rope)
        if workspace is None:
            workspace = torch.empty(need, dtype=torch.uint8, device=dev)
        _min_bytes(workspace, "workspace", need)
    if workspace is not None and not fuse_k_rope:
        _expect(workspace, "workspace", None, torch.uint8)
        ws_ptr, ws_bytes = _ptr(workspace), workspace.numel()
    with torch.cuda.device(dev):
        _ok(_attention(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, Lq, Lk, H, Hkv, d, float(scale), m,
                       tokens_per_frame, chunk_frames, window_back, window_fwd, q_frame_offset,
                       k_frame_offset, _rope_c(rope), _ptr(table), ws_ptr, ws_bytes, _stream(stream, dev)))


def vattn_attention_merge(o_parts, lse_parts, o, lse=None, stream=None):
    """Exact combination of R partial attentions over disjoint key sets:
    o_parts bf16 [R, B, L, H, d], lse_parts fp32 [R, B, H, L] -> o [B, L, H, d]
    (and lse [B, H, L])."""
    _rank(o_parts, "o_parts", 5)
    R, B, L, H, d = o_parts.shape
    _expect(o_parts, "o_parts", None, torch.bfloat16)
    _expect(lse_parts, "lse_parts", (R, B, H, L), torch.float32)
    _expect(o, "o", (B, L, H, d), torch.bfloat16)
    if lse is not None:
        _expect(lse, "lse", (B, H, L), torch.float32)
    dev = _device(("o_parts", o_parts), ("lse_parts", lse_parts), ("o", o), ("lse", lse))
    with torch.cuda.device(dev):
        _ok(_merge(_ptr(o_parts), _ptr(lse_parts), R, _ptr(o), _ptr(lse), B, L, H, d, _stream(stream, dev)))


# ---------------------------------------------------------------- KV ring
class KVCache:
    """Rolling KV cache over caller-owned ring storage (torch tensors).

    k_ring, v_ring: bf16 [capacity, B, F, Hkv, d]; frame_ids: int32 [capacity].
    """

    def __init__(self, k_ring, v_ring, frame_ids, stream=None):
        self._h = None
        _rank(k_ring, "k_ring", 5)
        cap, B, F, Hkv, d = k_ring.shape
        _expect(k_ring, "k_ring", None, torch.bfloat16)
        _expect(v_ring, "v_ring", (cap, B, F, Hkv, d), torch.bfloat16)
        _expect(frame_ids, "frame_ids", (cap,), torch.int32)
        self.device = _device(("k_ring", k_ring), ("v_ring", v_ring), ("frame_ids", frame_ids))
        self.k_ring, self.v_ring, self.frame_ids = k_ring, v_ring, frame_ids
        self.capacity, self.B, self.F, self.Hkv, self.d = cap, B, F, Hkv, d
        h = ctypes.c_void_p()
        with torch.cuda.device(self.device):
            _ok(_kv_init(ctypes.byref(h), _ptr(k_ring), _ptr(v_ring), _ptr(frame_ids), cap, B, F, Hkv, d,
                         _stream(stream, self.device)))
        self._h = h

    def append(self, k, v, frame_idx, stream=None):
        vattn_kvcache_append(self, k, v, frame_idx, stream)

    def attend(self, q, k_cur, v_cur, o, frame_idx, window_back, scale=None, lse=None,
               rope=None, table=None, stream=None):
        vattn_attention_stream(self, q, k_cur, v_cur, o, lse, frame_idx, window_back, scale, rope,
                               table, stream)

    def step(self, q, k_cur, v_cur, o, frame_idx, window_back, scale=None, lse=None, rope=None, table=None,
             window_relative=False, workspace=None, stream=None):
        """Attend and append frame frame_idx in one launch (vattn_kvcache_step)."""
        vattn_kvcache_step(self, q, k_cur, v_cur, o, lse, frame_idx, window_back, scale, rope, table,
                           window_relative, workspace, stream)

    def step_workspace(self, H, window_back):
        """A zero-filled workspace for step() (kept by the cache per (H, window_back))."""
        key = (H, window_back)
        ws = getattr(self, "_step_ws", {})
        if key not in ws:
            with torch.cuda.device(self.device):
                n = vattn_kvcache_step_workspace_bytes(self, H, window_back)
            if n == 0:
                raise VattnError(ERR_INVALID_ARG, "no step workspace for H=%d window_back=%d" % key)
            ws[key] = torch.zeros(n, dtype=torch.uint8, device=self.device)
            self._step_ws = ws
        return ws[key]

    def host_frame_ids(self):
        arr = (ctypes.c_int32 * self.capacity)()
        _ok(_kv_ids(self._h, arr))
        return list(arr)

    def restore(self, host_ids, stream=None):
        if len(host_ids) != self.capacity:
            raise ValueError("host_ids must have %d entries" % self.capacity)
        arr = (ctypes.c_int32 * self.capacity)(*host_ids)
        with torch.cuda.device(self.device):
            _ok(_kv_restore(self._h, arr, _stream(stream, self.device)))

    def enable_rope(self, k_ring_rot, rope: Rope, table, stream=None):
        """Rotated-key ring (bf16 [capacity + 1, B, F, Hkv, d]): keys rotated once per frame."""
        _expect(k_ring_rot, "k_ring_rot", (self.capacity + 1, self.B, self.F, self.Hkv, self.d), torch.bfloat16)
        _expect(table, "table", None, torch.float32)
        _min_bytes(table, "table", vattn_rope_table_bytes(rope, self.d))
        if _device(("k_ring_rot", k_ring_rot), ("table", table)) != self.device:
            raise ValueError("k_ring_rot and table must be on the cache's device %s" % self.device)
        self.k_ring_rot = k_ring_rot
        with torch.cuda.device(self.device):
            _ok(_kv_rope(self._h, _ptr(k_ring_rot), ctypes.byref(rope.c()), _ptr(table),
                         _stream(stream, self.device)))

    def close(self):
        if getattr(self, "_h", None):
            _kv_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def _frame_shape(cache, heads):
    return (cache.B, cache.F, heads, cache.d)


def _same_device(cache, *named):
    dev = _device(*named)
    if dev is not None and dev != cache.device:
        raise ValueError("tensors are on %s, the cache on %s" % (dev, cache.device))
    return cache.device


def vattn_kvcache_append(cache: KVCache, k, v, frame_idx, stream=None):
    _expect(k, "k", _frame_shape(cache, cache.Hkv), torch.bfloat16)
    _expect(v, "v", _frame_shape(cache, cache.Hkv), torch.bfloat16)
    dev = _same_device(cache, ("k", k), ("v", v))
    with torch.cuda.device(dev):
        _ok(_kv_append(cache._h, _ptr(k), _ptr(v), frame_idx, _stream(stream, dev)))


def vattn_attention_stream(cache: KVCache, q, k_cur, v_cur, o, lse, frame_idx, window_back,
                           scale=None, rope=None, table=None, stream=None):
    _rank(q, "q", 4)
    H = q.shape[2]
    _expect(q, "q", _frame_shape(cache, H), torch.bfloat16)
    _expect(k_cur, "k_cur", _frame_shape(cache, cache.Hkv), torch.bfloat16)
    _expect(v_cur, "v_cur", _frame_shape(cache, cache.Hkv), torch.bfloat16)
    _expect(o, "o", _frame_shape(cache, H), torch.bfloat16)
    if lse is not None:
        _expect(lse, "lse", (cache.B, H, cache.F), torch.float32)
    if (rope is None) != (table is None):
        raise ValueError("rope and table go together")
    if table is not None:
        _expect(table, "table", None, torch.float32)
        _min_bytes(table, "table", vattn_rope_table_bytes(rope, cache.d))
    if scale is None:
        scale = cache.d ** -0.5
    dev = _same_device(cache, ("q", q), ("k_cur", k_cur), ("v_cur", v_cur), ("o", o), ("lse", lse),
                       ("table", table))
    with torch.cuda.device(dev):
        _ok(_attention_stream(cache._h, _ptr(q), _ptr(k_cur), _ptr(v_cur), _ptr(o), _ptr(lse), H, frame_idx,
                              window_back, float(scale), _rope_c(rope), _ptr(table), _stream(stream, dev)))


def vattn_kvcache_step_workspace_bytes(cache: KVCache, H, window_back) -> int:
    return _kv_step_ws(cache._h, H, window_back)


def vattn_kvcache_step(cache: KVCache, q, k_cur, v_cur, o, lse, frame_idx, window_back, scale=None, rope=None,
                       table=None, window_relative=False, workspace=None, stream=None):
    _rank(q, "q", 4)
    H = q.shape[2]
    _expect(q, "q", _frame_shape(cache, H), torch.bfloat16)
    _expect(k_cur, "k_cur", _frame_shape(cache, cache.Hkv), torch.bfloat16)
    _expect(v_cur, "v_cur", _frame_shape(cache, cache.Hkv), torch.bfloat16)
    _expect(o, "o", _frame_shape(cache, H), torch.bfloat16)
    if lse is not None:
        _expect(lse, "lse", (cache.B, H, cache.F), torch.float32)
    if (rope is None) != (table is None):
        raise ValueError("rope and table go together")
    if table is not None:
        _expect(table, "table", None, torch.float32)
        _min_bytes(table, "table", vattn_rope_table_bytes(rope, cache.d))
    if scale is None:
        scale = cache.d ** -0.5
    dev = _same_device(cache, ("q", q), ("k_cur", k_cur), ("v_cur", v_cur), ("o", o), ("lse", lse),
                       ("table", table), ("workspace", workspace))
    if workspace is None:
        workspace = cache.step_workspace(H, window_back)
    with torch.cuda.device(dev):
        need = vattn_kvcache_step_workspace_bytes(cache, H, window_back)
        _min_bytes(workspace, "workspace", need)
        _ok(_kv_step(cache._h, _ptr(q), _ptr(k_cur), _ptr(v_cur), _ptr(o), _ptr(lse), H, frame_idx, window_back,
                     float(scale), _rope_c(rope), _ptr(table), int(bool(window_relative)), _ptr(workspace),
                     workspace.numel() * workspace.element_size(), _stream(stream, dev)))


# ----------------------------------------------------------------- hybrid
def vattn_hybrid_workspace_bytes(B, L, H, d, chunk_tokens) -> int:
    return _hyb_ws(B, L, H, d, chunk_tokens)


def _check_hybrid(q, k, v, o, S, z):
    _rank(q, "q", 4)
    B, L, H, d = q.shape
    for name, t in (("q", q), ("k", k), ("v", v), ("o", o)):
        _expect(t, name, (B, L, H, d), torch.bfloat16)
    _expect(S, "S", (B, H, d, d), torch.float32)
    _expect(z, "z", (B, H, d), torch.float32)
    return B, L, H, d


def vattn_hybrid_chunk(q, k, v, o, S, z, chunk_tokens, scale=None, workspace=None, stream=None):
    """Hybrid chunk attention; S [B,H,d,d] and z [B,H,d] fp32 are updated in place."""
    B, L, H, d = _check_hybrid(q, k, v, o, S, z)
    if scale is None:
        scale = d ** -0.5
    dev = _device(("q", q), ("k", k), ("v", v), ("o", o), ("S", S), ("z", z), ("workspace", workspace))
    need = vattn_hybrid_workspace_bytes(B, L, H, d, chunk_tokens)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    _min_bytes(workspace, "workspace", need)
    with torch.cuda.device(dev):
        _ok(_hybrid(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(S), _ptr(z), B, L, H, d, chunk_tokens,
                    float(scale), _ptr(workspace), workspace.numel() * workspace.element_size(),
                    _stream(stream, dev)))


def vattn_hybrid_workspace_bytes_ex(B, L, H, d, chunk_tokens, overlap_tokens) -> int:
    return _hyb_ws_ex(B, L, H, d, chunk_tokens, overlap_tokens)


def vattn_hybrid_chunk_ex(q, k, v, o, S, z, chunk_tokens, overlap_tokens=0, scale=None, coef=None,
                          workspace=None, stream=None):
    """Hybrid chunk attention with chunk overlap and, when coef (fp32 [2, H, 4],
    on the device) is given, the per-head degree-3 polynomial feature maps
    (elu + 1 otherwise)."""
    B, L, H, d = _check_hybrid(q, k, v, o, S, z)
    if scale is None:
        scale = d ** -0.5
    if coef is not None:
        _expect(coef, "coef", (2, H, 4), torch.float32)
    dev = _device(("q", q), ("k", k), ("v", v), ("o", o), ("S", S), ("z", z), ("coef", coef),
                  ("workspace", workspace))
    need = vattn_hybrid_workspace_bytes_ex(B, L, H, d, chunk_tokens, overlap_tokens)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    _min_bytes(workspace, "workspace", need)
    with torch.cuda.device(dev):
        _ok(_hybrid_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(S), _ptr(z), B, L, H, d, chunk_tokens,
                       overlap_tokens, float(scale), FMAP_POLY3 if coef is not None else FMAP_ELU1, _ptr(coef),
                       _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream, dev)))


def vattn_hybrid_delta(k, v, chunk_tokens, workspace, stream=None):
    """Per-chunk state deltas of k/v [B, L, H, d] into the workspace."""
    _rank(k, "k", 4)
    B, L, H, d = k.shape
    _expect(k, "k", None, torch.bfloat16)
    _expect(v, "v", (B, L, H, d), torch.bfloat16)
    _min_bytes(workspace, "workspace", vattn_hybrid_workspace_bytes(B, L, H, d, chunk_tokens))
    dev = _device(("k", k), ("v", v), ("workspace", workspace))
    with torch.cuda.device(dev):
        _ok(_hybrid_delta(_ptr(k), _ptr(v), B, L, H, d, chunk_tokens, _ptr(workspace),
                          workspace.numel() * workspace.element_size(), _stream(stream, dev)))


def vattn_hybrid_scan(S, z, L, chunk_tokens, workspace, stream=None):
    """Exclusive scan of the workspace's deltas over chunks; S [B,H,d,d], z [B,H,d] in/out."""
    _rank(S, "S", 4)
    B, H, d, _ = S.shape
    _expect(S, "S", (B, H, d, d), torch.float32)
    _expect(z, "z", (B, H, d), torch.float32)
    _min_bytes(workspace, "workspace", vattn_hybrid_workspace_bytes(B, L, H, d, chunk_tokens))
    dev = _device(("S", S), ("z", z), ("workspace", workspace))
    with torch.cuda.device(dev):
        _ok(_hybrid_scan(_ptr(S), _ptr(z), B, L, H, d, chunk_tokens, _ptr(workspace),
                         workspace.numel() * workspace.element_size(), _stream(stream, dev)))


def vattn_hybrid_chunk_noalloc(q, k, v, o, S, z, chunk_tokens, scale=None, stream=None):
    """vattn_hybrid_chunk for callers that cannot allocate device memory: the
    scratch is a static array inside libvattn (HYBRID_NOALLOC_MAX_BYTES);
    nothing is allocated here or in the library."""
    B, L, H, d = _check_hybrid(q, k, v, o, S, z)
    if scale is None:
        scale = d ** -0.5
    dev = _device(("q", q), ("k", k), ("v", v), ("o", o), ("S", S), ("z", z))
    with torch.cuda.device(dev):
        _ok(_hybrid_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(S), _ptr(z), B, L, H, d, chunk_tokens,
                            float(scale), _stream(stream, dev)))


# ------------------------------------------------------------------ misc
def vattn_check(stream=None):
    _ok(_check(_stream(stream)))


def vattn_selftest_umma(variant, a, b, out, stream=None):
    _ok(_selftest(variant, _bf16(a, "a"), _bf16(b, "b"), _ptr(out), _stream(stream)))


def vattn_selftest_wait_timeout(limit_us, stream=None):
    _ok(_selftest_timeout(limit_us, _stream(stream)))


def vattn_selftest_attention_timeout(q, k, v, o, limit_us, stream=None):
    """The two-tile attention kernel with one withheld softmax arrival and a
    short wait bound (include/vattn_selftest.h); q/k/v/o bf16 [1, L, H, d]."""
    _rank(q, "q", 4)
    B, L, H, d = q.shape
    if B != 1:
        raise ValueError("batch 1 only")
    for name, t in (("q", q), ("k", k), ("v", v), ("o", o)):
        _expect(t, name, (1, L, H, d), torch.bfloat16)
    dev = _device(("q", q), ("k", k), ("v", v), ("o", o))
    with torch.cuda.device(dev):
        _ok(_selftest_attn_timeout(_ptr(q), _ptr(k), _ptr(v), _ptr(o), L, H, d, limit_us, _stream(stream, dev)))


def vattn_selftest_ex2(variant, x, y, stream=None):
    """y = 2^x by the kernels' exponentials (0 polynomial, 1 packed polynomial, 2 MUFU)."""
    _expect(x, "x", None, torch.float32)
    _expect(y, "y", tuple(x.shape), torch.float32)
    dev = _device(("x", x), ("y", y))
    with torch.cuda.device(dev):
        _ok(_selftest_ex2(variant, _ptr(x), _ptr(y), x.numel(), _stream(stream, dev)))
