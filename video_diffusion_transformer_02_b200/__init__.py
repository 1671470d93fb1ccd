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
_kv_init = _sig("vattn_kvcache_init", _I, ctypes.POINTER(_P), _P, _P, _P, _I, _I, _I, _I, _I, _P)
_kv_append = _sig("vattn_kvcache_append", _I, _P, _P, _P, _I, _P)
_attention_stream = _sig("vattn_attention_stream", _I, _P, _P, _P, _P, _P, _P, _I, _I, _I, _F, _RP,
                         _P, _P)
_kv_ids = _sig("vattn_kvcache_frame_ids", _I, _P, _P)
_kv_restore = _sig("vattn_kvcache_restore", _I, _P, _P, _P)
_kv_rope = _sig("vattn_kvcache_enable_rope", _I, _P, _P, _RP, _P, _P)
_kv_destroy = _sig("vattn_kvcache_destroy", _I, _P)
_hyb_ws = _sig("vattn_hybrid_workspace_bytes", _S, _I, _I, _I, _I, _I)
_hybrid = _sig("vattn_hybrid_chunk", _I, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _F, _P, _S, _P)
_hybrid_noalloc = _sig("vattn_hybrid_chunk_noalloc", _I, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _F, _P)
_selftest = _sig("vattn_selftest_umma", _I, _I, _P, _P, _P, _P)
_selftest_timeout = _sig("vattn_selftest_wait_timeout", _I, ctypes.c_uint32, _P)
HYBRID_NOALLOC_MAX_BYTES = 32 << 20


def status_string(status: int) -> str:
    return _status_string(status).decode()


def last_error() -> str:
    return _last_error().decode()


def _ok(status: int):
    if status != OK:
        raise VattnError(status, last_error())


def _stream(stream=None) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
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


def _rope_c(rope):
    if rope is None:
        return None
    return ctypes.byref(rope.c())


# ------------------------------------------------------------------- RoPE
def vattn_rope_table_bytes(rope: Rope, d: int) -> int:
    return _table_bytes(ctypes.byref(rope.c()), d)


def vattn_rope_table_build(rope: Rope, d: int, table: torch.Tensor, stream=None):
    _ok(_table_build(ctypes.byref(rope.c()), d, _ptr(table), _stream(stream)))


def rope_table(rope: Rope, d: int, device="cuda") -> torch.Tensor:
    """Allocate (torch) and fill the fp32 cos/sin table of a configuration."""
    n = vattn_rope_table_bytes(rope, d)
    if n == 0:
        raise VattnError(ERR_INVALID_ARG, last_error())
    t = torch.empty(n // 4, dtype=torch.float32, device=device)
    vattn_rope_table_build(rope, d, t)
    return t


def vattn_rope_qk(q, k, q_out, k_out, rope: Rope, table, frame_offset=0, stream=None):
    ref = q if q is not None else k
    B, L = ref.shape[0], ref.shape[1]
    d = ref.shape[3]
    H = q.shape[2] if q is not None else 1
    Hkv = k.shape[2] if k is not None else 1
    _ok(_rope_qk(_bf16(q, "q") if q is not None else None, _bf16(k, "k") if k is not None else None,
                 _ptr(q_out), _ptr(k_out), B, L, H, Hkv, d, _rope_c(rope), _ptr(table),
                 frame_offset, _stream(stream)))


# -------------------------------------------------------------- attention
def vattn_attention_workspace_bytes(B, Lk, Hkv, d, rope: Rope | None) -> int:
    return _attn_ws(B, Lk, Hkv, d, _rope_c(rope))


def vattn_attention(q, k, v, o, lse=None, scale=None, mode="full", tokens_per_frame=0,
                    chunk_frames=1, window_back=0, window_fwd=0, q_frame_offset=0,
                    k_frame_offset=0, rope: Rope | None = None, table=None, workspace=None,
                    fuse_k_rope=False, stream=None):
    """o = masked softmax attention (see include/vattn.h); q/k/v/o [B, L, H, d] bf16.

    With rope, keys are rotated once into `workspace` (allocated here with
    torch when not given); fuse_k_rope=True passes no workspace, so the kernel
    rotates every K tile in shared memory instead.
    """
    B, Lq, H, d = q.shape
    Lk, Hkv = k.shape[1], k.shape[2]
    if scale is None:
        scale = d ** -0.5
    m = MODES[mode] if isinstance(mode, str) else int(mode)
    ws_ptr, ws_bytes = None, 0
    if rope is not None and not fuse_k_rope:
        need = vattn_attention_workspace_bytes(B, Lk, Hkv, d, rope)
        if workspace is None:
            workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
        ws_ptr, ws_bytes = _ptr(workspace), workspace.numel() * workspace.element_size()
    _ok(_attention(_bf16(q, "q"), _bf16(k, "k"), _bf16(v, "v"), _bf16(o, "o"), _ptr(lse), B, Lq, Lk,
                   H, Hkv, d, float(scale), m, tokens_per_frame, chunk_frames, window_back,
                   window_fwd, q_frame_offset, k_frame_offset, _rope_c(rope), _ptr(table), ws_ptr,
                   ws_bytes, _stream(stream)))


# ---------------------------------------------------------------- KV ring
class KVCache:
    """Rolling KV cache over caller-owned ring storage (torch tensors).

    k_ring, v_ring: bf16 [capacity, B, F, Hkv, d]; frame_ids: int32 [capacity].
    """

    def __init__(self, k_ring, v_ring, frame_ids, stream=None):
        cap, B, F, Hkv, d = k_ring.shape
        if frame_ids.dtype != torch.int32:
            raise TypeError("frame_ids must be int32")
        self.k_ring, self.v_ring, self.frame_ids = k_ring, v_ring, frame_ids
        self.capacity, self.B, self.F, self.Hkv, self.d = cap, B, F, Hkv, d
        h = ctypes.c_void_p()
        _ok(_kv_init(ctypes.byref(h), _bf16(k_ring, "k_ring"), _bf16(v_ring, "v_ring"), _ptr(frame_ids),
                     cap, B, F, Hkv, d, _stream(stream)))
        self._h = h

    def append(self, k, v, frame_idx, stream=None):
        vattn_kvcache_append(self, k, v, frame_idx, stream)

    def attend(self, q, k_cur, v_cur, o, frame_idx, window_back, scale=None, lse=None,
               rope=None, table=None, stream=None):
        vattn_attention_stream(self, q, k_cur, v_cur, o, lse, frame_idx, window_back, scale, rope,
                               table, stream)

    def host_frame_ids(self):
        arr = (ctypes.c_int32 * self.capacity)()
        _ok(_kv_ids(self._h, arr))
        return list(arr)

    def restore(self, host_ids, stream=None):
        arr = (ctypes.c_int32 * self.capacity)(*host_ids)
        _ok(_kv_restore(self._h, arr, _stream(stream)))

    def enable_rope(self, k_ring_rot, rope: Rope, table, stream=None):
        """Rotated-key ring (bf16 [capacity + 1, B, F, Hkv, d]): keys rotated once per frame."""
        self.k_ring_rot = k_ring_rot
        _ok(_kv_rope(self._h, _bf16(k_ring_rot, "k_ring_rot"), ctypes.byref(rope.c()), _ptr(table),
                     _stream(stream)))

    def close(self):
        if getattr(self, "_h", None):
            _kv_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def vattn_kvcache_append(cache: KVCache, k, v, frame_idx, stream=None):
    _ok(_kv_append(cache._h, _bf16(k, "k"), _bf16(v, "v"), frame_idx, _stream(stream)))


def vattn_attention_stream(cache: KVCache, q, k_cur, v_cur, o, lse, frame_idx, window_back,
                           scale=None, rope=None, table=None, stream=None):
    H = q.shape[2]
    if scale is None:
        scale = cache.d ** -0.5
    _ok(_attention_stream(cache._h, _bf16(q, "q"), _bf16(k_cur, "k_cur"), _bf16(v_cur, "v_cur"),
                          _bf16(o, "o"), _ptr(lse), H, frame_idx, window_back, float(scale),
                          _rope_c(rope), _ptr(table), _stream(stream)))


# ----------------------------------------------------------------- hybrid
def vattn_hybrid_workspace_bytes(B, L, H, d, chunk_tokens) -> int:
    return _hyb_ws(B, L, H, d, chunk_tokens)


def vattn_hybrid_chunk(q, k, v, o, S, z, chunk_tokens, scale=None, workspace=None, stream=None):
    """Hybrid chunk attention; S [B,H,d,d] and z [B,H,d] fp32 are updated in place."""
    B, L, H, d = q.shape
    if scale is None:
        scale = d ** -0.5
    need = vattn_hybrid_workspace_bytes(B, L, H, d, chunk_tokens)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    _ok(_hybrid(_bf16(q, "q"), _bf16(k, "k"), _bf16(v, "v"), _bf16(o, "o"), _ptr(S), _ptr(z), B, L,
                H, d, chunk_tokens, float(scale), _ptr(workspace), workspace.numel() * workspace.element_size(),
                _stream(stream)))


def vattn_hybrid_chunk_noalloc(q, k, v, o, S, z, chunk_tokens, scale=None, stream=None):
    """vattn_hybrid_chunk for callers that cannot allocate device memory: the
    scratch is a static array inside libvattn (HYBRID_NOALLOC_MAX_BYTES);
    nothing is allocated here or in the library."""
    B, L, H, d = q.shape
    if scale is None:
        scale = d ** -0.5
    _ok(_hybrid_noalloc(_bf16(q, "q"), _bf16(k, "k"), _bf16(v, "v"), _bf16(o, "o"), _ptr(S), _ptr(z), B, L,
                        H, d, chunk_tokens, float(scale), _stream(stream)))


# ------------------------------------------------------------------ misc
def vattn_check(stream=None):
    _ok(_check(_stream(stream)))


def vattn_selftest_umma(variant, a, b, out, stream=None):
    _ok(_selftest(variant, _bf16(a, "a"), _bf16(b, "b"), _ptr(out), _stream(stream)))


def vattn_selftest_wait_timeout(limit_us, stream=None):
    _ok(_selftest_timeout(limit_us, _stream(stream)))
