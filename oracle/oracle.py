"""Python access to the fp64 CPU oracle (oracle.cpp) and its ring-buffer model.

TEST INFRASTRUCTURE ONLY.  The oracle is the checker: only the tests, the
smoke check and the benchmark's CPU-baseline leg import this module.  It
never imports the CUDA package and the CUDA package never imports it.

All tensors in: numpy uint16 arrays of bfloat16 bit patterns, layout
[B, L, H, d].  All results out: float64 numpy arrays.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.cpp")
_LIB = os.path.join(_HERE, "liboracle.so")

MODES = {"full": 0, "chunk_causal": 1, "sliding": 2}


def build(force: bool = False) -> str:
    """Compile oracle.cpp into liboracle.so with g++ and OpenMP."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(["g++", "-O2", "-std=c++17", "-fopenmp", "-fPIC", "-shared",
                               "-o", tmp, _SRC])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        i, d, l = ctypes.c_int, ctypes.c_double, ctypes.c_long
        _lib.oracle_rope.argtypes = [P, P, i, i, i, i, i, i, i, i, i, d, i]
        _lib.oracle_attention.argtypes = [P, P, P, i, i, i, i, i, i, d, i, i, i, i, i, i, i,
                                          P, d, P, l, P, P]
        _lib.oracle_stream.argtypes = [P, P, P, i, i, i, i, i, i, d, i, P, d, P, l, P, P, i]
        _lib.oracle_hybrid_parallel.argtypes = [P, P, P, i, i, i, i, i, d, P, P, P, l, P]
        _lib.oracle_hybrid_recurrent.argtypes = [P, P, P, i, i, i, i, i, d, P, P, P, P]
        _lib.oracle_hybrid2_parallel.argtypes = [P, P, P, i, i, i, i, i, i, d, i, P, P, P, P, l, P]
        _lib.oracle_hybrid2_recurrent.argtypes = [P, P, P, i, i, i, i, i, i, d, i, P, P, P, P, P]
        _lib.oracle_merge.argtypes = [P, P, i, l, i, P, P]
        for f in ("oracle_rope", "oracle_attention", "oracle_stream",
                  "oracle_hybrid_parallel", "oracle_hybrid_recurrent", "oracle_hybrid2_parallel",
                  "oracle_hybrid2_recurrent", "oracle_merge", "oracle_num_threads"):
            getattr(_lib, f).restype = ctypes.c_int
    return _lib


def num_threads() -> int:
    return lib().oracle_num_threads()


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _bits(x):
    x = np.ascontiguousarray(x)
    assert x.dtype == np.uint16, "oracle inputs are bfloat16 bit patterns (uint16)"
    return x


def _rope_args(rope):
    if rope is None:
        return None, 0.0, None
    cfg = np.array([rope["Hg"], rope["Wg"], *rope["pairs"]], dtype=np.int32)
    return cfg, float(rope["theta"]), cfg


def rope(x, Hg, Wg, pairs, theta, t_offset=0):
    """3D-RoPE of x [B, L, H, d] (bf16 bits) -> float64 [B, L, H, d]."""
    x = _bits(x)
    B, L, H, d = x.shape
    out = np.empty(x.shape, dtype=np.float64)
    rc = lib().oracle_rope(_ptr(x), _ptr(out), B, L, H, d, Hg, Wg, pairs[0], pairs[1],
                           pairs[2], float(theta), t_offset)
    assert rc == 0, "oracle_rope rejected its arguments"
    return out


def attention(q, k, v, scale, mode="full", F=0, chunk=1, wb=0, wf=0,
              q_frame_offset=0, k_frame_offset=0, rope=None, rows=None):
    """Masked softmax attention.

    rope: None or dict(Hg=, Wg=, pairs=(t, h, w), theta=).
    rows: None (all rows; returns o [B, Lq, H, d], lse [B, H, Lq]) or an
    int32 array [n, 3] of (b, h, i) (returns o [n, d], lse [n]).
    """
    q, k, v = _bits(q), _bits(k), _bits(v)
    B, Lq, H, d = q.shape
    Lk, Hkv = k.shape[1], k.shape[2]
    if rows is None:
        o = np.empty((B, Lq, H, d))
        lse = np.empty((B, H, Lq))
        n = 0
    else:
        rows = np.ascontiguousarray(rows, dtype=np.int32)
        n = rows.shape[0]
        o = np.empty((n, d))
        lse = np.empty((n,))
    cfg, theta, _ = _rope_args(rope)
    rc = lib().oracle_attention(_ptr(q), _ptr(k), _ptr(v), B, Lq, Lk, H, Hkv, d, float(scale),
                                MODES[mode], F, chunk, wb, wf, q_frame_offset, k_frame_offset,
                                _ptr(cfg), theta, _ptr(rows), n, _ptr(o), _ptr(lse))
    assert rc == 0, "oracle_attention rejected its arguments"
    return o, lse


def stream(q, k, v, F, scale, wb, rope=None, rows=None, window_relative=False):
    """Frame-by-frame streaming attention over a whole sequence of frames.

    q/k/v: [B, n_frames * F, H, d].  Returns o [n, d], lse [n] for rows
    (b, h, i); rows=None evaluates every row (o [B, L, H, d]).  With rope, a
    stream frame of F tokens holds F / (Hg * Wg) latent frames; RoPE t counts
    latent frames from 0 (absolute) or from the first frame of the query's
    window (window_relative).
    """
    q, k, v = _bits(q), _bits(k), _bits(v)
    B, L, H, d = q.shape
    Hkv = k.shape[2]
    full = rows is None
    if full:
        bb, ii, hh = np.meshgrid(np.arange(B), np.arange(L), np.arange(H), indexing="ij")
        rows = np.stack([bb.ravel(), hh.ravel(), ii.ravel()], axis=1)
    rows = np.ascontiguousarray(rows, dtype=np.int32)
    n = rows.shape[0]
    o = np.empty((n, d))
    lse = np.empty((n,))
    cfg, theta, _ = _rope_args(rope)
    rc = lib().oracle_stream(_ptr(q), _ptr(k), _ptr(v), B, L // F, F, H, Hkv, d, float(scale), wb,
                             _ptr(cfg), theta, _ptr(rows), n, _ptr(o), _ptr(lse), int(bool(window_relative)))
    assert rc == 0
    if full:
        return o.reshape(B, L, H, d), lse.reshape(B, L, H).transpose(0, 2, 1)
    return o, lse


def ring_model(k_frames, v_frames, capacity):
    """Expected ring contents after appending frames 0..n-1 in order.

    k_frames/v_frames: [n, B, F, Hkv, d] uint16.  The ring keeps frame f in
    slot f mod capacity; frame_ids[slot] is the last frame written there,
    -1 for a slot never written.  Returns (k_ring, v_ring, frame_ids) with
    ring layout [capacity, B, F, Hkv, d].
    """
    n = k_frames.shape[0]
    shape = (capacity,) + tuple(k_frames.shape[1:])
    kr = np.zeros(shape, dtype=np.uint16)
    vr = np.zeros(shape, dtype=np.uint16)
    ids = np.full(capacity, -1, dtype=np.int32)
    for f in range(n):
        s = f % capacity
        kr[s] = k_frames[f]
        vr[s] = v_frames[f]
        ids[s] = f
    return kr, vr, ids


def hybrid_parallel(q, k, v, chunk_tokens, scale, rows, S0=None, z0=None):
    """Hybrid chunk attention, parallel form, for rows (b, h, i) -> o [n, d]."""
    q, k, v = _bits(q), _bits(k), _bits(v)
    B, L, H, d = q.shape
    rows = np.ascontiguousarray(rows, dtype=np.int32)
    o = np.empty((rows.shape[0], d))
    S0 = None if S0 is None else np.ascontiguousarray(S0, dtype=np.float64)
    z0 = None if z0 is None else np.ascontiguousarray(z0, dtype=np.float64)
    rc = lib().oracle_hybrid_parallel(_ptr(q), _ptr(k), _ptr(v), B, L, H, d, chunk_tokens,
                                      float(scale), _ptr(S0), _ptr(z0), _ptr(rows),
                                      rows.shape[0], _ptr(o))
    assert rc == 0
    return o


def hybrid_recurrent(q, k, v, chunk_tokens, scale, S=None, z=None, row_mask=None):
    """Hybrid chunk attention, recurrent form.

    Returns (o [B, L, H, d], S_out [B, H, d, d], z_out [B, H, d]).  S / z are
    the incoming state (zeros when None).  row_mask [B, H, L] (bool) limits
    which output rows are evaluated (others are left as NaN).
    """
    q, k, v = _bits(q), _bits(k), _bits(v)
    B, L, H, d = q.shape
    S_io = np.zeros((B, H, d, d)) if S is None else np.array(S, dtype=np.float64, copy=True)
    z_io = np.zeros((B, H, d)) if z is None else np.array(z, dtype=np.float64, copy=True)
    o = np.full((B, L, H, d), np.nan)
    m = None if row_mask is None else np.ascontiguousarray(row_mask, dtype=np.int8)
    rc = lib().oracle_hybrid_recurrent(_ptr(q), _ptr(k), _ptr(v), B, L, H, d, chunk_tokens,
                                       float(scale), _ptr(S_io), _ptr(z_io), _ptr(m), _ptr(o))
    assert rc == 0
    return o, S_io, z_io


def _coef(fmap, coef, H):
    if fmap == "elu":
        return 0, None
    c = np.ascontiguousarray(coef, dtype=np.float64)
    assert c.shape == (2, H, 4), "coef: [2 (q, k), H, 4] polynomial coefficients a0..a3"
    return 1, c


def hybrid2_parallel(q, k, v, chunk_tokens, scale, rows, overlap=0, fmap="elu", coef=None, S0=None, z0=None):
    """General hybrid chunk attention (polynomial feature map, chunk
    overlap), parallel form, for rows (b, h, i) -> o [n, d]."""
    q, k, v = _bits(q), _bits(k), _bits(v)
    B, L, H, d = q.shape
    fm, c = _coef(fmap, coef, H)
    rows = np.ascontiguousarray(rows, dtype=np.int32)
    o = np.empty((rows.shape[0], d))
    S0 = None if S0 is None else np.ascontiguousarray(S0, dtype=np.float64)
    z0 = None if z0 is None else np.ascontiguousarray(z0, dtype=np.float64)
    rc = lib().oracle_hybrid2_parallel(_ptr(q), _ptr(k), _ptr(v), B, L, H, d, chunk_tokens, overlap,
                                       float(scale), fm, _ptr(c), _ptr(S0), _ptr(z0), _ptr(rows),
                                       rows.shape[0], _ptr(o))
    assert rc == 0
    return o


def hybrid2_recurrent(q, k, v, chunk_tokens, scale, overlap=0, fmap="elu", coef=None, S=None, z=None,
                      row_mask=None):
    """General hybrid chunk attention, recurrent form.  Returns
    (o [B, L, H, d], S_out [B, H, d, d], z_out [B, H, d])."""
    q, k, v = _bits(q), _bits(k), _bits(v)
    B, L, H, d = q.shape
    fm, c = _coef(fmap, coef, H)
    S_io = np.zeros((B, H, d, d)) if S is None else np.array(S, dtype=np.float64, copy=True)
    z_io = np.zeros((B, H, d)) if z is None else np.array(z, dtype=np.float64, copy=True)
    o = np.full((B, L, H, d), np.nan)
    m = None if row_mask is None else np.ascontiguousarray(row_mask, dtype=np.int8)
    rc = lib().oracle_hybrid2_recurrent(_ptr(q), _ptr(k), _ptr(v), B, L, H, d, chunk_tokens, overlap,
                                        float(scale), fm, _ptr(c), _ptr(S_io), _ptr(z_io), _ptr(m), _ptr(o))
    assert rc == 0
    return o, S_io, z_io


def merge(o_parts, lse_parts):
    """Combination of R partial attentions over disjoint key sets:
    o_parts [R, n, d], lse_parts [R, n] (float64) -> (o [n, d], lse [n])."""
    o_parts = np.ascontiguousarray(o_parts, dtype=np.float64)
    lse_parts = np.ascontiguousarray(lse_parts, dtype=np.float64)
    R, n, d = o_parts.shape
    assert lse_parts.shape == (R, n)
    o = np.empty((n, d))
    lse = np.empty((n,))
    rc = lib().oracle_merge(_ptr(o_parts), _ptr(lse_parts), R, n, d, _ptr(o), _ptr(lse))
    assert rc == 0
    return o, lse
