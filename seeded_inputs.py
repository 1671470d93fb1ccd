"""Seeded synthetic inputs for the spatiotemporal attention workloads.

This module is the only thing the fp64 oracle and the CUDA path have in
common: it draws the random tensors both sides consume.  It holds none of the
method's arithmetic (no rotary embedding, no softmax, no masks): only a
counter-based random generator, a Gaussian transform, the rounding of doubles
to bfloat16 bit patterns, and the workload shapes.

Generator (stated so that it can be re-implemented anywhere):
  * splitmix64 (Steele, Lea, Flood, "Fast splittable pseudorandom number
    generators", OOPSLA 2014): element i of stream ``seed`` is
    mix(seed + (i + 1) * 0x9E3779B97F4A7C15) with the published finaliser.
  * uniforms u = ((z >> 11) + 0.5) * 2**-53, strictly inside (0, 1).
  * Box-Muller on consecutive uniform pairs (u1, u2):
    r = sqrt(-2 ln u1), x0 = r cos(2 pi u2), x1 = r sin(2 pi u2), in double.
  * each double is rounded once, to nearest with ties to even, to bfloat16
    (8 significant bits); the result is returned as uint16 bit patterns.

Seeds follow 0x5EED0000 + 16 * config_index + {0: q, 1: k, 2: v}.
"""
from __future__ import annotations

import numpy as np

_GOLDEN = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)


def splitmix64(seed: int, n: int, start: int = 0) -> np.ndarray:
    """Elements start..start+n-1 of the splitmix64 stream for ``seed``."""
    with np.errstate(over="ignore"):
        idx = np.arange(start + 1, start + n + 1, dtype=np.uint64)
        z = np.uint64(seed & 0xFFFFFFFFFFFFFFFF) + idx * _GOLDEN
        z = (z ^ (z >> np.uint64(30))) * _M1
        z = (z ^ (z >> np.uint64(27))) * _M2
        z = z ^ (z >> np.uint64(31))
    return z


def uniform01(seed: int, n: int, start: int = 0) -> np.ndarray:
    z = splitmix64(seed, n, start)
    return ((z >> np.uint64(11)).astype(np.float64) + 0.5) * (2.0 ** -53)


def normal_f64(seed: int, n: int) -> np.ndarray:
    """n standard normal doubles (Box-Muller on consecutive uniform pairs)."""
    m = (n + 1) // 2
    u = uniform01(seed, 2 * m)
    u1, u2 = u[0::2], u[1::2]
    r = np.sqrt(-2.0 * np.log(u1))
    out = np.empty(2 * m, dtype=np.float64)
    out[0::2] = r * np.cos(2.0 * np.pi * u2)
    out[1::2] = r * np.sin(2.0 * np.pi * u2)
    return out[:n]


def f64_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round doubles to bfloat16 (nearest, ties to even) in a single rounding.

    Values are kept to 8 significant bits via frexp / rint (rint rounds half
    to even); the rounded value is exact in float32, whose upper 16 bits are
    the bfloat16 pattern.  Finite inputs within float32 range only.
    """
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)                      # x = m * 2**e, 0.5 <= |m| < 1
    r = np.ldexp(np.rint(np.ldexp(m, 8)), e - 8)
    bits = r.astype(np.float32).view(np.uint32)
    return (bits >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f64(b: np.ndarray) -> np.ndarray:
    """Widen bfloat16 bit patterns to doubles (exact)."""
    b = np.asarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def normal_bf16(seed: int, shape) -> np.ndarray:
    """N(0, 1) samples rounded to bfloat16, as a uint16 array of ``shape``."""
    n = int(np.prod(shape))
    return f64_to_bf16_bits(normal_f64(seed, n)).reshape(shape)


def seed_for(config_index: int, which: str) -> int:
    return 0x5EED0000 + 16 * config_index + {"q": 0, "k": 1, "v": 2}[which]


# --------------------------------------------------------------------------
# Workload shapes (synthetic stand-ins for the pages' latent videos).
# Token n of a T x Hg x Wg latent grid is (t, h, w) in row-major order.
# --------------------------------------------------------------------------
CONFIGS = {
    # index 0: tiny full bidirectional 3D-RoPE attention
    "tiny": dict(index=0, B=1, H=2, d=64, T=3, Hg=4, Wg=4,
                 pairs=(12, 10, 10), theta=10000.0, mode="full"),
    # index 1: Wan2.1-1.3B-like full attention (480x832, 81 frames)
    "wan13b": dict(index=1, B=1, H=12, d=128, T=21, Hg=30, Wg=52,
                   pairs=(22, 21, 21), theta=10000.0, mode="full"),
    # index 2: FlashDecoder-style streaming (34x60 tokens per frame)
    "stream": dict(index=2, B=1, H=16, d=64, T=32, Hg=34, Wg=60,
                   pairs=(12, 10, 10), theta=10000.0, mode="stream",
                   window_back=4, capacity=4),
    # index 3: MobileWan-style hybrid chunk attention (31 frames of 15x26)
    "hybrid": dict(index=3, B=1, H=24, d=128, T=31, Hg=15, Wg=26,
                   pairs=None, theta=None, mode="hybrid", chunk_frames=3),
    # the MobileWan page variant on the same inputs as "hybrid": chunks of
    # T_c = 4 latent frames whose softmax reaches T_o = 2 frames into the
    # previous chunk, degree-3 polynomial feature maps (synthetic
    # coefficients, poly_coef(seed 0x9017, H))
    "hybrid_page": dict(index=3, B=1, H=24, d=128, T=31, Hg=15, Wg=26,
                        pairs=None, theta=None, mode="hybrid", chunk_frames=4,
                        overlap_frames=2, coef_seed=0x9017),
    # index 4: Wan2.1-14B-like 720p, full and chunk-causal (chunk = 3 frames)
    "wan14b": dict(index=4, B=1, H=40, d=128, T=21, Hg=45, Wg=80,
                   pairs=(22, 21, 21), theta=10000.0, mode="full+chunk",
                   chunk_frames=3),
    # indices 5-7: FlashDecoder-XL-shaped streaming (24 query heads sharing 3
    # KV heads, head dim 64, window W_frm = 2: itself + 1 previous frame),
    # Wan2.2 latent grids of 480p (30x52) and 720p (45x80), positions
    # relative to the window; xl480_refine: a temporal-refinement layer
    # (r_t = 4 latent frames of 30x52 per step, window r_t * W_frm frames)
    "xl480": dict(index=5, B=1, H=24, Hkv=3, d=64, T=16, Hg=30, Wg=52, sub=1,
                  pairs=(12, 10, 10), theta=10000.0, mode="stream",
                  window_back=1, capacity=2),
    "xl720": dict(index=6, B=1, H=24, Hkv=3, d=64, T=16, Hg=45, Wg=80, sub=1,
                  pairs=(12, 10, 10), theta=10000.0, mode="stream",
                  window_back=1, capacity=2),
    "xl480_refine": dict(index=7, B=1, H=24, Hkv=3, d=64, T=8, Hg=30, Wg=52, sub=4,
                         pairs=(12, 10, 10), theta=10000.0, mode="stream",
                         window_back=1, capacity=2),
}


def poly_coef(seed: int, H: int) -> np.ndarray:
    """Synthetic coefficients (a0, a1, a2, a3) of degree-3 polynomial feature
    maps, one per head for q (index 0) and for k (index 1): [2, H, 4]
    float64 values that are exactly representable in fp32.  Ranges keep the
    maps positive on average over N(0, 1) inputs: a0 in [0.5, 1), a1 in
    [0.2, 0.5), a2 in [0.1, 0.3), a3 in [0, 0.05)."""
    u = uniform01(seed, 2 * H * 4).reshape(2, H, 4)
    lo = np.array([0.5, 0.2, 0.1, 0.0])
    hi = np.array([1.0, 0.5, 0.3, 0.05])
    return (lo + u * (hi - lo)).astype(np.float32).astype(np.float64)


def qkv(config: str, L: int | None = None, H: int | None = None):
    """Seeded q, k, v (uint16 bf16 bits, layout [B, L, H, d]) for a config.

    ``L`` / ``H`` may shrink the token or head count (same seeds, prefix of
    the same stream order is NOT implied: a smaller shape is a new draw).
    """
    c = CONFIGS[config]
    L = c["T"] * c.get("sub", 1) * c["Hg"] * c["Wg"] if L is None else L
    H = c["H"] if H is None else H
    Hkv = c.get("Hkv", H) if H == c["H"] else H
    return (normal_bf16(seed_for(c["index"], "q"), (c["B"], L, H, c["d"])),
            normal_bf16(seed_for(c["index"], "k"), (c["B"], L, Hkv, c["d"])),
            normal_bf16(seed_for(c["index"], "v"), (c["B"], L, Hkv, c["d"])))


def sample_rows(seed: int, n: int, B: int, H: int, L: int, forced=()) -> np.ndarray:
    """n seeded (b, h, i) query-row triples plus forced token indices.

    Forced tokens are given as token indices i; each is paired with a seeded
    (b, h).  Returns an int32 array of shape [rows, 3], duplicates removed,
    sorted by (b, h, i).
    """
    z = splitmix64(seed ^ 0x5A5A5A5A, 3 * n + 2 * len(forced))
    b = (z[0:n] % np.uint64(B)).astype(np.int64)
    h = (z[n:2 * n] % np.uint64(H)).astype(np.int64)
    i = (z[2 * n:3 * n] % np.uint64(L)).astype(np.int64)
    rows = [np.stack([b, h, i], axis=1)]
    if len(forced):
        f = np.asarray([x for x in forced if 0 <= x < L], dtype=np.int64)
        zf = z[3 * n:3 * n + 2 * len(f)]
        fb = (zf[0::2][:len(f)] % np.uint64(B)).astype(np.int64)
        fh = (zf[1::2][:len(f)] % np.uint64(H)).astype(np.int64)
        rows.append(np.stack([fb, fh, f], axis=1))
    r = np.unique(np.concatenate(rows, axis=0), axis=0)
    return r.astype(np.int32)


def boundary_tokens(L: int, period: int, tile: int = 128) -> list:
    """Forced edge rows: first/last token, tile edges 127/128/129, every
    ``period`` boundary +-1 (frames or chunks) and the last partial tile."""
    s = {0, L - 1, 127, 128, 129, (L // tile) * tile, (L // tile) * tile - 1}
    if period:
        for p in range(period, L, period):
            s.update({p - 1, p, p + 1})
    return sorted(x for x in s if 0 <= x < L)
