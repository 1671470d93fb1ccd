"""Pins for the fp64 oracle: checks against what the pages and mathematics fix.

Each test ties an oracle function to something other than itself: textbook
values of cos/sin, closed forms of attention outputs for inputs whose weights
are known, identities between masking modes that the pages' definitions
imply, equivalence of the recurrent and parallel forms of causal linear
attention, and an explicit-matrix brute force on tiny grids.
"""
import math

import numpy as np
import pytest

import oracle
import seeded_inputs as si

TINY = si.CONFIGS["tiny"]


def bf16(x):
    return si.f64_to_bf16_bits(np.asarray(x, dtype=np.float64))


# ----------------------------------------------------------------- generator
def test_splitmix64_published_vector():
    # splitmix64 from state 0: the first outputs published with the algorithm
    # (Vigna's reference splitmix64.c / Java SplittableRandom).
    z = si.splitmix64(0, 3)
    assert [int(x) for x in z] == [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F]


def test_bf16_round_nearest_even():
    one = 1.0
    vals = [one, one + 2 ** -8, one + 3 * 2 ** -8, one + 2 ** -8 + 2 ** -30, -2.5, 0.0]
    got = [int(b) for b in si.f64_to_bf16_bits(np.array(vals))]
    # 1+2^-8 is a tie -> even (1.0); 1+3*2^-8 is a tie -> even (1+2^-6 = 0x3F82);
    # just above the tie rounds up.
    assert got == [0x3F80, 0x3F80, 0x3F82, 0x3F81, 0xC020, 0x0000]
    x = si.normal_f64(7, 1000)
    back = si.bf16_bits_to_f64(si.f64_to_bf16_bits(x))
    assert np.all(np.abs(back - x) <= np.abs(x) * 2.0 ** -8 + 1e-300)


def test_normal_moments():
    x = si.normal_f64(123, 200000)
    assert abs(x.mean()) < 0.01 and abs(x.std() - 1.0) < 0.01


# ---------------------------------------------------------------------- RoPE
def _rope_grid(T, Hg, Wg, pairs, d):
    return dict(Hg=Hg, Wg=Wg, pairs=pairs, theta=10000.0)


def _unit_pair_tensor(L, H, d, j):
    x = np.zeros((1, L, H, d))
    x[..., 2 * j] = 1.0
    return bf16(x)


@pytest.mark.parametrize("axis_pair,pos,expect", [
    # t-group pair i=0 at t=1: angle 1 rad
    ((0, "t"), 1, (0.5403023058681398, 0.8414709848078965)),
    # t-group pair i=3 of n_t=12: omega = 10000^(-3/12) = 0.1
    ((3, "t"), 1, (0.9950041652780258, 0.09983341664682815)),
    # t-group pair i=6 of n_t=12: omega = 0.01, at t=2: angle 0.02
    ((6, "t"), 2, (0.9998000066665778, 0.019998666693333080)),
    # h-group first pair at h=2: angle 2
    ((0, "h"), 2, (-0.4161468365471424, 0.9092974268256817)),
    # w-group first pair at w=3: angle 3
    ((0, "w"), 3, (-0.9899924966004454, 0.1411200080598672)),
])
def test_rope_textbook_angles(axis_pair, pos, expect):
    i, axis = axis_pair
    pt, ph, pw = 12, 10, 10
    d, Hg, Wg = 64, 4, 5
    j = {"t": i, "h": pt + i, "w": pt + ph + i}[axis]
    t, h, w = {"t": (pos, 0, 0), "h": (0, pos, 0), "w": (0, 0, pos)}[axis]
    n = (t * Hg + h) * Wg + w
    L = n + 1
    x = _unit_pair_tensor(L, 1, d, j)
    out = oracle.rope(x, Hg, Wg, (pt, ph, pw), 10000.0)
    c, s = out[0, n, 0, 2 * j], out[0, n, 0, 2 * j + 1]
    assert abs(c - expect[0]) < 1e-15 and abs(s - expect[1]) < 1e-15
    # all other channels stay zero
    rest = np.delete(out[0, n, 0], [2 * j, 2 * j + 1])
    assert np.all(rest == 0.0)


def test_rope_identity_at_origin_and_norm():
    q, _, _ = si.qkv("tiny")
    out = oracle.rope(q, 4, 4, TINY["pairs"], TINY["theta"])
    x = si.bf16_bits_to_f64(q)
    assert np.array_equal(out[:, 0], x[:, 0])          # token 0 sits at (0,0,0)
    assert np.allclose(np.linalg.norm(out, axis=-1), np.linalg.norm(x, axis=-1), rtol=0, atol=1e-12)


def test_rope_relative_offset_invariance():
    # Rotations compose: (R_{p+c} q).(R_{p'+c} k) == (R_p q).(R_p' k) for a
    # shift c on any of the three axes.
    rng = np.random.default_rng(0)
    d, Hg, Wg, T = 64, 6, 7, 5
    pairs = (12, 10, 10)
    qv = rng.standard_normal(d)
    kv = rng.standard_normal(d)
    L = T * Hg * Wg
    Q = np.broadcast_to(bf16(qv), (1, L, 1, d)).copy()
    K = np.broadcast_to(bf16(kv), (1, L, 1, d)).copy()
    Rq = oracle.rope(Q, Hg, Wg, pairs, 1e4)[0, :, 0]
    Rk = oracle.rope(K, Hg, Wg, pairs, 1e4)[0, :, 0]

    def tok(t, h, w):
        return (t * Hg + h) * Wg + w

    cases = [((0, 1, 2), (2, 3, 1), (1, 0, 0)), ((0, 1, 2), (2, 3, 1), (0, 2, 0)),
             ((0, 1, 2), (2, 3, 1), (0, 0, 4)), ((1, 0, 0), (0, 2, 3), (2, 3, 3))]
    for a, b, c in cases:
        base = Rq[tok(*a)] @ Rk[tok(*b)]
        sa = tuple(x + y for x, y in zip(a, c))
        sb = tuple(x + y for x, y in zip(b, c))
        shifted = Rq[tok(*sa)] @ Rk[tok(*sb)]
        assert abs(base - shifted) < 1e-12


def test_rope_frame_offset_shifts_t():
    q, _, _ = si.qkv("tiny")
    F = 16
    a = oracle.rope(q[:, F:], 4, 4, TINY["pairs"], 1e4, t_offset=1)
    b = oracle.rope(q, 4, 4, TINY["pairs"], 1e4)[:, F:]
    assert np.array_equal(a, b)


# ----------------------------------------------------------------- attention
def brute_attention(q, k, v, scale, allowed):
    """Explicit matrix definition: S = scale Q K^T, masked, softmax, times V."""
    S = scale * (q @ k.T)
    S = np.where(allowed, S, -np.inf)
    m = S.max(axis=1, keepdims=True)
    P = np.exp(S - m)
    P /= P.sum(axis=1, keepdims=True)
    return P @ v


def frame_mask(Lq, Lk, F, mode, chunk=1, wb=0, wf=0, qoff=0, koff=0):
    fq = qoff + np.arange(Lq)[:, None] // F
    fk = koff + np.arange(Lk)[None, :] // F
    if mode == "full":
        return np.ones((Lq, Lk), dtype=bool)
    if mode == "chunk_causal":
        return (fk // chunk) <= (fq // chunk)
    return (fk >= fq - wb) & (fk <= fq + wf)


@pytest.mark.parametrize("mode,kw", [("full", {}), ("chunk_causal", dict(chunk=2)),
                                     ("sliding", dict(wb=1, wf=0)), ("sliding", dict(wb=0, wf=1))])
def test_attention_brute_force_tiny(mode, kw):
    q, k, v = si.qkv("tiny")
    B, L, H, d = q.shape
    F = 16
    scale = 1 / 8
    o, lse = oracle.attention(q, k, v, scale, mode=mode, F=F, **kw)
    Q, K, V = (si.bf16_bits_to_f64(x) for x in (q, k, v))
    mask = frame_mask(L, L, F, mode, **kw)
    for h in range(H):
        ref = brute_attention(Q[0, :, h], K[0, :, h], V[0, :, h], scale, mask)
        assert np.max(np.abs(o[0, :, h] - ref)) < 1e-12


def test_attention_brute_force_tiny_rope():
    q, k, v = si.qkv("tiny")
    rope = dict(Hg=4, Wg=4, pairs=TINY["pairs"], theta=1e4)
    o, _ = oracle.attention(q, k, v, 1 / 8, rope=rope)
    Rq = oracle.rope(q, 4, 4, TINY["pairs"], 1e4)
    Rk = oracle.rope(k, 4, 4, TINY["pairs"], 1e4)
    V = si.bf16_bits_to_f64(v)
    for h in range(2):
        ref = brute_attention(Rq[0, :, h], Rk[0, :, h], V[0, :, h], 1 / 8, np.ones((48, 48), bool))
        assert np.max(np.abs(o[0, :, h] - ref)) < 1e-12


def test_softmax_rows_sum_to_one():
    q, k, _ = si.qkv("tiny")
    ones = bf16(np.ones((1, 48, 2, 64)))
    for mode, kw in [("full", {}), ("chunk_causal", dict(chunk=2)), ("sliding", dict(wb=1, wf=1))]:
        o, _ = oracle.attention(q, k, ones, 1 / 8, mode=mode, F=16, **kw)
        assert np.max(np.abs(o - 1.0)) <= 1e-12


@pytest.mark.parametrize("mode,kw", [("full", {}), ("chunk_causal", dict(chunk=2)),
                                     ("chunk_causal", dict(chunk=3)),
                                     ("sliding", dict(wb=2, wf=0)), ("sliding", dict(wb=1, wf=2))])
def test_mask_closed_form_uniform_weights(mode, kw):
    # q = 0 makes every visible key weigh the same; V = one-hot of the key's
    # frame gives o[i, f] = 1 / (#visible frames) for each visible frame f
    # (every frame has F tokens).  lse = ln(#visible keys).
    T, F, d = 7, 5, 16
    L = T * F
    q = bf16(np.zeros((1, L, 1, d)))
    k = si.normal_bf16(3, (1, L, 1, d))
    onehot = np.zeros((1, L, 1, d))
    for n in range(L):
        onehot[0, n, 0, n // F] = 1.0
    v = bf16(onehot)
    o, lse = oracle.attention(q, k, v, 0.125, mode=mode, F=F, **kw)
    for i in range(L):
        f = i // F
        if mode == "full":
            vis = range(T)
        elif mode == "chunk_causal":
            c = kw["chunk"]
            vis = range(0, min(T, (f // c + 1) * c))
        else:
            vis = range(max(0, f - kw["wb"]), min(T - 1, f + kw["wf"]) + 1)
        expect = np.zeros(d)
        expect[list(vis)] = 1.0 / len(vis)
        assert np.max(np.abs(o[0, i, 0] - expect)) < 1e-14
        assert abs(lse[0, 0, i] - math.log(len(vis) * F)) < 1e-12


def test_mode_identities():
    # SLIDING with a window covering the sequence is FULL; CHUNK_CAUSAL with
    # one chunk is FULL; SLIDING(wb >= T, wf = 0) is CHUNK_CAUSAL(chunk = 1).
    q, k, v = si.qkv("tiny")
    F, T = 16, 3
    full, _ = oracle.attention(q, k, v, 1 / 8)
    sl, _ = oracle.attention(q, k, v, 1 / 8, mode="sliding", F=F, wb=T, wf=T)
    ch, _ = oracle.attention(q, k, v, 1 / 8, mode="chunk_causal", F=F, chunk=T)
    assert np.array_equal(full, sl) and np.array_equal(full, ch)
    sl0, _ = oracle.attention(q, k, v, 1 / 8, mode="sliding", F=F, wb=T, wf=0)
    ch1, _ = oracle.attention(q, k, v, 1 / 8, mode="chunk_causal", F=F, chunk=1)
    assert np.array_equal(sl0, ch1)


def test_rope_attention_shift_invariance():
    # Shifting every frame index of queries and keys by the same amount leaves
    # full attention unchanged (q.k depends only on relative offsets).
    q, k, v = si.qkv("tiny")
    rope = dict(Hg=4, Wg=4, pairs=TINY["pairs"], theta=1e4)
    a, la = oracle.attention(q, k, v, 1 / 8, rope=rope)
    b, lb = oracle.attention(q, k, v, 1 / 8, rope=rope, q_frame_offset=5, k_frame_offset=5)
    assert np.max(np.abs(a - b)) < 1e-12 and np.max(np.abs(la - lb)) < 1e-12
    c, _ = oracle.attention(q, k, v, 1 / 8, rope=rope, q_frame_offset=5, k_frame_offset=4)
    assert np.max(np.abs(a - c)) > 1e-3          # a relative shift does change it


def test_gqa_equals_repeated_heads():
    q, k, v = si.qkv("tiny")
    kk, vv = k[:, :, :1], v[:, :, :1]
    a, _ = oracle.attention(q, kk, vv, 1 / 8)
    b, _ = oracle.attention(q, np.repeat(kk, 2, axis=2), np.repeat(vv, 2, axis=2), 1 / 8)
    assert np.array_equal(a, b)


def test_row_subset_matches_full():
    q, k, v = si.qkv("tiny")
    o, lse = oracle.attention(q, k, v, 1 / 8, mode="sliding", F=16, wb=1)
    rows = si.sample_rows(5, 20, 1, 2, 48, forced=[0, 47, 15, 16])
    os_, ls = oracle.attention(q, k, v, 1 / 8, mode="sliding", F=16, wb=1, rows=rows)
    for r, (b, h, i) in enumerate(rows):
        assert np.array_equal(os_[r], o[b, i, h]) and ls[r] == lse[b, h, i]


# ----------------------------------------------------------------- streaming
def test_stream_equals_one_shot_sliding():
    # Frame-by-frame processing over a window of 4 past frames equals a
    # single SLIDING(wb=4, wf=0) pass over the whole sequence (FlashDecoder:
    # causality by processing order instead of a mask).
    T, Hg, Wg, H, d = 7, 3, 4, 2, 64
    F = Hg * Wg
    L = T * F
    q = si.normal_bf16(11, (1, L, H, d))
    k = si.normal_bf16(12, (1, L, H, d))
    v = si.normal_bf16(13, (1, L, H, d))
    rope = dict(Hg=Hg, Wg=Wg, pairs=(12, 10, 10), theta=1e4)
    os_, ls = oracle.stream(q, k, v, F, 1 / 8, wb=4, rope=rope)
    oa, la = oracle.attention(q, k, v, 1 / 8, mode="sliding", F=F, wb=4, wf=0, rope=rope)
    assert np.array_equal(os_, oa) and np.array_equal(ls, la)


def test_ring_model():
    n, cap = 7, 4
    kf = np.arange(n * 6, dtype=np.uint16).reshape(n, 1, 3, 1, 2)
    kr, vr, ids = oracle.ring_model(kf, kf + 1, cap)
    assert list(ids) == [4, 5, 6, 3]
    assert np.array_equal(kr[1], kf[5]) and np.array_equal(vr[3], kf[3] + 1)


# -------------------------------------------------------------------- hybrid
def _hyb_inputs(L=40, H=2, d=16, seed=21):
    return (si.normal_bf16(seed, (1, L, H, d)), si.normal_bf16(seed + 1, (1, L, H, d)),
            si.normal_bf16(seed + 2, (1, L, H, d)))


def _all_rows(B, H, L):
    return np.array([(b, h, i) for b in range(B) for h in range(H) for i in range(L)], np.int32)


def test_hybrid_recurrent_equals_parallel():
    q, k, v = _hyb_inputs()
    ct, scale = 12, 0.25
    o_rec, _, _ = oracle.hybrid_recurrent(q, k, v, ct, scale)
    rows = _all_rows(1, 2, 40)
    o_par = oracle.hybrid_parallel(q, k, v, ct, scale, rows)
    ref = np.stack([o_rec[0, i, h] for _, h, i in rows])
    assert np.max(np.abs(o_par - ref) / (np.abs(ref) + 1e-30)) < 1e-10


def test_hybrid_single_chunk_is_softmax():
    q, k, v = _hyb_inputs()
    o, _, _ = oracle.hybrid_recurrent(q, k, v, 40, 0.25)
    ref, _ = oracle.attention(q, k, v, 0.25)
    assert np.max(np.abs(o - ref)) < 1e-12


def test_hybrid_chunk0_rows_are_local_softmax():
    q, k, v = _hyb_inputs()
    o, _, _ = oracle.hybrid_recurrent(q, k, v, 12, 0.25)
    ref, _ = oracle.attention(q, k, v, 0.25, mode="sliding", F=12, wb=0, wf=0)
    assert np.max(np.abs(o[:, :12] - ref[:, :12])) < 1e-12


@pytest.mark.parametrize("x,phix", [(1.0, 2.0), (-1.0, 0.36787944117144233), (0.0, 1.0)])
def test_hybrid_closed_form_constant_keys(x, phix):
    # q = 0: softmax weights are exp(0) = 1 and phi(q) = 1 (elu(0)+1), so an
    # earlier key with every entry x weighs phi(q).phi(k) = d * phi(x):
    # o_i = (sum_{own} v + d phi(x) sum_{earlier} v) / (|own| + d phi(x) |earlier|)
    L, H, d, ct = 30, 1, 8, 7
    q = bf16(np.zeros((1, L, H, d)))
    k = bf16(np.full((1, L, H, d), x))
    v = si.normal_bf16(5, (1, L, H, d))
    V = si.bf16_bits_to_f64(v)[0, :, 0]
    o, S, z = oracle.hybrid_recurrent(q, k, v, ct, 0.5)
    for i in range(L):
        c0 = (i // ct) * ct
        c1 = min(L, c0 + ct)
        w = d * phix
        num = V[c0:c1].sum(0) + w * V[:c0].sum(0)
        den = (c1 - c0) + w * c0
        assert np.max(np.abs(o[0, i, 0] - num / den)) < 1e-13
    assert np.allclose(z[0, 0], np.full(d, L * phix), rtol=1e-14)
    assert np.allclose(S[0, 0], phix * np.tile(V.sum(0), (d, 1)), rtol=1e-12, atol=1e-12)


def test_hybrid_state_resume():
    # Running chunks [0, c) and then resuming from the saved (S, z) equals one
    # run over all chunks (the RNN view of the model).
    q, k, v = _hyb_inputs(L=48)
    ct = 12
    o_all, S_all, z_all = oracle.hybrid_recurrent(q, k, v, ct, 0.25)
    o1, S1, z1 = oracle.hybrid_recurrent(q[:, :24], k[:, :24], v[:, :24], ct, 0.25)
    o2, S2, z2 = oracle.hybrid_recurrent(q[:, 24:], k[:, 24:], v[:, 24:], ct, 0.25, S=S1, z=z1)
    assert np.max(np.abs(np.concatenate([o1, o2], axis=1) - o_all)) < 1e-12
    assert np.max(np.abs(S2 - S_all)) < 1e-9 and np.max(np.abs(z2 - z_all)) < 1e-9
    # the parallel form with the same incoming state agrees too
    rows = _all_rows(1, 2, 24)
    op = oracle.hybrid_parallel(q[:, 24:], k[:, 24:], v[:, 24:], ct, 0.25, rows, S0=S1, z0=z1)
    ref = np.stack([o2[0, i, h] for _, h, i in rows])
    assert np.max(np.abs(op - ref) / (np.abs(ref) + 1e-30)) < 1e-10


# ------------------------------------------- window-relative RoPE positions
@pytest.mark.parametrize("sub", [1, 2])
def test_stream_window_relative_positions(sub):
    # FlashDecoder "Long Video Decoding" (Sec. 4.3): positions relative to the
    # current window.  (a) By RoPE's relative property the attention equals
    # the absolute-position one (to rounding); (b) a query frame's rows equal
    # plain attention over its window's tokens with the query at latent frame
    # sub * (f - f0) and the keys from latent frame 0, evaluated by
    # oracle_attention (a separate code path); (c) frames before the window
    # fills (f < wb) are unchanged bit for bit.  sub = latent frames per
    # stream frame (2: a temporal-refinement step of r_t = 2 frames).
    T, Hg, Wg, H, d, wb = 7, 3, 4, 2, 64, 2
    F = sub * Hg * Wg
    L = T * F
    q = si.normal_bf16(111, (1, L, H, d))
    k = si.normal_bf16(112, (1, L, H, d))
    v = si.normal_bf16(113, (1, L, H, d))
    rope = dict(Hg=Hg, Wg=Wg, pairs=(12, 10, 10), theta=1e4)
    o_abs, l_abs = oracle.stream(q, k, v, F, 1 / 8, wb, rope=rope)
    o_rel, l_rel = oracle.stream(q, k, v, F, 1 / 8, wb, rope=rope, window_relative=True)
    assert np.max(np.abs(o_rel - o_abs)) < 1e-12 and np.max(np.abs(l_rel - l_abs)) < 1e-12
    assert np.array_equal(o_rel[:, :wb * F], o_abs[:, :wb * F])
    for f in range(T):
        f0 = max(0, f - wb)
        qf = q[:, f * F:(f + 1) * F]
        kw, vw = k[:, f0 * F:(f + 1) * F], v[:, f0 * F:(f + 1) * F]
        ow, lw = oracle.attention(qf, kw, vw, 1 / 8, rope=rope, q_frame_offset=sub * (f - f0), k_frame_offset=0)
        assert np.array_equal(ow, o_rel[:, f * F:(f + 1) * F]), "frame %d" % f


# ------------------------------------------------ hybrid, general form
POLY = np.array([[[0.7, 0.3, 0.2, 0.05]], [[1.0, 0.5, 0.25, 1.0 / 24.0]]])   # [q/k][H=1][a0..a3]


def test_hybrid2_elu_no_overlap_reproduces_the_hybrid():
    q, k, v = _hyb_inputs()
    S0 = si.normal_f64(31, 2 * 16 * 16).reshape(1, 2, 16, 16)
    z0 = np.abs(si.normal_f64(32, 2 * 16)).reshape(1, 2, 16) + 1.0
    o1, S1, z1 = oracle.hybrid_recurrent(q, k, v, 12, 0.25, S=S0, z=z0)
    o2, S2, z2 = oracle.hybrid2_recurrent(q, k, v, 12, 0.25, S=S0, z=z0)
    assert np.max(np.abs(o1 - o2)) < 1e-12
    assert np.max(np.abs(S1 - S2)) < 1e-10 and np.max(np.abs(z1 - z2)) < 1e-10
    rows = _all_rows(1, 2, 40)
    p1 = oracle.hybrid_parallel(q, k, v, 12, 0.25, rows, S0=S0, z0=z0)
    p2 = oracle.hybrid2_parallel(q, k, v, 12, 0.25, rows, S0=S0, z0=z0)
    assert np.max(np.abs(p1 - p2)) < 1e-12


@pytest.mark.parametrize("fmap,overlap", [("elu", 5), ("poly", 0), ("poly", 7), ("poly", 30)])
def test_hybrid2_recurrent_equals_parallel(fmap, overlap):
    q, k, v = _hyb_inputs()
    coef = np.concatenate([POLY, POLY * 0.9], axis=1)        # H = 2
    S0 = np.abs(si.normal_f64(33, 2 * 16 * 16)).reshape(1, 2, 16, 16)
    z0 = np.abs(si.normal_f64(34, 2 * 16)).reshape(1, 2, 16) + 1.0
    o_rec, _, _ = oracle.hybrid2_recurrent(q, k, v, 12, 0.25, overlap=overlap, fmap=fmap, coef=coef, S=S0, z=z0)
    rows = _all_rows(1, 2, 40)
    o_par = oracle.hybrid2_parallel(q, k, v, 12, 0.25, rows, overlap=overlap, fmap=fmap, coef=coef, S0=S0, z0=z0)
    ref = np.stack([o_rec[0, i, h] for _, h, i in rows])
    assert np.max(np.abs(o_par - ref) / (np.abs(ref) + 1e-30)) < 1e-10


# phi_k(x) = 1 + x/2 + x^2/4 + x^3/24, by hand: phi_k(2) = 1 + 1 + 1 + 1/3,
# phi_k(-1) = 1 - 1/2 + 1/4 - 1/24, phi_k(0) = 1; phi_q(0) = a0 = 0.7.
@pytest.mark.parametrize("x,phix", [(2.0, 10.0 / 3.0), (-1.0, 17.0 / 24.0), (0.0, 1.0)])
@pytest.mark.parametrize("overlap", [0, 3, 7, 9])
def test_hybrid2_closed_form_polynomial_and_overlap(x, phix, overlap):
    # q = 0: softmax weights are exp(0) = 1; phi_q(0) = 0.7 on every channel,
    # so a key with every entry x weighs 0.7 * d * phi_k(x) in the linear
    # part.  With the softmax window [w0, w1) = [max(0, c ct - ov), end of
    # chunk c):  o_i = (sum_{window} v + lam sum_{j < w0} v) / (|window| + lam w0).
    L, H, d, ct = 30, 1, 8, 7
    q = bf16(np.zeros((1, L, H, d)))
    k = bf16(np.full((1, L, H, d), x))
    v = si.normal_bf16(6, (1, L, H, d))
    V = si.bf16_bits_to_f64(v)[0, :, 0]
    o, S, z = oracle.hybrid2_recurrent(q, k, v, ct, 0.5, overlap=overlap, fmap="poly", coef=POLY)
    lam = 0.7 * d * phix
    for i in range(L):
        c = i // ct
        w0, w1 = max(0, c * ct - overlap), min(L, (c + 1) * ct)
        num = V[w0:w1].sum(0) + lam * V[:w0].sum(0)
        den = (w1 - w0) + lam * w0
        assert np.max(np.abs(o[0, i, 0] - num / den)) < 1e-13, (i, w0, w1)
    assert np.allclose(z[0, 0], np.full(d, L * phix), rtol=1e-13)
    assert np.allclose(S[0, 0], phix * np.tile(V.sum(0), (d, 1)), rtol=1e-12, atol=1e-12)


def test_hybrid2_limits():
    q, k, v = _hyb_inputs()
    coef = np.concatenate([POLY, POLY], axis=1)
    # one chunk covering everything: pure softmax whatever the feature map
    o, _, _ = oracle.hybrid2_recurrent(q, k, v, 40, 0.25, overlap=3, fmap="poly", coef=coef)
    ref, _ = oracle.attention(q, k, v, 0.25)
    assert np.max(np.abs(o - ref)) < 1e-12
    # an overlap reaching back to token 0 leaves no linear part: every query
    # sees all keys up to the end of its chunk (chunk-causal softmax)
    o, _, _ = oracle.hybrid2_recurrent(q, k, v, 12, 0.25, overlap=40, fmap="poly", coef=coef)
    ref, _ = oracle.attention(q, k, v, 0.25, mode="chunk_causal", F=12, chunk=1)
    assert np.max(np.abs(o - ref)) < 1e-12
    # chunk-0 rows are the local softmax of chunk 0 for any overlap
    o, _, _ = oracle.hybrid2_recurrent(q, k, v, 12, 0.25, overlap=5, fmap="poly", coef=coef)
    ref, _ = oracle.attention(q, k, v, 0.25, mode="sliding", F=12, wb=0, wf=0)
    assert np.max(np.abs(o[:, :12] - ref[:, :12])) < 1e-12


def test_hybrid2_state_resume_polynomial():
    # Without overlap, two calls carrying (S, z) equal one call (RNN view).
    q, k, v = _hyb_inputs()
    coef = np.concatenate([POLY, POLY], axis=1)
    o, S, z = oracle.hybrid2_recurrent(q, k, v, 8, 0.25, fmap="poly", coef=coef)
    o1, S1, z1 = oracle.hybrid2_recurrent(q[:, :16], k[:, :16], v[:, :16], 8, 0.25, fmap="poly", coef=coef)
    o2, S2, z2 = oracle.hybrid2_recurrent(q[:, 16:], k[:, 16:], v[:, 16:], 8, 0.25, fmap="poly", coef=coef,
                                          S=S1, z=z1)
    assert np.max(np.abs(np.concatenate([o1, o2], axis=1) - o)) < 1e-12
    assert np.max(np.abs(S2 - S)) < 1e-10 and np.max(np.abs(z2 - z)) < 1e-10


# --------------------------------------------------------------------- merge
def test_merge_of_key_shards_is_attention_over_all_keys():
    # Ring attention's join (ReGenVC Sec. 3.5): partial attentions over
    # disjoint key shards, combined through their log-sum-exp, equal one
    # attention over all keys.
    L, H, d, R = 48, 2, 16, 3
    q = si.normal_bf16(121, (1, L, H, d))
    k = si.normal_bf16(122, (1, L, H, d))
    v = si.normal_bf16(123, (1, L, H, d))
    ref, lref = oracle.attention(q, k, v, 0.25)
    cuts = [0, 10, 31, 48]
    parts = [oracle.attention(q, k[:, a:b], v[:, a:b], 0.25) for a, b in zip(cuts, cuts[1:])]
    o_p = np.stack([p[0].transpose(0, 2, 1, 3).reshape(-1, d) for p in parts])   # [R, (b h i), d]
    l_p = np.stack([p[1].reshape(-1) for p in parts])                              # [R, (b h i)]
    o, lse = oracle.merge(o_p, l_p)
    assert np.max(np.abs(o - ref.transpose(0, 2, 1, 3).reshape(-1, d))) < 1e-12
    assert np.max(np.abs(lse - lref.reshape(-1))) < 1e-12


def test_merge_closed_form_and_empty_part():
    # weights e^0 : e^{ln 3} = 1 : 3; a part with lse = -inf has weight 0.
    o_p = np.array([[[1.0, 0.0]], [[0.0, 1.0]], [[5.0, 5.0]]])
    l_p = np.array([[0.0], [math.log(3.0)], [-np.inf]])
    o, lse = oracle.merge(o_p, l_p)
    assert np.allclose(o, [[0.25, 0.75]], rtol=0, atol=1e-15)
    assert abs(lse[0] - math.log(4.0)) < 1e-15
    o, lse = oracle.merge(o_p[2:], l_p[2:])
    assert np.array_equal(o, [[0.0, 0.0]]) and lse[0] == -np.inf
