"""GPU parity of the individual kernels against plain definitions and the
fp64 oracle, on small shapes that still span several tiles and a ragged
tail.  All calls go through the C ABI (ctypes binding)."""
import numpy as np
import pytest

import oracle
import seeded_inputs as si
from helpers import assert_parity, bits_of, check_guards, errors, from_dev, gather_rows, guarded, to_dev

pytestmark = pytest.mark.gpu
LSE_TOL = 1e-2


@pytest.fixture(scope="module")
def va():
    import video_diffusion_transformer_02_b200 as va
    return va


# ------------------------------------------------------- tensor-core layouts
@pytest.mark.parametrize("variant", [0, 1, 2, 3])
def test_umma_layouts(va, variant):
    import torch
    a = si.normal_bf16(100 + variant, (128, 128))
    b = si.normal_bf16(200 + variant, (128, 128))
    out = torch.full((128, 128), float("nan"), dtype=torch.float32, device="cuda")
    va.vattn_selftest_umma(variant, to_dev(a), to_dev(b), out)
    va.vattn_check()
    A, Bm = si.bf16_bits_to_f64(a), si.bf16_bits_to_f64(b)
    ref = {0: A @ Bm.T, 1: A @ Bm, 2: A @ Bm, 3: A.T @ Bm}[variant]
    got = out.cpu().numpy().astype(np.float64)
    assert np.max(np.abs(got - ref)) < 1e-3 * np.max(np.abs(ref)), "layout variant %d" % variant


# ------------------------------------------------------------------- RoPE
def _rope(va, Hg, Wg, pairs, max_pos):
    return va.Rope(Hg=Hg, Wg=Wg, pairs=pairs, max_pos=max_pos, theta=10000.0)


@pytest.mark.parametrize("shape,grid,pairs,off", [
    ((1, 48, 2, 64), (4, 4), (12, 10, 10), 0),
    ((2, 300, 3, 128), (6, 10), (22, 21, 21), 3),
])
def test_rope_qk(va, shape, grid, pairs, off):
    import torch
    B, L, H, d = shape
    q = si.normal_bf16(1, shape)
    k = si.normal_bf16(2, (B, L, 1, d))
    r = _rope(va, grid[0], grid[1], pairs, 16)
    tab = va.rope_table(r, d)
    qo = torch.empty(shape, dtype=torch.bfloat16, device="cuda")
    ko = torch.empty((B, L, 1, d), dtype=torch.bfloat16, device="cuda")
    va.vattn_rope_qk(to_dev(q), to_dev(k), qo, ko, r, tab, frame_offset=off)
    rq = oracle.rope(q, grid[0], grid[1], pairs, 1e4, t_offset=off)
    rk = oracle.rope(k, grid[0], grid[1], pairs, 1e4, t_offset=off)
    for got, ref in ((from_dev(qo), rq), (from_dev(ko), rk)):
        # fp32 rotation rounded once to bf16: within one bf16 ulp of the exact value
        assert np.all(np.abs(got - ref) <= np.abs(ref) * 2.0 ** -8 + 1e-6)


# -------------------------------------------------------------- attention
CASES = [
    # (B, T, Hg, Wg, H, Hkv, d, mode, kwargs, rope)
    (1, 3, 4, 4, 2, 2, 64, "full", {}, True),                       # the tiny config
    (1, 5, 6, 10, 2, 2, 128, "full", {}, False),                    # 300 tokens: ragged tail
    (2, 5, 6, 10, 4, 2, 64, "full", {}, True),                      # GQA, batch 2
    (1, 7, 5, 9, 2, 2, 128, "chunk_causal", dict(chunk=2), True),   # chunks not tile aligned
    (1, 7, 5, 9, 2, 2, 64, "chunk_causal", dict(chunk=3), False),
    (1, 9, 4, 10, 2, 2, 128, "sliding", dict(wb=2, wf=0), True),
    (1, 9, 4, 10, 2, 2, 64, "sliding", dict(wb=1, wf=1), False),
    (1, 6, 8, 16, 2, 1, 128, "sliding", dict(wb=4, wf=0), True),    # F = 128: tile aligned frames
]


def _attention_case(va, B, T, Hg, Wg, H, Hkv, d, mode, kw, use_rope, seed=0, qoff=0, koff=0,
                    fuse_k=False):
    import torch
    F = Hg * Wg
    L = T * F
    q = si.normal_bf16(10 + seed, (B, L, H, d))
    k = si.normal_bf16(11 + seed, (B, L, Hkv, d))
    v = si.normal_bf16(12 + seed, (B, L, Hkv, d))
    scale = d ** -0.5
    og = guarded((B, L, H, d), torch.bfloat16, float("nan"))
    lg = guarded((B, H, L), torch.float32, float("nan"))
    o, lse = og.t, lg.t
    rope = tab = None
    orope = None
    pairs = (12, 10, 10) if d == 64 else (22, 21, 21)
    if use_rope:
        rope = _rope(va, Hg, Wg, pairs, max(T + qoff + koff, Hg, Wg) + 1)
        tab = va.rope_table(rope, d)
        orope = dict(Hg=Hg, Wg=Wg, pairs=pairs, theta=1e4)
    va.vattn_attention(to_dev(q), to_dev(k), to_dev(v), o, lse, scale=scale, mode=mode,
                       tokens_per_frame=F, chunk_frames=kw.get("chunk", 1),
                       window_back=kw.get("wb", 0), window_fwd=kw.get("wf", 0),
                       q_frame_offset=qoff, k_frame_offset=koff, rope=rope, table=tab,
                       fuse_k_rope=fuse_k)
    va.vattn_check()
    check_guards(og, lg, what="attention o / lse")
    ro, rl = oracle.attention(q, k, v, scale, mode=mode, F=F, chunk=kw.get("chunk", 1),
                              wb=kw.get("wb", 0), wf=kw.get("wf", 0), q_frame_offset=qoff,
                              k_frame_offset=koff, rope=orope)
    return from_dev(o), lse.cpu().numpy().astype(np.float64), ro, rl


@pytest.mark.parametrize("case", CASES, ids=lambda c: "%s-d%d-T%dx%dx%d-H%d/%d%s" % (
    c[7], c[6], c[1], c[2], c[3], c[4], c[5], "-rope" if c[9] else ""))
@pytest.mark.parametrize("fuse_k", [False, True], ids=["k-prerotated", "k-fused"])
def test_attention_parity(va, case, fuse_k):
    B, T, Hg, Wg, H, Hkv, d, mode, kw, use_rope = case
    if fuse_k and not use_rope:
        pytest.skip("no rope")
    got, glse, ref, rlse = _attention_case(va, B, T, Hg, Wg, H, Hkv, d, mode, kw, use_rope, fuse_k=fuse_k)
    assert_parity(got, ref, "attention %s" % (case,))
    # lse: the kernel rounds rotated q, k to bf16 before the products, which
    # moves each score by ~2e-3 rms (2^-9 relative per operand over d terms);
    # lse is a convex combination of those score errors.
    assert np.max(np.abs(glse - rlse)) < LSE_TOL, "lse"


@pytest.mark.parametrize("fuse_k", [False, True])
def test_attention_frame_offsets(va, fuse_k):
    # Offsets move the frames of queries and keys (masks and RoPE t).
    got, _, ref, _ = _attention_case(va, 1, 6, 5, 8, 2, 2, 128, "sliding", dict(wb=1, wf=0), True,
                                     qoff=2, koff=1, fuse_k=fuse_k)
    assert_parity(got, ref, "offsets")


def test_attention_single_token_and_tiny_lengths(va):
    import torch
    for L in (1, 7, 129):
        q = si.normal_bf16(70, (1, L, 1, 64))
        k = si.normal_bf16(71, (1, L, 1, 64))
        v = si.normal_bf16(72, (1, L, 1, 64))
        o = torch.empty((1, L, 1, 64), dtype=torch.bfloat16, device="cuda")
        va.vattn_attention(to_dev(q), to_dev(k), to_dev(v), o, scale=0.125)
        va.vattn_check()
        ref, _ = oracle.attention(q, k, v, 0.125)
        assert_parity(from_dev(o), ref, "L=%d" % L)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("mode,kw", [("full", {}), ("sliding", dict(wb=1, wf=0))])
def test_attention_large_logit_jumps(va, d, mode, kw):
    # Every block of 64 keys is scaled by its own seeded factor 2^(0..9), so
    # a row's max jumps by up to ~2000 log2 units from one sub-tile to the
    # next, in both directions: the reference max must move (O rescaled)
    # and exponentials taken against a stale reference must be redone.
    import torch
    B, H, F, T = 1, 2, 100, 15
    L = F * T
    q = si.normal_bf16(80 + d, (B, L, H, d))
    k = si.normal_bf16(81 + d, (B, L, H, d))
    v = si.normal_bf16(82 + d, (B, L, H, d))
    f = 2.0 ** np.floor(10.0 * si.uniform01(83 + d, (L + 63) // 64))
    kf = si.bf16_bits_to_f64(k) * np.repeat(f, 64)[:L][None, :, None, None]
    k = si.f64_to_bf16_bits(kf)
    og = guarded((B, L, H, d), torch.bfloat16, float("nan"))
    lg = guarded((B, H, L), torch.float32, float("nan"))
    va.vattn_attention(to_dev(q), to_dev(k), to_dev(v), og.t, lg.t, scale=d ** -0.5, mode=mode,
                       tokens_per_frame=F, window_back=kw.get("wb", 0), window_fwd=kw.get("wf", 0))
    va.vattn_check()
    check_guards(og, lg, what="o / lse")
    ro, rl = oracle.attention(q, k, v, d ** -0.5, mode=mode, F=F, wb=kw.get("wb", 0), wf=kw.get("wf", 0))
    assert_parity(from_dev(og.t), ro, "large logit jumps d=%d %s" % (d, mode))
    # |lse| reaches ~1e3 here; fp32 holds it to ~1e-4 absolute
    assert np.max(np.abs(lg.t.cpu().numpy().astype(np.float64) - rl)) < LSE_TOL, "lse"


def test_bounded_wait_reports_timeout_and_context_survives(va):
    # A barrier nothing arrives on: the kernel's bounded wait gives up after
    # 50 ms, the status word reports a timeout, and the next call still works.
    import torch
    va.vattn_check()                                   # start from a clear status word
    va.vattn_selftest_wait_timeout(50000)
    with pytest.raises(va.VattnError) as e:
        va.vattn_check()
    assert e.value.status == va.ERR_TIMEOUT
    va.vattn_check()                                   # cleared
    q = si.normal_bf16(75, (1, 200, 1, 64))
    k = si.normal_bf16(76, (1, 200, 1, 64))
    v = si.normal_bf16(77, (1, 200, 1, 64))
    o = torch.empty((1, 200, 1, 64), dtype=torch.bfloat16, device="cuda")
    va.vattn_attention(to_dev(q), to_dev(k), to_dev(v), o, scale=0.125)
    va.vattn_check()
    ref, _ = oracle.attention(q, k, v, 0.125)
    assert_parity(from_dev(o), ref, "after timeout")


def test_bounded_wait_in_the_attention_kernel(va):
    # The real two-tile kernel with one softmax arrival withheld and a 5 ms
    # wait bound: tile A's MMA issuer gives up, the CTA tears down (drains its
    # copies and MMAs, frees TMEM) and returns; the status word reports a
    # timeout, and the next normal call on the same context is correct.
    import torch
    va.vattn_check()
    for d in (64, 128):
        L, H = 512, 2
        q = si.normal_bf16(80, (1, L, H, d))
        k = si.normal_bf16(81, (1, L, H, d))
        v = si.normal_bf16(82, (1, L, H, d))
        qd, kd, vd = to_dev(q), to_dev(k), to_dev(v)
        o = torch.zeros((1, L, H, d), dtype=torch.bfloat16, device="cuda")
        va.vattn_selftest_attention_timeout(qd, kd, vd, o, 5000)
        with pytest.raises(va.VattnError) as e:
            va.vattn_check()
        assert e.value.status == va.ERR_TIMEOUT
        va.vattn_check()                               # cleared
        og = guarded((1, L, H, d), torch.bfloat16, float("nan"))
        va.vattn_attention(qd, kd, vd, og.t, scale=d ** -0.5)
        va.vattn_check()
        check_guards(og, what="attention after timeout")
        ref, _ = oracle.attention(q, k, v, d ** -0.5)
        assert_parity(from_dev(og.t), ref, "attention after an aborted launch (d=%d)" % d)


def test_exp2_functions_against_fp64(va):
    # The softmax's exponentials over the whole range they see (arguments
    # are <= 8 after the running-max subtraction, far below it for masked
    # or stale entries): the FMA-pipe polynomial within its stated relative
    # bound for x >= -125 and a value in [0, 2^-124] below, the packed form
    # equal to the scalar one bit for bit, MUFU ex2 within 2^-20 relative.  (The Remez fit's bound is 7.48e-5 in exact arithmetic; the
    # fp32 evaluation of the polynomial adds at most a few 1e-7.)
    import torch
    x = np.concatenate([np.linspace(-130.0, 64.0, 400001), np.arange(-130, 64, dtype=np.float64),
                        np.arange(-130, 64, dtype=np.float64) + 0.5,
                        si.normal_f64(0xE2, 100000) * 8.0]).astype(np.float32)
    x = x[: len(x) // 2 * 2]
    xd = torch.from_numpy(x).cuda()
    ys = {}
    for variant in (0, 1, 2):
        y = torch.full_like(xd, float("nan"))
        va.vattn_selftest_ex2(variant, xd, y)
        va.vattn_check()
        ys[variant] = y.cpu().numpy()
    exact = np.exp2(x.astype(np.float64))
    inr = x >= -125.0
    rel = np.abs(ys[0][inr] - exact[inr]) / exact[inr]
    assert rel.max() <= 7.6e-5, "polynomial exp2: max relative error %.3e" % rel.max()
    low = ys[0][~inr].astype(np.float64)
    assert np.all((low >= 0.0) & (low <= 2.0 ** -124)), "arguments below -125 give a value in [0, 2^-124]"
    assert np.array_equal(ys[0].view(np.uint32), ys[1].view(np.uint32)), "packed and scalar forms differ"
    relm = np.abs(ys[2][inr] - exact[inr]) / exact[inr]
    assert relm.max() <= 2.0 ** -20, "ex2.approx: max relative error %.3e" % relm.max()
