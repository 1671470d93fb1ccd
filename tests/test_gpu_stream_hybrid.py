"""GPU parity of the streaming step (rolling KV ring) and of hybrid chunk
attention against the fp64 oracle."""
import numpy as np
import pytest

import oracle
import seeded_inputs as si
from helpers import assert_parity, bits_of, check_guards, from_dev, gather_rows, guarded, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def va():
    import video_diffusion_transformer_02_b200 as va
    return va


def _run_stream(va, q, k, v, F, H, Hkv, d, cap, wb, rope, tab, check_ring=None, rot_ring=False):
    """Frame-by-frame decode through the ring; returns o [B, L, H, d]."""
    import torch
    B, L = q.shape[0], q.shape[1]
    T = L // F
    g_k = guarded((cap, B, F, Hkv, d), torch.bfloat16)
    g_v = guarded((cap, B, F, Hkv, d), torch.bfloat16)
    g_ids = guarded((cap,), torch.int32, 0)
    kr, vr, ids = g_k.t, g_v.t, g_ids.t
    guards = [g_k, g_v, g_ids]
    cache = va.KVCache(kr, vr, ids)
    if rot_ring:
        g_rot = guarded((cap + 1, B, F, Hkv, d), torch.bfloat16)
        guards.append(g_rot)
        cache.enable_rope(g_rot.t, rope, tab)
    qd, kd, vd = to_dev(q), to_dev(k), to_dev(v)
    o = torch.full((B, L, H, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    g_o = guarded((B, F, H, d), torch.bfloat16, float("nan"))
    guards.append(g_o)
    for f in range(T):
        sl = slice(f * F, (f + 1) * F)
        qf, kf, vf = qd[:, sl].contiguous(), kd[:, sl].contiguous(), vd[:, sl].contiguous()
        of = g_o.t
        cache.attend(qf, kf, vf, of, f, wb, scale=d ** -0.5, rope=rope, table=tab)
        cache.append(kf, vf, f)
        o[:, sl] = of
        if check_ring is not None:
            check_ring(f, kr, vr, ids, cache)
        check_guards(*guards, what="stream frame %d" % f)
    va.vattn_check()
    cache.close()
    return o


@pytest.mark.parametrize("rot_ring", [False, True], ids=["k-fused", "k-rotated-ring"])
def test_stream_small_with_ring_bit_exact(va, rot_ring):
    T, Hg, Wg, H, d, cap, wb = 9, 5, 30, 2, 64, 4, 4     # F = 150: ragged frame tiles
    F = Hg * Wg
    L = T * F
    q = si.normal_bf16(31, (1, L, H, d))
    k = si.normal_bf16(32, (1, L, H, d))
    v = si.normal_bf16(33, (1, L, H, d))
    rope = va.Rope(Hg=Hg, Wg=Wg, pairs=(12, 10, 10), max_pos=64)
    tab = va.rope_table(rope, d)
    kf = k.reshape(1, T, F, H, d).transpose(1, 0, 2, 3, 4)
    vf = v.reshape(1, T, F, H, d).transpose(1, 0, 2, 3, 4)

    def check_ring(f, kr, vr, ids, cache):
        ek, ev, eids = oracle.ring_model(kf[:f + 1], vf[:f + 1], cap)
        assert np.array_equal(bits_of(kr), ek), "K ring differs after frame %d" % f
        assert np.array_equal(bits_of(vr), ev), "V ring differs after frame %d" % f
        assert list(ids.cpu().numpy()) == list(eids) == cache.host_frame_ids()

    o = _run_stream(va, q, k, v, F, H, H, d, cap, wb, rope, tab, check_ring, rot_ring=rot_ring)
    ref, _ = oracle.stream(q, k, v, F, d ** -0.5, wb, rope=dict(Hg=Hg, Wg=Wg, pairs=(12, 10, 10),
                                                                  theta=1e4))
    assert_parity(from_dev(o), ref, "stream")


def test_stream_equals_one_shot_sliding_on_gpu(va):
    import torch
    T, Hg, Wg, H, d = 7, 4, 40, 2, 64
    F = Hg * Wg
    L = T * F
    q = si.normal_bf16(41, (1, L, H, d))
    k = si.normal_bf16(42, (1, L, H, d))
    v = si.normal_bf16(43, (1, L, H, d))
    rope = va.Rope(Hg=Hg, Wg=Wg, pairs=(12, 10, 10), max_pos=64)
    tab = va.rope_table(rope, d)
    o_stream = _run_stream(va, q, k, v, F, H, H, d, 4, 4, rope, tab)
    o_once = torch.empty_like(o_stream)
    va.vattn_attention(to_dev(q), to_dev(k), to_dev(v), o_once, scale=d ** -0.5, mode="sliding",
                       tokens_per_frame=F, window_back=4, rope=rope, table=tab)
    va.vattn_check()
    a, b = from_dev(o_stream), from_dev(o_once)
    assert np.max(np.abs(a - b)) < 1e-2


@pytest.mark.parametrize("L,chunk", [(700, 300), (12090 // 3 + 7, 1170)])
def test_hybrid_parity_all_rows(va, L, chunk):
    import torch
    H, d = 2, 128
    q = si.normal_bf16(51, (1, L, H, d))
    k = si.normal_bf16(52, (1, L, H, d))
    v = si.normal_bf16(53, (1, L, H, d))
    gS, gz = guarded((1, H, d, d), torch.float32), guarded((1, H, d), torch.float32)
    go = guarded((1, L, H, d), torch.bfloat16, float("nan"))
    S, z, o = gS.t, gz.t, go.t
    va.vattn_hybrid_chunk(to_dev(q), to_dev(k), to_dev(v), o, S, z, chunk, scale=d ** -0.5)
    va.vattn_check()
    check_guards(gS, gz, go, what="hybrid o / S / z")
    ro, rS, rz = oracle.hybrid_recurrent(q, k, v, chunk, d ** -0.5)
    assert_parity(from_dev(o), ro, "hybrid o")
    assert_parity(S.cpu().numpy(), rS, "hybrid S", max_abs=np.inf)
    assert_parity(z.cpu().numpy(), rz, "hybrid z", max_abs=np.inf)


def test_hybrid_softmax_half_with_zero_state(va):
    # chunk-0 rows have no linear part: they are pure in-chunk softmax, which
    # the linear term would otherwise dominate (checked separately).
    import torch
    L, chunk, H, d = 900, 390, 2, 128
    q = si.normal_bf16(61, (1, L, H, d))
    k = si.normal_bf16(62, (1, L, H, d))
    v = si.normal_bf16(63, (1, L, H, d))
    S = torch.zeros((1, H, d, d), dtype=torch.float32, device="cuda")
    z = torch.zeros((1, H, d), dtype=torch.float32, device="cuda")
    o = torch.empty((1, L, H, d), dtype=torch.bfloat16, device="cuda")
    va.vattn_hybrid_chunk(to_dev(q), to_dev(k), to_dev(v), o, S, z, chunk)
    va.vattn_check()
    ref, _ = oracle.attention(q, k, v, d ** -0.5, mode="sliding", F=chunk)
    assert_parity(from_dev(o)[:, :chunk], ref[:, :chunk], "chunk-0 softmax rows")


def test_hybrid_state_resume(va):
    # Two calls carrying (S, z) equal one call over the whole sequence.
    import torch
    L, chunk, H, d = 1200, 300, 1, 128
    q = si.normal_bf16(71, (1, L, H, d))
    k = si.normal_bf16(72, (1, L, H, d))
    v = si.normal_bf16(73, (1, L, H, d))
    S = torch.zeros((1, H, d, d), dtype=torch.float32, device="cuda")
    z = torch.zeros((1, H, d), dtype=torch.float32, device="cuda")
    o = torch.empty((1, L, H, d), dtype=torch.bfloat16, device="cuda")
    qd, kd, vd = to_dev(q), to_dev(k), to_dev(v)
    half = 600
    o1 = torch.empty((1, half, H, d), dtype=torch.bfloat16, device="cuda")
    o2 = torch.empty((1, L - half, H, d), dtype=torch.bfloat16, device="cuda")
    va.vattn_hybrid_chunk(qd[:, :half].contiguous(), kd[:, :half].contiguous(), vd[:, :half].contiguous(),
                          o1, S, z, chunk)
    va.vattn_hybrid_chunk(qd[:, half:].contiguous(), kd[:, half:].contiguous(), vd[:, half:].contiguous(),
                          o2, S, z, chunk)
    va.vattn_check()
    ro, rS, rz = oracle.hybrid_recurrent(q, k, v, chunk, d ** -0.5)
    got = np.concatenate([from_dev(o1), from_dev(o2)], axis=1)
    assert_parity(got, ro, "resumed hybrid")
    assert_parity(S.cpu().numpy(), rS, "resumed S", max_abs=np.inf)


def test_rotated_ring_contents(va):
    # The rotated-key ring holds each frame's keys rotated at its absolute
    # frame: within one bf16 ulp of the exact rotation.
    import torch
    T, Hg, Wg, H, d, cap = 6, 4, 32, 2, 64, 4
    F = Hg * Wg
    k = si.normal_bf16(81, (1, T * F, H, d))
    v = si.normal_bf16(82, (1, T * F, H, d))
    rope = va.Rope(Hg=Hg, Wg=Wg, pairs=(12, 10, 10), max_pos=64)
    tab = va.rope_table(rope, d)
    kr = torch.zeros((cap, 1, F, H, d), dtype=torch.bfloat16, device="cuda")
    cache = va.KVCache(kr, torch.zeros_like(kr), torch.zeros(cap, dtype=torch.int32, device="cuda"))
    rot = torch.zeros((cap + 1, 1, F, H, d), dtype=torch.bfloat16, device="cuda")
    cache.enable_rope(rot, rope, tab)
    kd, vd = to_dev(k), to_dev(v)
    for f in range(T):
        cache.append(kd[:, f * F:(f + 1) * F].contiguous(), vd[:, f * F:(f + 1) * F].contiguous(), f)
    va.vattn_check()
    exact = oracle.rope(k, Hg, Wg, (12, 10, 10), 1e4)
    for f in range(T - cap - 1 + 1, T):
        got = from_dev(rot[f % (cap + 1)])[0]
        ref = exact[0, f * F:(f + 1) * F]
        assert np.all(np.abs(got - ref) <= np.abs(ref) * 2.0 ** -8 + 1e-6), "frame %d" % f
    cache.close()


def test_stream_checkpoint_resume(va):
    # Decode frames 0..k-1, copy the ring out, restore it into a fresh cache
    # and continue: outputs and ring contents equal an unsplit run.
    import torch
    T, Hg, Wg, H, d, cap, wb, split = 9, 5, 30, 2, 64, 4, 4, 5
    F = Hg * Wg
    q = si.normal_bf16(91, (1, T * F, H, d))
    k = si.normal_bf16(92, (1, T * F, H, d))
    v = si.normal_bf16(93, (1, T * F, H, d))
    rope = va.Rope(Hg=Hg, Wg=Wg, pairs=(12, 10, 10), max_pos=64)
    tab = va.rope_table(rope, d)
    qd, kd, vd = to_dev(q), to_dev(k), to_dev(v)

    def new_cache():
        kr = torch.zeros((cap, 1, F, H, d), dtype=torch.bfloat16, device="cuda")
        c = va.KVCache(kr, torch.zeros_like(kr), torch.zeros(cap, dtype=torch.int32, device="cuda"))
        c.enable_rope(torch.zeros((cap + 1, 1, F, H, d), dtype=torch.bfloat16, device="cuda"), rope, tab)
        return c

    def step(c, f):
        sl = slice(f * F, (f + 1) * F)
        of = torch.empty((1, F, H, d), dtype=torch.bfloat16, device="cuda")
        c.attend(qd[:, sl].contiguous(), kd[:, sl].contiguous(), vd[:, sl].contiguous(), of, f, wb,
                 rope=rope, table=tab)
        c.append(kd[:, sl].contiguous(), vd[:, sl].contiguous(), f)
        return of

    a = new_cache()
    full = [step(a, f) for f in range(T)]
    b = new_cache()
    first = [step(b, f) for f in range(split)]
    saved = (b.k_ring.clone(), b.v_ring.clone(), b.frame_ids.clone(), b.host_frame_ids())
    b.close()
    c = new_cache()
    c.k_ring.copy_(saved[0])
    c.v_ring.copy_(saved[1])
    c.frame_ids.copy_(saved[2])
    c.restore(saved[3])
    rest = [step(c, f) for f in range(split, T)]
    va.vattn_check()
    for f, (x, y) in enumerate(zip(full, first + rest)):
        assert torch.equal(x, y), "frame %d differs after resume" % f
    assert torch.equal(a.k_ring, c.k_ring) and torch.equal(a.v_ring, c.v_ring)
    assert a.host_frame_ids() == c.host_frame_ids()
    a.close()
    c.close()
