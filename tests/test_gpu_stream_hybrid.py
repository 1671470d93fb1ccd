"""GPU parity of the streaming step (rolling KV ring) and of hybrid chunk
attention against the fp64 oracle."""
import numpy as np
import pytest

import oracle
import seeded_inputs as si
from helpers import assert_parity, bits_of, from_dev, gather_rows, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def va():
    import video_diffusion_transformer_02_b200 as va
    return va


def _run_stream(va, q, k, v, F, H, Hkv, d, cap, wb, rope, tab, check_ring=None):
    """Frame-by-frame decode through the ring; returns o [B, L, H, d]."""
    import torch
    B, L = q.shape[0], q.shape[1]
    T = L // F
    kr = torch.zeros((cap, B, F, Hkv, d), dtype=torch.bfloat16, device="cuda")
    vr = torch.zeros_like(kr)
    ids = torch.zeros(cap, dtype=torch.int32, device="cuda")
    cache = va.KVCache(kr, vr, ids)
    qd, kd, vd = to_dev(q), to_dev(k), to_dev(v)
    o = torch.full((B, L, H, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    for f in range(T):
        sl = slice(f * F, (f + 1) * F)
        qf, kf, vf = qd[:, sl].contiguous(), kd[:, sl].contiguous(), vd[:, sl].contiguous()
        of = torch.empty((B, F, H, d), dtype=torch.bfloat16, device="cuda")
        cache.attend(qf, kf, vf, of, f, wb, scale=d ** -0.5, rope=rope, table=tab)
        cache.append(kf, vf, f)
        o[:, sl] = of
        if check_ring is not None:
            check_ring(f, kr, vr, ids, cache)
    va.vattn_check()
    cache.close()
    return o


def test_stream_small_with_ring_bit_exact(va):
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

    o = _run_stream(va, q, k, v, F, H, H, d, cap, wb, rope, tab, check_ring)
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
    S = torch.zeros((1, H, d, d), dtype=torch.float32, device="cuda")
    z = torch.zeros((1, H, d), dtype=torch.float32, device="cuda")
    o = torch.full((1, L, H, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    va.vattn_hybrid_chunk(to_dev(q), to_dev(k), to_dev(v), o, S, z, chunk, scale=d ** -0.5)
    va.vattn_check()
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
