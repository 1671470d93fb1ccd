"""GPU parity of the fused streaming step (vattn_kvcache_step: attend and
append in one launch) against the fp64 oracle: ring contents bit for bit
after every frame, outputs within the parity bar, absolute and
window-relative RoPE positions, several latent frames per step (temporal
refinement), GQA, key splits merged in the kernel, and the FlashDecoder-XL
shapes at full size on sampled rows."""
import numpy as np
import pytest

import oracle
import seeded_inputs as si
from helpers import assert_parity, bits_of, check_guards, from_dev, gather_rows, guarded, to_dev

pytestmark = pytest.mark.gpu
N_ROWS = 4096


@pytest.fixture(scope="module")
def va():
    import video_diffusion_transformer_02_b200 as va
    return va


def _decode(va, q, k, v, F, H, Hkv, d, cap, wb, rope, tab, window_relative=False, check=None):
    """Frame-by-frame steps through a guarded ring; returns o [B, L, H, d]."""
    import torch
    B, L = q.shape[0], q.shape[1]
    T = L // F
    gk, gv = guarded((cap, B, F, Hkv, d), torch.bfloat16), guarded((cap, B, F, Hkv, d), torch.bfloat16)
    gi = guarded((cap,), torch.int32, 0)
    guards = [gk, gv, gi]
    cache = va.KVCache(gk.t, gv.t, gi.t)
    if rope is not None:
        gr = guarded((cap + 1, B, F, Hkv, d), torch.bfloat16)
        guards.append(gr)
        cache.enable_rope(gr.t, rope, tab)
    nws = va.vattn_kvcache_step_workspace_bytes(cache, H, wb)
    gw = guarded((nws,), torch.uint8, 0)
    guards.append(gw)
    qd, kd, vd = to_dev(q), to_dev(k), to_dev(v)
    o = torch.full((B, L, H, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    go = guarded((B, F, H, d), torch.bfloat16, float("nan"))
    gl = guarded((B, H, F), torch.float32, float("nan"))
    guards += [go, gl]
    for f in range(T):
        sl = slice(f * F, (f + 1) * F)
        qf, kf, vf = qd[:, sl].contiguous(), kd[:, sl].contiguous(), vd[:, sl].contiguous()
        cache.step(qf, kf, vf, go.t, f, wb, scale=d ** -0.5, lse=gl.t, rope=rope, table=tab,
                   window_relative=window_relative, workspace=gw.t)
        o[:, sl] = go.t
        if check is not None:
            check(f, gk.t, gv.t, gi.t, cache)
        check_guards(*guards, what="step frame %d" % f)
    va.vattn_check()
    # every step leaves its counters at zero (the workspace's first 256 bytes)
    assert int(gw.t[:256].count_nonzero()) == 0, "step counters not reset"
    cache.close()
    return o, nws


@pytest.mark.parametrize("use_rope", [True, False], ids=["rope", "no-rope"])
@pytest.mark.parametrize("window_relative", [False, True], ids=["absolute", "window-relative"])
def test_step_ring_bit_exact_and_parity(va, use_rope, window_relative):
    if window_relative and not use_rope:
        pytest.skip("window-relative positions need rope")
    T, Hg, Wg, H, d, wb = 9, 5, 30, 2, 64, 4      # F = 150: ragged frame tiles
    cap = wb + 1
    F = Hg * Wg
    L = T * F
    q = si.normal_bf16(131, (1, L, H, d))
    k = si.normal_bf16(132, (1, L, H, d))
    v = si.normal_bf16(133, (1, L, H, d))
    rope = va.Rope(Hg=Hg, Wg=Wg, pairs=(12, 10, 10), max_pos=64) if use_rope else None
    tab = va.rope_table(rope, d) if use_rope else None
    kf = k.reshape(1, T, F, H, d).transpose(1, 0, 2, 3, 4)
    vf = v.reshape(1, T, F, H, d).transpose(1, 0, 2, 3, 4)

    def check_ring(f, kr, vr, ids, cache):
        ek, ev, eids = oracle.ring_model(kf[:f + 1], vf[:f + 1], cap)
        assert np.array_equal(bits_of(kr), ek), "K ring differs after frame %d" % f
        assert np.array_equal(bits_of(vr), ev), "V ring differs after frame %d" % f
        assert list(ids.cpu().numpy()) == list(eids) == cache.host_frame_ids()

    o, nws = _decode(va, q, k, v, F, H, H, d, cap, wb, rope, tab, window_relative, check_ring)
    orope = dict(Hg=Hg, Wg=Wg, pairs=(12, 10, 10), theta=1e4) if use_rope else None
    ref, _ = oracle.stream(q, k, v, F, d ** -0.5, wb, rope=orope, window_relative=window_relative)
    assert_parity(from_dev(o), ref, "step")
    # 4 (pair, head) work units over up to 15 key tiles: the key tiles are
    # split across CTAs (the workspace holds partial results)
    assert nws > 256 + 4 * 4, "no key split for a 4-unit launch"


def test_step_equals_stream_then_append(va):
    # The one-launch step and the three-launch form (rotate, attend, append)
    # produce the same outputs and the same ring.
    import torch
    T, Hg, Wg, H, d, wb = 7, 4, 40, 2, 64, 3
    cap, F = wb + 1, Hg * Wg
    q = si.normal_bf16(141, (1, T * F, H, d))
    k = si.normal_bf16(142, (1, T * F, H, d))
    v = si.normal_bf16(143, (1, T * F, H, d))
    rope = va.Rope(Hg=Hg, Wg=Wg, pairs=(12, 10, 10), max_pos=64)
    tab = va.rope_table(rope, d)
    qd, kd, vd = to_dev(q), to_dev(k), to_dev(v)
    caches = []
    for _ in range(2):
        kr = torch.zeros((cap, 1, F, H, d), dtype=torch.bfloat16, device="cuda")
        c = va.KVCache(kr, torch.zeros_like(kr), torch.zeros(cap, dtype=torch.int32, device="cuda"))
        c.enable_rope(torch.zeros((cap + 1, 1, F, H, d), dtype=torch.bfloat16, device="cuda"), rope, tab)
        caches.append(c)
    for f in range(T):
        sl = slice(f * F, (f + 1) * F)
        qf, kf, vf = qd[:, sl].contiguous(), kd[:, sl].contiguous(), vd[:, sl].contiguous()
        o1 = torch.empty_like(qf)
        o2 = torch.empty_like(qf)
        caches[0].attend(qf, kf, vf, o1, f, wb, rope=rope, table=tab)
        caches[0].append(kf, vf, f)
        caches[1].step(qf, kf, vf, o2, f, wb, rope=rope, table=tab)
        va.vattn_check()
        a, b = from_dev(o1), from_dev(o2)
        assert np.max(np.abs(a - b)) < 1e-2, "frame %d" % f
    assert torch.equal(caches[0].k_ring, caches[1].k_ring) and torch.equal(caches[0].v_ring, caches[1].v_ring)
    assert torch.equal(caches[0].frame_ids, caches[1].frame_ids)
    for c in caches:
        c.close()


def test_step_window_relative_long_stream_small_table(va):
    # Positions relative to the window keep every RoPE t below r * (W + 1):
    # a 14-step stream (28 latent frames) runs on a 6-row table that absolute
    # positions would overrun from the third step on.  Two latent frames per
    # step (temporal refinement), GQA 4 / 2 heads.
    Hg, Wg, sub, T, H, Hkv, d, wb = 2, 6, 2, 14, 4, 2, 64, 2
    F = sub * Hg * Wg            # 24 tokens per step
    q = si.normal_bf16(151, (1, T * F, H, d))
    k = si.normal_bf16(152, (1, T * F, Hkv, d))
    v = si.normal_bf16(153, (1, T * F, Hkv, d))
    rope = va.Rope(Hg=Hg, Wg=Wg, pairs=(12, 10, 10), max_pos=sub * (wb + 1))
    tab = va.rope_table(rope, d)
    o, _ = _decode(va, q, k, v, F, H, Hkv, d, wb + 1, wb, rope, tab, window_relative=True)
    ref, _ = oracle.stream(q, k, v, F, d ** -0.5, wb, rope=dict(Hg=Hg, Wg=Wg, pairs=(12, 10, 10), theta=1e4),
                           window_relative=True)
    assert_parity(from_dev(o), ref, "window-relative step")


@pytest.mark.parametrize("name", ["xl480", "xl720", "xl480_refine", "stream"])
def test_step_config_sampled_rows(va, name):
    # Full-size FlashDecoder-XL-shaped streams (24 heads on 3 KV heads, head
    # dim 64, window 2, positions relative to the window; the refinement layer
    # with 4 latent frames per step) and the 16-head stream config (ring of
    # W + 1 = 5 frames, absolute positions) through the one-launch step.
    import torch
    c = si.CONFIGS[name]
    T, Hg, Wg, H, d, wb = c["T"], c["Hg"], c["Wg"], c["H"], c["d"], c["window_back"]
    Hkv, sub = c.get("Hkv", H), c.get("sub", 1)
    rel = name != "stream"
    F = sub * Hg * Wg
    L = T * F
    q, k, v = si.qkv(name)
    rope = va.Rope(Hg=Hg, Wg=Wg, pairs=c["pairs"], max_pos=max(64, Hg, Wg), theta=c["theta"])
    tab = va.rope_table(rope, d)
    o, _ = _decode(va, q, k, v, F, H, Hkv, d, wb + 1, wb, rope, tab, window_relative=rel)
    rows = si.sample_rows(0x5EED0000 + 16 * c["index"] + 7, N_ROWS, 1, H, L, forced=si.boundary_tokens(L, F))
    ref, _ = oracle.stream(q, k, v, F, d ** -0.5, wb,
                           rope=dict(Hg=Hg, Wg=Wg, pairs=c["pairs"], theta=c["theta"]), rows=rows,
                           window_relative=rel)
    assert_parity(gather_rows(from_dev(o), rows), ref, "%s step" % name)
    assert not torch.isnan(o.float()).any(), "unwritten output element"
