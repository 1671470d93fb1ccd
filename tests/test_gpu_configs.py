"""GPU parity at the full configuration sizes, in the launch configuration
the benchmark times, on seeded-sampled query rows (4096 plus forced edge
rows: first/last token, tile edges, every frame or chunk boundary +-1, the
last partial tile) against the fp64 oracle."""
import numpy as np
import pytest

import oracle
import seeded_inputs as si
from helpers import assert_parity, check_guards, from_dev, gather_rows, guarded, to_dev

pytestmark = pytest.mark.gpu
N_ROWS = 4096


@pytest.fixture(scope="module")
def va():
    import video_diffusion_transformer_02_b200 as va
    return va


def _dev_qkv(name):
    q, k, v = si.qkv(name)
    return (q, k, v), (to_dev(q), to_dev(k), to_dev(v))


@pytest.mark.parametrize("name,mode", [("wan13b", "full"), ("wan14b", "full"), ("wan14b", "chunk_causal")])
def test_large_attention_sampled_rows(va, name, mode):
    import torch
    c = si.CONFIGS[name]
    T, Hg, Wg, H, d = c["T"], c["Hg"], c["Wg"], c["H"], c["d"]
    F, L = Hg * Wg, T * Hg * Wg
    (q, k, v), (qd, kd, vd) = _dev_qkv(name)
    rope = va.Rope(Hg=Hg, Wg=Wg, pairs=c["pairs"], max_pos=max(T, Hg, Wg), theta=c["theta"])
    tab = va.rope_table(rope, d)
    go = guarded(qd.shape, torch.bfloat16, float("nan"))
    o = go.t
    chunk = c.get("chunk_frames", 1)
    va.vattn_attention(qd, kd, vd, o, scale=d ** -0.5, mode=mode, tokens_per_frame=F,
                       chunk_frames=chunk, rope=rope, table=tab)
    va.vattn_check()
    check_guards(go, what="%s %s o" % (name, mode))
    period = F * chunk if mode == "chunk_causal" else F
    rows = si.sample_rows(0x5EED0000 + 16 * c["index"] + 7, N_ROWS, 1, H, L,
                          forced=si.boundary_tokens(L, period))
    ref, _ = oracle.attention(q, k, v, d ** -0.5, mode=mode, F=F, chunk=chunk,
                              rope=dict(Hg=Hg, Wg=Wg, pairs=c["pairs"], theta=c["theta"]), rows=rows)
    got = gather_rows(from_dev(o), rows)
    assert_parity(got, ref, "%s %s" % (name, mode))
    assert not torch.isnan(o.float()).any(), "unwritten output element"


def test_stream_config_sampled_rows(va):
    import torch
    c = si.CONFIGS["stream"]
    T, Hg, Wg, H, d, cap, wb = c["T"], c["Hg"], c["Wg"], c["H"], c["d"], c["capacity"], c["window_back"]
    F, L = Hg * Wg, T * Hg * Wg
    (q, k, v), (qd, kd, vd) = _dev_qkv("stream")
    rope = va.Rope(Hg=Hg, Wg=Wg, pairs=c["pairs"], max_pos=64, theta=c["theta"])
    tab = va.rope_table(rope, d)
    gk, gv = guarded((cap, 1, F, H, d), torch.bfloat16), guarded((cap, 1, F, H, d), torch.bfloat16)
    gi, gr = guarded((cap,), torch.int32, 0), guarded((cap + 1, 1, F, H, d), torch.bfloat16)
    kr, vr, ids = gk.t, gv.t, gi.t
    cache = va.KVCache(kr, vr, ids)
    cache.enable_rope(gr.t, rope, tab)
    o = torch.full(qd.shape, float("nan"), dtype=torch.bfloat16, device="cuda")
    for f in range(T):
        sl = slice(f * F, (f + 1) * F)
        qf, kf, vf = qd[:, sl].contiguous(), kd[:, sl].contiguous(), vd[:, sl].contiguous()
        of = torch.empty_like(qf)
        cache.attend(qf, kf, vf, of, f, wb, rope=rope, table=tab)
        cache.append(kf, vf, f)
        o[:, sl] = of
    va.vattn_check()
    check_guards(gk, gv, gi, gr, what="stream config ring")
    # ring holds frames 28..31 bit for bit
    kb = k.reshape(T, F, H, d)
    for slot in range(cap):
        fr = ids[slot].item()
        assert fr == T - cap + ((slot - (T - cap)) % cap)
        got = kr[slot, 0].contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
        assert np.array_equal(got, kb[fr])
    rows = si.sample_rows(0x5EED0000 + 16 * 2 + 7, N_ROWS, 1, H, L, forced=si.boundary_tokens(L, F))
    ref, _ = oracle.stream(q, k, v, F, d ** -0.5, wb,
                           rope=dict(Hg=Hg, Wg=Wg, pairs=c["pairs"], theta=c["theta"]), rows=rows)
    assert_parity(gather_rows(from_dev(o), rows), ref, "stream config")
    cache.close()


def test_hybrid_config(va):
    import torch
    c = si.CONFIGS["hybrid"]
    T, Hg, Wg, H, d = c["T"], c["Hg"], c["Wg"], c["H"], c["d"]
    L, ct = T * Hg * Wg, c["chunk_frames"] * Hg * Wg
    (q, k, v), (qd, kd, vd) = _dev_qkv("hybrid")
    gS, gz = guarded((1, H, d, d), torch.float32), guarded((1, H, d), torch.float32)
    go = guarded(qd.shape, torch.bfloat16, float("nan"))
    S, z, o = gS.t, gz.t, go.t
    va.vattn_hybrid_chunk(qd, kd, vd, o, S, z, ct, scale=d ** -0.5)
    va.vattn_check()
    check_guards(gS, gz, go, what="hybrid config o / S / z")
    rows = si.sample_rows(0x5EED0000 + 16 * 3 + 7, N_ROWS, 1, H, L, forced=si.boundary_tokens(L, ct))
    mask = np.zeros((1, H, L), dtype=bool)
    mask[rows[:, 0], rows[:, 1], rows[:, 2]] = True
    ro, rS, rz = oracle.hybrid_recurrent(q, k, v, ct, d ** -0.5, row_mask=mask)
    assert_parity(gather_rows(from_dev(o), rows), gather_rows(ro, rows), "hybrid config")
    assert_parity(S.cpu().numpy(), rS, "hybrid S", max_abs=np.inf)
    assert_parity(z.cpu().numpy(), rz, "hybrid z", max_abs=np.inf)
    assert not torch.isnan(o.float()).any(), "unwritten output element"
