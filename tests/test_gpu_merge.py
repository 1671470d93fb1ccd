"""Ring attention's exact join on one GPU: K/V split into R shards along the
sequence (frame-aligned, so masks and RoPE positions carry over through the
frame offsets), one vattn_attention call per shard with its lse, then
vattn_attention_merge.  The merged result must match the fp64 oracle's
attention over all keys (and the one-shot call); a shard that a row cannot
see (lse = -inf) must weigh nothing."""
import numpy as np
import pytest

import oracle
import seeded_inputs as si
from helpers import assert_parity, check_guards, from_dev, guarded, to_dev

pytestmark = pytest.mark.gpu
LSE_TOL = 1e-2


@pytest.fixture(scope="module")
def va():
    import video_diffusion_transformer_02_b200 as va
    return va


CASES = [
    # (T, Hg, Wg, H, Hkv, d, mode, kwargs, R, rope)
    (6, 5, 10, 2, 2, 128, "full", {}, 3, True),
    (6, 5, 10, 4, 2, 64, "full", {}, 2, False),
    (8, 4, 10, 2, 2, 64, "chunk_causal", dict(chunk=2), 4, True),    # later shards invisible to early rows
    (8, 4, 10, 2, 1, 128, "sliding", dict(wb=1, wf=0), 4, True),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "%s-d%d-R%d%s" % (c[6], c[5], c[8], "-rope" if c[9] else ""))
def test_merge_of_key_shards(va, case):
    import torch
    from video_diffusion_transformer_02_b200 import usp
    T, Hg, Wg, H, Hkv, d, mode, kw, R, use_rope = case
    F = Hg * Wg
    L = T * F
    q = si.normal_bf16(171, (1, L, H, d))
    k = si.normal_bf16(172, (1, L, Hkv, d))
    v = si.normal_bf16(173, (1, L, Hkv, d))
    qd, kd, vd = to_dev(q), to_dev(k), to_dev(v)
    pairs = (12, 10, 10) if d == 64 else (22, 21, 21)
    rope = va.Rope(Hg=Hg, Wg=Wg, pairs=pairs, max_pos=max(T, Hg, Wg) + 1) if use_rope else None
    tab = va.rope_table(rope, d) if use_rope else None
    attend = usp.gpu_attend(d ** -0.5, mode=mode, tokens_per_frame=F, chunk_frames=kw.get("chunk", 1),
                            window_back=kw.get("wb", 0), window_fwd=kw.get("wf", 0), rope=rope, table=tab)
    frames = np.linspace(0, T, R + 1).round().astype(int)
    o_parts, l_parts = [], []
    for a, b in zip(frames, frames[1:]):
        o, lse = attend(qd, kd[:, a * F:b * F].contiguous(), vd[:, a * F:b * F].contiguous(), 0, a * F)
        o_parts.append(o)
        l_parts.append(lse)
    op, lp = torch.stack(o_parts), torch.stack(l_parts)
    if mode == "chunk_causal":
        assert torch.isinf(lp).any(), "some row must see no key of some shard"
    go = guarded((1, L, H, d), torch.bfloat16, float("nan"))
    gl = guarded((1, H, L), torch.float32, float("nan"))
    va.vattn_attention_merge(op, lp, go.t, gl.t)
    va.vattn_check()
    check_guards(go, gl, what="merge o / lse")
    orope = dict(Hg=Hg, Wg=Wg, pairs=pairs, theta=1e4) if use_rope else None
    ref, rl = oracle.attention(q, k, v, d ** -0.5, mode=mode, F=F, chunk=kw.get("chunk", 1), wb=kw.get("wb", 0),
                               wf=kw.get("wf", 0), rope=orope)
    assert_parity(from_dev(go.t), ref, "merged shards")
    assert np.max(np.abs(gl.t.cpu().numpy() - rl)) < LSE_TOL
    one, _ = attend(qd, kd, vd, 0, 0)
    assert np.max(np.abs(from_dev(one) - from_dev(go.t))) < 2e-2


def test_merge_closed_form(va):
    # Two parts with lse 0 and ln 3 weigh 1 : 3; a part with lse = -inf
    # weighs nothing; a row with every lse = -inf is 0 with lse -inf.
    import torch
    o_parts = torch.zeros((3, 1, 2, 1, 8), dtype=torch.bfloat16, device="cuda")
    o_parts[0, 0, :, 0, 0] = 1.0
    o_parts[1, 0, :, 0, 1] = 1.0
    o_parts[2, 0, :, 0, :] = 5.0
    lse = torch.tensor([[[[0.0, -float("inf")]]], [[[np.log(3.0), -float("inf")]]],
                        [[[-float("inf"), -float("inf")]]]], dtype=torch.float32, device="cuda")
    o = torch.full((1, 2, 1, 8), float("nan"), dtype=torch.bfloat16, device="cuda")
    lo = torch.full((1, 1, 2), float("nan"), dtype=torch.float32, device="cuda")
    va.vattn_attention_merge(o_parts, lse, o, lo)
    va.vattn_check()
    got = o.float().cpu().numpy()[0, :, 0]
    assert abs(got[0, 0] - 0.25) < 2e-3 and abs(got[0, 1] - 0.75) < 4e-3 and np.all(got[0, 2:] == 0)
    assert np.all(got[1] == 0) and lo[0, 0, 1].item() == -float("inf")
    assert abs(lo[0, 0, 0].item() - np.log(4.0)) < 1e-5
