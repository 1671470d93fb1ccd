"""GPU parity of the tail split of FULL attention calls.

With a zero-filled workspace of vattn_attention_workspace_bytes_ex bytes, a
call whose (query-tile pair, head, batch) work units leave a last partial
wave of at most half the SMs runs each unit of that wave as several CTAs
over parts of its keys and merges them exactly in the kernel.  Checked
here, each through the C ABI:
  - the split call against the fp64 oracle on sampled rows of every tail
    unit plus seeded rows elsewhere (output and lse);
  - every row outside the tail units is bit-identical to the same call
    without the split (those CTAs run the unchanged path);
  - tail rows agree with the unsplit call within rounding;
  - the arrival counters are back at zero and a second call on the same
    workspace gives bit-identical results;
  - nothing is written outside the output buffers (guard regions).
Shapes cover d = 64 and 128, GQA, RoPE, ragged query and key tails, and an
odd query-tile count (a last pair with a single tile)."""
import numpy as np
import pytest

import oracle
import seeded_inputs as si
from helpers import assert_parity, bits_of, check_guards, from_dev, guarded, to_dev

pytestmark = pytest.mark.gpu
LSE_TOL = 1e-2


@pytest.fixture(scope="module")
def va():
    import video_diffusion_transformer_02_b200 as va
    return va


def _tail(B, Lq, Lk, H, sms):
    """(units before the tail, tail units, splits) as the library lays them
    out: units ordered pair-fastest, then head, then batch."""
    pairs = ((Lq + 127) // 128 + 1) // 2
    items = pairs * H * B
    waves, r = divmod(items, sms)
    kt = (Lk + 127) // 128
    if waves < 1 or r == 0 or 2 * r > sms or kt < 2:
        return None
    sp = min(sms // r, 16, kt)
    per = -(-kt // sp)
    sp = -(-kt // per)
    return (items - r, r, sp) if sp >= 2 else None


CASES = [
    # B, Lq, Lk, H, Hkv, d, rope grid (Hg, Wg) or None
    (1, 10240, 3001, 4, 4, 128, None),
    (1, 12700, 12700, 3, 1, 64, (10, 10)),
    (2, 19000, 19000, 2, 1, 128, (10, 10)),
]


@pytest.mark.parametrize("case", CASES, ids=["d128_ragged_keys", "d64_gqa_rope", "d128_odd_tiles_rope"])
def test_tail_split_parity(va, case):
    import torch
    B, Lq, Lk, H, Hkv, d, grid = case
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    lay = _tail(B, Lq, Lk, H, sms)
    if lay is None:
        pytest.skip("no tail split for this shape on %d SMs" % sms)
    n_normal, r, sp = lay
    seed = 0x7A11 + 31 * Lq + H
    q = si.normal_bf16(seed, (B, Lq, H, d))
    k = si.normal_bf16(seed + 1, (B, Lk, Hkv, d))
    v = si.normal_bf16(seed + 2, (B, Lk, Hkv, d))
    qd, kd, vd = to_dev(q), to_dev(k), to_dev(v)
    rope = tab = None
    F = 0
    if grid is not None:
        Hg, Wg = grid
        F = Hg * Wg
        T = -(-max(Lq, Lk) // F)
        pairs = (d // 2 - 2 * (d // 6), d // 6, d // 6)
        rope = va.Rope(Hg=Hg, Wg=Wg, pairs=pairs, max_pos=max(T, Hg, Wg), theta=10000.0)
        tab = va.rope_table(rope, d)
    plain = va.vattn_attention_workspace_bytes(B, Lk, Hkv, d, rope)
    need = va.vattn_attention_workspace_bytes_ex(B, Lq, Lk, H, Hkv, d, "full", rope)
    assert need > plain, "the shape should enable the tail split"
    ws = guarded((need,), torch.uint8, 0)

    def run(workspace):
        go = guarded((B, Lq, H, d), torch.bfloat16, float("nan"))
        gl = guarded((B, H, Lq), torch.float32, float("nan"))
        va.vattn_attention(qd, kd, vd, go.t, gl.t, scale=d ** -0.5, mode="full", tokens_per_frame=F,
                           rope=rope, table=tab, workspace=workspace)
        va.vattn_check()
        check_guards(go, what="o")
        check_guards(gl, what="lse")
        return go.t, gl.t

    o_s, l_s = run(ws.t)
    check_guards(ws, what="workspace")
    # the counters (first r 32-bit words after the rotated keys) are back at zero
    base = (plain + 255) // 256 * 256 if rope is not None else 0
    assert int(ws.t[base:base + 4 * r].sum()) == 0, "tail arrival counters not reset"
    o_s2, l_s2 = run(ws.t)
    assert torch.equal(o_s, o_s2) and torch.equal(l_s, l_s2), "second call on the same workspace differs"
    o_p, l_p = run(torch.empty(plain, dtype=torch.uint8, device="cuda") if rope is not None else None)
    assert not torch.isnan(o_s.float()).any() and not torch.isnan(l_s).any(), "unwritten output element"

    # units: pair fastest, then head, then batch; the tail is the last r units
    pairs = ((Lq + 127) // 128 + 1) // 2
    tok = np.arange(Lq)
    unit = (tok // 256)[None, None, :] + pairs * (np.arange(H)[None, :, None] + H * np.arange(B)[:, None, None])
    tail_mask = torch.from_numpy(unit >= n_normal).cuda()                       # [B, H, Lq]
    ob_s, ob_p = bits_of(o_s), bits_of(o_p)                                      # [B, Lq, H, d]
    keep = ~tail_mask.permute(0, 2, 1).cpu().numpy()                             # [B, Lq, H]
    assert np.array_equal(ob_s[keep], ob_p[keep]), "rows outside the tail changed"
    assert torch.equal(l_s[~tail_mask], l_p[~tail_mask]), "lse outside the tail changed"
    tm = tail_mask.permute(0, 2, 1)
    diff = (o_s.float() - o_p.float())[tm].abs().max().item()
    assert diff <= 2e-2, "tail rows differ from the unsplit call by %.3e" % diff
    assert (l_s - l_p)[tail_mask].abs().max().item() <= 1e-3

    # oracle: rows of every tail unit (its first, last and seeded rows) plus seeded rows
    tb, th, ti = np.nonzero(unit >= n_normal)
    rng = si.sample_rows(seed + 3, 256, B, H, Lq, forced=[0, Lq - 1])
    pick = si.sample_rows(seed + 4, 512, 1, 1, len(ti))[:, 2]
    tail_rows = np.stack([tb[pick], th[pick], ti[pick]], axis=1)
    edges = []
    for u in range(n_normal, n_normal + r):
        pr, rest = u % pairs, u // pairs
        h, b = rest % H, rest // H
        lo, hi = 256 * pr, min(Lq, 256 * pr + 256) - 1
        edges += [(b, h, lo), (b, h, hi), (b, h, min(hi, lo + 128))]
    rows = np.concatenate([rng, tail_rows, np.array(edges)]).astype(np.int32)
    rope_o = None if grid is None else dict(Hg=grid[0], Wg=grid[1], pairs=rope.pairs, theta=10000.0)
    ref_o, ref_l = oracle.attention(q, k, v, d ** -0.5, mode="full", F=F, rope=rope_o, rows=rows)
    of = from_dev(o_s)
    lf = l_s.double().cpu().numpy()
    got_o = np.stack([of[b, i, h] for b, h, i in rows])
    got_l = np.array([lf[b, h, i] for b, h, i in rows])
    assert_parity(got_o, ref_o, "tail split o")
    assert np.max(np.abs(got_l - ref_l)) <= LSE_TOL, "tail split lse"
