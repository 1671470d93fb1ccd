"""GPU parity of the general hybrid chunk attention (vattn_hybrid_chunk_ex):
the MobileWan page variant's degree-3 polynomial feature maps and softmax
chunks overlapping the previous chunk, against the fp64 oracle's recurrent
form; with elu + 1 and no overlap it must equal vattn_hybrid_chunk bit for
bit."""
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


def _run(va, q, k, v, ct, ov, coef):
    import torch
    B, L, H, d = q.shape
    gS, gz = guarded((B, H, d, d), torch.float32), guarded((B, H, d), torch.float32)
    go = guarded((B, L, H, d), torch.bfloat16, float("nan"))
    cd = None if coef is None else torch.from_numpy(coef.astype(np.float32)).cuda()
    va.vattn_hybrid_chunk_ex(to_dev(q), to_dev(k), to_dev(v), go.t, gS.t, gz.t, ct, ov, scale=d ** -0.5, coef=cd)
    va.vattn_check()
    check_guards(gS, gz, go, what="hybrid_ex o / S / z")
    return go.t, gS.t, gz.t


@pytest.mark.parametrize("L,ct,ov,poly", [(700, 300, 0, True), (700, 300, 120, True), (700, 300, 300, False),
                                          (1300, 390, 450, True), (500, 128, 700, True)])
def test_hybrid_ex_parity_all_rows(va, L, ct, ov, poly):
    H, d = 2, 128
    q = si.normal_bf16(181, (1, L, H, d))
    k = si.normal_bf16(182, (1, L, H, d))
    v = si.normal_bf16(183, (1, L, H, d))
    coef = si.poly_coef(0x9017, H) if poly else None
    o, S, z = _run(va, q, k, v, ct, ov, coef)
    ro, rS, rz = oracle.hybrid2_recurrent(q, k, v, ct, d ** -0.5, overlap=ov, fmap="poly" if poly else "elu",
                                          coef=coef)
    assert_parity(from_dev(o), ro, "hybrid_ex o")
    assert_parity(S.cpu().numpy(), rS, "hybrid_ex S", max_abs=np.inf)
    assert_parity(z.cpu().numpy(), rz, "hybrid_ex z", max_abs=np.inf)


def test_hybrid_ex_reduces_to_the_hybrid_call(va):
    import torch
    L, ct, H, d = 900, 390, 2, 128
    q, k, v = (to_dev(si.normal_bf16(191 + i, (1, L, H, d))) for i in range(3))
    outs = []
    for ex in (False, True):
        S = torch.zeros((1, H, d, d), dtype=torch.float32, device="cuda")
        z = torch.zeros((1, H, d), dtype=torch.float32, device="cuda")
        o = torch.empty_like(q)
        if ex:
            va.vattn_hybrid_chunk_ex(q, k, v, o, S, z, ct, 0)
        else:
            va.vattn_hybrid_chunk(q, k, v, o, S, z, ct)
        outs.append((o, S, z))
    va.vattn_check()
    for a, b in zip(*outs):
        assert torch.equal(a, b)


def test_hybrid_page_variant_config(va):
    # The page variant at the workload's size: 31 frames of 15 x 26 tokens,
    # 24 heads, chunks of 4 frames overlapping 2 frames of the previous one,
    # polynomial feature maps; 4096 sampled rows plus every chunk boundary.
    import torch
    c = si.CONFIGS["hybrid_page"]
    T, Hg, Wg, H, d = c["T"], c["Hg"], c["Wg"], c["H"], c["d"]
    L, ct, ov = T * Hg * Wg, c["chunk_frames"] * Hg * Wg, c["overlap_frames"] * Hg * Wg
    q, k, v = si.qkv("hybrid_page")
    coef = si.poly_coef(c["coef_seed"], H)
    o, S, z = _run(va, q, k, v, ct, ov, coef)
    rows = si.sample_rows(0x5EED0000 + 16 * c["index"] + 9, N_ROWS, 1, H, L, forced=si.boundary_tokens(L, ct))
    mask = np.zeros((1, H, L), dtype=bool)
    mask[rows[:, 0], rows[:, 1], rows[:, 2]] = True
    ro, rS, rz = oracle.hybrid2_recurrent(q, k, v, ct, d ** -0.5, overlap=ov, fmap="poly", coef=coef, row_mask=mask)
    assert_parity(gather_rows(from_dev(o), rows), gather_rows(ro, rows), "hybrid page variant")
    assert_parity(S.cpu().numpy(), rS, "hybrid page S", max_abs=np.inf)
    assert_parity(z.cpu().numpy(), rz, "hybrid page z", max_abs=np.inf)
    assert not torch.isnan(o.float()).any(), "unwritten output element"
