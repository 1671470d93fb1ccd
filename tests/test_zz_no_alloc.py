"""vattn_hybrid_chunk_noalloc: hybrid chunk attention for callers that
cannot allocate device memory (their scratch comes from a static array in
the library instead of a caller workspace).

Checked against the workspace entry point vattn_hybrid_chunk, through the C
ABI, on two calls in a row (the second call finds the previous call's
contents in the shared array).  Both entry points launch the same kernels
on the same inputs with scratch of the same layout, so the outputs and the
states must agree bit for bit.  This file is collected last on purpose."""
import ctypes

import pytest

import seeded_inputs as si
from helpers import to_dev


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_point_twice():
    import torch
    import video_diffusion_transformer_02_b200 as va
    c = si.CONFIGS["hybrid"]
    H, d = c["H"], c["d"]
    L = c["T"] * c["Hg"] * c["Wg"]
    ct = c["chunk_frames"] * c["Hg"] * c["Wg"]
    assert va.vattn_hybrid_workspace_bytes(1, L, H, d, ct) <= va.HYBRID_NOALLOC_MAX_BYTES
    q, k, v = (to_dev(x) for x in si.qkv("hybrid"))

    def zero_state():
        return (torch.zeros((1, H, d, d), dtype=torch.float32, device="cuda"),
                torch.zeros((1, H, d), dtype=torch.float32, device="cuda"))

    S_ref, z_ref = zero_state()
    o_ref = torch.empty_like(q)
    va.vattn_hybrid_chunk(q, k, v, o_ref, S_ref, z_ref, ct)
    va.vattn_check()
    for call in range(2):
        S, z = zero_state()
        o = torch.full_like(q, float("nan"))
        va.vattn_hybrid_chunk_noalloc(q, k, v, o, S, z, ct)
        va.vattn_check()
        assert torch.equal(o, o_ref), "no-alloc call %d: output differs from the workspace call" % call
        assert torch.equal(S, S_ref), "no-alloc call %d: S differs from the workspace call" % call
        assert torch.equal(z, z_ref), "no-alloc call %d: z differs from the workspace call" % call


def test_noalloc_rejects_oversized_scratch():
    # Runs without a GPU: the size check precedes every CUDA call.
    from conftest import load_build_module
    lib = ctypes.CDLL(load_build_module().build())
    f = lib.vattn_hybrid_chunk_noalloc
    P, I = ctypes.c_void_p, ctypes.c_int
    f.restype = I
    f.argtypes = [P, P, P, P, P, P, I, I, I, I, I, ctypes.c_float, P]
    big = 0x10000
    # 64 chunks x 24 heads x (128*128 + 128) x 4 bytes = 101 MB > 32 MiB
    assert f(big, big, big, big, big, big, 1, 64 * 100, 24, 128, 100, 0.1, None) == 2
    lib.vattn_last_error.restype = ctypes.c_char_p
    assert b"static scratch" in lib.vattn_last_error()
