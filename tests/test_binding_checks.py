"""The Python binding rejects tensors whose shape, dtype or device disagree
with the call before anything reaches the library (no GPU needed: the
checks run on CPU tensors).  A kernel given a smaller output, or fp32 state
in bf16, would otherwise write past the end of the tensor."""
import pytest
import torch

from helpers import Guarded

va = pytest.importorskip("video_diffusion_transformer_02_b200")


def bf(*shape):
    return torch.zeros(shape, dtype=torch.bfloat16)


def f32(*shape):
    return torch.zeros(shape, dtype=torch.float32)


def test_attention_rejects_mismatched_tensors():
    q, k, v = bf(1, 256, 4, 64), bf(1, 256, 2, 64), bf(1, 256, 2, 64)
    with pytest.raises(ValueError, match="o must have shape"):
        va.vattn_attention(q, k, v, bf(1, 255, 4, 64))
    with pytest.raises(ValueError, match="v must have shape"):
        va.vattn_attention(q, k, bf(1, 256, 4, 64), bf(1, 256, 4, 64))
    with pytest.raises(TypeError, match="v must be"):
        va.vattn_attention(q, k, f32(1, 256, 2, 64), bf(1, 256, 4, 64))
    with pytest.raises(ValueError, match="lse must have shape"):
        va.vattn_attention(q, k, v, bf(1, 256, 4, 64), lse=f32(1, 4, 255))
    with pytest.raises(TypeError, match="lse must be"):
        va.vattn_attention(q, k, v, bf(1, 256, 4, 64), lse=bf(1, 4, 256))
    with pytest.raises(ValueError, match="q must have 4 dimensions"):
        va.vattn_attention(bf(256, 4, 64), k, v, bf(1, 256, 4, 64))
    # right shapes, but not on a CUDA device
    with pytest.raises(ValueError, match="CUDA device"):
        va.vattn_attention(q, k, v, bf(1, 256, 4, 64))


def test_hybrid_rejects_wrong_state_dtype_and_shape():
    q = bf(1, 300, 2, 128)
    o = bf(1, 300, 2, 128)
    for fn in (va.vattn_hybrid_chunk, va.vattn_hybrid_chunk_noalloc):
        with pytest.raises(TypeError, match="S must be"):
            fn(q, q, q, o, torch.zeros((1, 2, 128, 128), dtype=torch.bfloat16), f32(1, 2, 128), 100)
        with pytest.raises(ValueError, match="S must have shape"):
            fn(q, q, q, o, f32(1, 2, 128, 64), f32(1, 2, 128), 100)
        with pytest.raises(ValueError, match="z must have shape"):
            fn(q, q, q, o, f32(1, 2, 128, 128), f32(1, 1, 128), 100)
        with pytest.raises(ValueError, match="o must have shape"):
            fn(q, q, q, bf(1, 299, 2, 128), f32(1, 2, 128, 128), f32(1, 2, 128), 100)
        with pytest.raises(ValueError, match="CUDA device"):
            fn(q, q, q, o, f32(1, 2, 128, 128), f32(1, 2, 128), 100)


def test_kvcache_rejects_mismatched_ring():
    with pytest.raises(ValueError, match="v_ring must have shape"):
        va.KVCache(bf(4, 1, 64, 2, 64), bf(4, 1, 64, 2, 128), torch.zeros(4, dtype=torch.int32))
    with pytest.raises(TypeError, match="frame_ids must be"):
        va.KVCache(bf(4, 1, 64, 2, 64), bf(4, 1, 64, 2, 64), torch.zeros(4, dtype=torch.int64))
    with pytest.raises(ValueError, match="frame_ids must have shape"):
        va.KVCache(bf(4, 1, 64, 2, 64), bf(4, 1, 64, 2, 64), torch.zeros(5, dtype=torch.int32))
    with pytest.raises(ValueError, match="CUDA device"):
        va.KVCache(bf(4, 1, 64, 2, 64), bf(4, 1, 64, 2, 64), torch.zeros(4, dtype=torch.int32))


def test_rope_rejects_mismatched_outputs():
    r = va.Rope(Hg=4, Wg=4, pairs=(12, 10, 10), max_pos=8)
    with pytest.raises(ValueError, match="q_out must have shape"):
        va.vattn_rope_qk(bf(1, 48, 2, 64), None, bf(1, 48, 1, 64), None, r, f32(8 * 32 * 2))
    with pytest.raises(ValueError, match="go together"):
        va.vattn_rope_qk(bf(1, 48, 2, 64), None, None, None, r, f32(8 * 32 * 2))


def test_guard_regions_detect_an_overrun():
    # The guard helper of the GPU tests, checked on the CPU: one byte written
    # just past the end of the buffer is caught.
    g = Guarded((3, 5), torch.float32, fill=0.0, device="cpu")
    g.check("clean")
    g.buf[g.g + 15] = 1.0          # the first element after the tensor
    with pytest.raises(AssertionError, match="after the buffer"):
        g.check("overrun")
