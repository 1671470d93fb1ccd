"""Shared test utilities: bf16 bit patterns <-> torch tensors, error metrics,
and the parity bar (max-abs <= 2e-2, relative L2 <= 5e-3 against the fp64
oracle)."""
import numpy as np

MAX_ABS = 2e-2
REL_L2 = 5e-3


def to_dev(bits):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)
    return t.cuda()


def from_dev(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def bits_of(t):
    import torch
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def errors(got, ref):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    d = got - ref
    max_abs = float(np.max(np.abs(d))) if d.size else 0.0
    rel = float(np.linalg.norm(d) / max(np.linalg.norm(ref), 1e-300))
    return max_abs, rel


def assert_parity(got, ref, what="", max_abs=MAX_ABS, rel_l2=REL_L2):
    ma, rl = errors(got, ref)
    assert np.all(np.isfinite(got)), "%s: non-finite values in the CUDA result" % what
    assert ma <= max_abs and rl <= rel_l2, "%s: max-abs %.3e (bar %.1e), rel-L2 %.3e (bar %.1e)" % (
        what, ma, max_abs, rl, rel_l2)
    return ma, rl


def gather_rows(o, rows):
    """o [B, L, H, d] (numpy) at rows (b, h, i) -> [n, d]."""
    return np.stack([o[b, i, h] for b, h, i in rows])
