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


# ------------------------------------------------------------ guard regions
# Every output, ring and state buffer a GPU test hands to the library sits
# inside a larger allocation whose first and last GUARD_BYTES hold a fixed
# byte pattern; check_guards() after a call proves that nothing was written
# past either end of the buffer.
GUARD_BYTES = 4096
GUARD_BYTE = 0xA5


class Guarded:
    """A contiguous tensor of `shape`/`dtype` with guard regions around it."""

    def __init__(self, shape, dtype, fill=0.0, device="cuda"):
        import torch
        itemsize = torch.empty((), dtype=dtype).element_size()
        self.g = GUARD_BYTES // itemsize
        n = int(np.prod(shape)) if len(shape) else 1
        self.buf = torch.empty(n + 2 * self.g, dtype=dtype, device=device)
        self.buf.view(torch.uint8).fill_(GUARD_BYTE)
        self.t = self.buf[self.g:self.g + n].view(shape)
        if fill is not None:
            self.t.fill_(fill)

    def check(self, what=""):
        import torch
        raw = self.buf.view(torch.uint8)
        nb = self.g * self.buf.element_size()
        head, tail = raw[:nb], raw[raw.numel() - nb:]
        bad_head = int((head != GUARD_BYTE).sum())
        bad_tail = int((tail != GUARD_BYTE).sum())
        assert bad_head == 0 and bad_tail == 0, (
            "%s: %d guard bytes before and %d after the buffer were overwritten" % (what, bad_head, bad_tail))


def guarded(shape, dtype, fill=0.0, device="cuda"):
    return Guarded(tuple(shape), dtype, fill, device)


def check_guards(*gs, what=""):
    for g in gs:
        g.check(what)
