"""Host-side checks of the C ABI (no GPU needed): the library builds for
sm_100a, loads, exports every entry point that include/*.h declares, and
rejects invalid arguments before touching the device."""
import ctypes
import glob
import os
import re

import pytest

from conftest import load_build_module

_build = load_build_module()

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    return ctypes.CDLL(_build.build())


def declared_functions():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names.update(re.findall(r"\b(vattn_[a-z0-9_]+)\s*\(", text))
    return sorted(names)


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert len(names) >= 15
    for n in names:
        assert hasattr(lib, n), "libvattn.so does not export %s" % n


def _sig(lib, name, res, *args):
    f = getattr(lib, name)
    f.restype, f.argtypes = res, list(args)
    return f


P, I, F = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
FAKE = 0x10000   # a 16-byte aligned non-NULL value: rejected calls never dereference it


def test_status_strings(lib):
    f = _sig(lib, "vattn_status_string", ctypes.c_char_p, I)
    assert f(0) == b"ok" and f(4) == b"kernel wait timed out"


def test_attention_argument_checks(lib):
    att = _sig(lib, "vattn_attention", I, P, P, P, P, P, I, I, I, I, I, I, F, I, I, I, I, I, I, I, P,
               P, P, ctypes.c_size_t, P)
    good = dict(B=1, Lq=48, Lk=48, H=2, Hkv=2, d=64)

    def call(q=FAKE, k=FAKE, v=FAKE, o=FAKE, d=64, H=2, Hkv=2, mode=0, tpf=16, chunk=1, wb=0, wf=0,
             qoff=0, koff=0, scale=0.125):
        return att(q, k, v, o, None, 1, 48, 48, H, Hkv, d, scale, mode, tpf, chunk, wb, wf, qoff, koff,
                   None, None, None, 0, None)

    assert call(q=None) == 1                       # NULL
    assert call(q=FAKE + 8) == 1                   # misaligned
    assert call(d=96) == 2                         # unsupported head dim
    assert call(H=3, Hkv=2) == 1                   # GQA group mismatch
    assert call(mode=7) == 1
    assert call(mode=1, chunk=0) == 1
    assert call(mode=2, wb=-1) == 1
    assert call(mode=1, tpf=0) == 1
    assert call(qoff=-1) == 1
    assert call(scale=float("inf")) == 1
    last = _sig(lib, "vattn_last_error", ctypes.c_char_p)
    assert b"window" in last() or len(last()) > 0


def test_rope_table_size(lib):
    class Rope(ctypes.Structure):
        _fields_ = [("Hg", I), ("Wg", I), ("pt", I), ("ph", I), ("pw", I), ("max_pos", I),
                    ("theta", ctypes.c_double)]
    f = _sig(lib, "vattn_rope_table_bytes", ctypes.c_size_t, ctypes.POINTER(Rope), I)
    assert f(ctypes.byref(Rope(45, 80, 22, 21, 21, 80, 1e4)), 128) == 80 * 64 * 8
    assert f(ctypes.byref(Rope(45, 80, 22, 21, 20, 80, 1e4)), 128) == 0   # pairs do not sum to d/2
    assert f(ctypes.byref(Rope(45, 80, 22, 21, 21, 40, 1e4)), 128) == 0   # grid beyond table


def test_hybrid_workspace_and_checks(lib):
    ws = _sig(lib, "vattn_hybrid_workspace_bytes", ctypes.c_size_t, I, I, I, I, I)
    assert ws(1, 12090, 24, 128, 1170) == 11 * 24 * (128 * 128 + 128) * 4
    hyb = _sig(lib, "vattn_hybrid_chunk", I, P, P, P, P, P, P, I, I, I, I, I, F, P, ctypes.c_size_t, P)
    assert hyb(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1, 100, 2, 64, 50, 0.1, FAKE, 1 << 30, None) == 2
    assert hyb(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1, 100, 2, 128, 50, 0.1, FAKE, 16, None) == 1
    assert hyb(FAKE, FAKE, FAKE, FAKE, FAKE, None, 1, 100, 2, 128, 50, 0.1, FAKE, 1 << 30, None) == 1


def _tail_bytes(B, Lq, Lk, H, d, sms=148):
    """The tail-split workspace layout as include/vattn.h documents it: r
    arrival counters, then lse fp32 [r][s][256] and o fp32 [r][s][256][d],
    each part from a 256-byte boundary; 0 when the split does not apply."""
    up = lambda x: (x + 255) // 256 * 256
    items = ((Lq + 127) // 128 + 1) // 2 * H * B
    waves, r = divmod(items, sms)
    kt = (Lk + 127) // 128
    if waves < 1 or r == 0 or 2 * r > sms or kt < 2:
        return 0
    s = min(sms // r, 16, kt)
    per = -(-kt // s)
    s = -(-kt // per)
    if s < 2:
        return 0
    off_o = up(r * 4) + up(r * s * 256 * 4)
    return off_o + r * s * 256 * d * 4


@pytest.mark.parametrize("shape", [
    (1, 32760, 32760, 12, 12, 128),    # the 1.3B-like call: 10 waves + 56 pairs, 2 splits each
    (1, 10240, 3001, 4, 4, 128),       # 160 pairs: 12 left over, 12 splits
    (1, 12700, 12700, 3, 1, 64),       # GQA, 2 left over, 15 splits (16 would leave one empty)
    (1, 75600, 75600, 40, 40, 128),    # the 14B-like call: exactly 80 waves, no split
    (1, 2040, 2040, 16, 16, 64),       # one partial wave only: no split
])
@pytest.mark.parametrize("with_rope", [False, True])
def test_attention_workspace_sizes(lib, shape, with_rope):
    # Without a GPU the library sizes for 148 SMs (a B200).
    class Rope(ctypes.Structure):
        _fields_ = [("Hg", I), ("Wg", I), ("pt", I), ("ph", I), ("pw", I), ("max_pos", I),
                    ("theta", ctypes.c_double)]
    B, Lq, Lk, H, Hkv, d = shape
    base = _sig(lib, "vattn_attention_workspace_bytes", ctypes.c_size_t, I, I, I, I, ctypes.POINTER(Rope))
    ex = _sig(lib, "vattn_attention_workspace_bytes_ex", ctypes.c_size_t, I, I, I, I, I, I, I,
              ctypes.POINTER(Rope))
    rope = ctypes.byref(Rope(10, 10, d // 2 - 2 * (d // 6), d // 6, d // 6, 8192, 1e4)) if with_rope else None
    rot = B * Lk * Hkv * d * 2 if with_rope else 0
    assert base(B, Lk, Hkv, d, rope) == rot
    tail = _tail_bytes(B, Lq, Lk, H, d)
    want = ((rot + 255) // 256 * 256 + tail) if tail else rot
    assert ex(B, Lq, Lk, H, Hkv, d, 0, rope) == want
    for mode in (1, 2):   # masked modes never split the tail
        assert ex(B, Lq, Lk, H, Hkv, d, mode, rope) == rot
    if shape[:3] == (1, 32760, 32760) and with_rope:
        assert want == 115433728   # the size the 1.3B-like benchmark allocates


def test_kvcache_checks(lib):
    init = _sig(lib, "vattn_kvcache_init", I, ctypes.POINTER(P), P, P, P, I, I, I, I, I, P)
    h = P()
    assert init(ctypes.byref(h), FAKE, FAKE, FAKE, 0, 1, 2040, 16, 64, None) == 2   # capacity 0
    assert init(ctypes.byref(h), FAKE, FAKE, FAKE, 9, 1, 2040, 16, 64, None) == 2   # > 7 segments
    assert init(ctypes.byref(h), FAKE, FAKE, FAKE, 4, 1, 2040, 16, 80, None) == 2   # head dim
    assert init(ctypes.byref(h), None, FAKE, FAKE, 4, 1, 2040, 16, 64, None) == 1


def test_package_refuses_without_library(tmp_path, monkeypatch):
    # The Python package must fail loudly when the CUDA library is absent.
    import importlib.util
    import shutil
    pkg = os.path.join(ROOT, "video_diffusion_transformer_02_b200")
    dst = tmp_path / "video_diffusion_transformer_02_b200"
    shutil.copytree(pkg, dst, ignore=shutil.ignore_patterns("*.so", "csrc", "__pycache__"))
    spec = importlib.util.spec_from_file_location("vattn_copy", dst / "__init__.py")
    mod = importlib.util.module_from_spec(spec)
    with pytest.raises(ImportError):
        spec.loader.exec_module(mod)
