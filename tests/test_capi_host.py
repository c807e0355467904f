"""Host-side checks of the C ABI: the library loads, exports every symbol the
header declares, builds the same code book as the oracle, and rejects bad
arguments before launching anything (no GPU needed)."""
import ctypes
import os
import re
import subprocess

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "qlora_nf4.h")


@pytest.fixture(scope="module")
def api():
    from bit_nf4_quantised_codebook_b200 import build
    build.build()
    from bit_nf4_quantised_codebook_b200 import api as a
    return a


def _declared():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"^(?:qlora_status|const char \*)\s*(qlora_\w+)\s*\(", src, re.M)))


def test_header_declares_expected_entry_points():
    names = _declared()
    for n in ["qlora_build_codebook", "qlora_quantize", "qlora_dequantize", "qlora_linear_forward",
              "qlora_linear_backward", "qlora_nf4_sizes", "qlora_workspace_size", "qlora_status_string"]:
        assert n in names


def test_library_exports_every_declared_symbol(api):
    L = api.lib()
    out = subprocess.run(["nm", "-D", "--defined-only", api.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(ln.split()[-1] for ln in out.splitlines() if ln.strip())
    for n in _declared():
        assert n in exported, n
        assert hasattr(L, n)


def test_codebook_matches_oracle(api):
    from oracle import nf4
    lv, th = api.qlora_build_codebook()
    lv = np.array(lv, np.float32)
    th = np.array(th, np.float32)
    assert np.array_equal(lv.view(np.uint32), nf4.nf4_levels().view(np.uint32))
    assert np.array_equal(th.view(np.uint32), nf4.nf4_thresholds(nf4.nf4_levels()).view(np.uint32))


def test_sizes(api):
    from oracle import nf4
    cb, qb, sb = api.qlora_nf4_sizes(4096, 4096)
    assert cb + qb + sb + 4 == nf4.storage_bytes(4096, 4096)
    cb, qb, sb = api.qlora_nf4_sizes(3, 6400)
    assert (cb, qb, sb) == (9600, 300, 8)


def test_validation_errors(api):
    L = api.lib()
    n = ctypes.c_size_t()
    assert L.qlora_nf4_sizes(16, 100, None, None, None) == 2          # K % 64
    assert L.qlora_workspace_size(1, 4, 16, 64, 12, ctypes.byref(n)) == 2   # r % 8
    assert L.qlora_workspace_size(1, 4, 16, 64, 8, None) == 1
    assert L.qlora_workspace_size(7, 4, 16, 64, 8, ctypes.byref(n)) == 1
    assert L.qlora_workspace_size(1, 4096, 4096, 4096, 64, ctypes.byref(n)) == 0 and n.value > 0
    w = api._Weight(16, 100, 16, 16, 16, 16)
    assert L.qlora_quantize(16, ctypes.byref(w), 16, 1 << 20, None, None) == 2
    w = api._Weight(16, 128, 16, 16, 16, 16)
    assert L.qlora_quantize(None, ctypes.byref(w), 16, 1 << 20, None, None) == 1
    w = api._Weight(16, 128, 0, 16, 16, 16)
    assert L.qlora_quantize(16, ctypes.byref(w), 16, 1 << 20, None, None) == 1
    w = api._Weight(16, 128, 17, 16, 16, 16)
    assert L.qlora_quantize(16, ctypes.byref(w), 16, 1 << 20, None, None) == 3
    w = api._Weight(12, 128, 16, 16, 16, 16)                           # N % 8 for the linear layer
    assert L.qlora_linear_forward(ctypes.byref(w), 16, 4, 16, 16, 8, ctypes.c_float(1.0), 16, None, 16,
                                  1 << 20, None, None) == 2
    assert api.lib().qlora_status_string(3) == b"pointer not 16-byte aligned"


def test_merge_validation(api):
    """qlora_merge_requantize rejects bad arguments before any launch (1 = invalid
    argument, 2 = unsupported shape, 3 = misaligned); every case here fails
    before the device is touched."""
    L = api.lib()
    W = api._Weight
    w = W(16, 128, 4096, 8192, 12288, 16384)             # codes 1 KiB, c2q 32 B, c1 4 B, mean
    out = W(16, 128, 65536, 69632, 73728, 77824)
    f = ctypes.c_float(0.25)
    ok = dict(A=1 << 20, B=1 << 21, r=16)

    def call(w_=w, out_=out, A=ok["A"], B=ok["B"], r=ok["r"], wm=None):
        return L.qlora_merge_requantize(ctypes.byref(w_), A, B, r, f, ctypes.byref(out_), wm, 1 << 22, 1 << 20,
                                        None, None)

    assert call(out_=W(24, 128, 65536, 69632, 73728, 77824)) == 1   # shape mismatch
    assert call(A=None) == 1
    assert call(B=None) == 1
    assert call(r=0) == 1
    assert call(r=12) == 2
    assert call(r=264) == 2
    assert call(w_=W(12, 128, 4096, 8192, 12288, 16384), out_=W(12, 128, 65536, 69632, 73728, 77824)) == 2
    assert call(A=(1 << 20) + 8) == 3
    assert call(wm=4104) == 3
    assert call(out_=W(16, 128, 4096 + 512, 69632, 73728, 77824)) == 1   # partial overlap of codes
    assert call(out_=W(16, 128, 65536, 4096, 73728, 77824)) == 1         # out.c2q inside w.codes
    assert call(wm=8192 - 16) == 1                                        # W_merged over w's buffers


def test_format_code_books_match_oracle(api):
    """Levels bit-exact; thresholds give the oracle's nearest level (ties to the
    lower index, the upper of two equal levels never chosen)."""
    from oracle import formats, nf4
    rng = np.random.default_rng(3)
    for cb in formats.CODEBOOKS:
        lv, th = api.qlora_format_codebook(cb)
        lv = np.array(lv, np.float32)
        th = np.array(th, np.float32)
        ref = formats.codebook(cb)
        assert np.array_equal(lv.view(np.uint32), ref.view(np.uint32)), cb
        assert np.all(np.diff(th) >= 0), cb
        m = (ref[:-1].astype(np.float64) + ref[1:].astype(np.float64)) / 2
        x = np.concatenate([rng.uniform(-1, 1, 50000), m[np.abs(m) <= 1], [0.0, -1.0, 1.0, 1e-30, -1e-30]])
        x = x.astype(np.float32)
        x = np.concatenate([x, np.nextafter(x, np.float32(2)), np.nextafter(x, np.float32(-2))])
        x = x[np.abs(x) <= 1]
        codes = np.searchsorted(th, x, side="right")          # #{i : x >= t_i}
        assert np.array_equal(codes, nf4.nearest_level(x, ref)), cb
    assert api.lib().qlora_format_codebook(4, None, None) == 1


def test_format_validation(api):
    L = api.lib()
    F, Q = api._Format, api._QWeight
    n = ctypes.c_size_t()
    assert L.qlora_format_sizes(ctypes.byref(F(0, 48, 1)), 16, 96, None, None, None) == 2      # block
    assert L.qlora_format_sizes(ctypes.byref(F(4, 64, 1)), 16, 128, None, None, None) == 1     # code book
    assert L.qlora_format_sizes(ctypes.byref(F(0, 64, 3)), 16, 128, None, None, None) == 1     # constants
    assert L.qlora_format_sizes(ctypes.byref(F(0, 128, 1)), 16, 192, None, None, None) == 2    # K % block
    a, b, c = ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_size_t()
    assert L.qlora_format_sizes(ctypes.byref(F(2, 32, 0)), 16, 128, ctypes.byref(a), ctypes.byref(b),
                                ctypes.byref(c)) == 0
    assert (a.value, b.value, c.value) == (1024, 64 * 4, 0)
    assert L.qlora_format_sizes(ctypes.byref(F(1, 256, 2)), 16, 4096, ctypes.byref(a), ctypes.byref(b),
                                ctypes.byref(c)) == 0
    assert (a.value, b.value, c.value) == (32768, 256, 4)
    assert L.qlora_format_workspace_size(ctypes.byref(F(0, 32, 1)), 16, 128, ctypes.byref(n)) == 0 and n.value > 0
    w = Q(16, 128, F(0, 64, 1), 4096, 8192, 12288, 16384)
    assert L.qlora_quantize_format(None, ctypes.byref(w), 1 << 20, 1 << 20, None, None) == 1
    assert L.qlora_quantize_format(17 * 16 + 1, ctypes.byref(w), 1 << 20, 1 << 20, None, None) == 3
    assert L.qlora_quantize_format(1 << 21, ctypes.byref(Q(16, 128, F(0, 64, 1), 4096, 8192, 0, 16384)),
                                   1 << 20, 1 << 20, None, None) == 1                         # c1 needed
    assert L.qlora_quantize_format(1 << 21, ctypes.byref(w), 1 << 20, 8, None, None) == 5     # workspace
    assert L.qlora_dequantize_format(ctypes.byref(Q(16, 100, F(0, 64, 0), 4096, 8192, 0, 0)), 1 << 21, None) == 2
    assert L.qlora_quant_error(None, 16, 8, 16, None) == 1
    assert L.qlora_quant_error(16, 16, 0, 16, None) == 1
    assert L.qlora_quant_error(16, 16, 8, 12, None) == 3


def test_product_path_has_no_cpu_fallback():
    """The binding never imports the oracle; the package refuses to run without the library."""
    pkg = os.path.join(ROOT, "bit_nf4_quantised_codebook_b200")
    for f in os.listdir(pkg):
        if f.endswith(".py"):
            txt = open(os.path.join(pkg, f)).read()
            assert "import oracle" not in txt and "from oracle" not in txt, f


def test_adamw_validation(api):
    """qlora_adamw_step rejects bad arguments before any launch (1 = invalid argument,
    3 = misaligned pointer)."""
    L = api.lib()
    T = api._AdamwTensor
    good = (T * 1)(T(16, 0, 32, 48, 64, 8))  # 16-byte aligned (fake) addresses; never dereferenced
    args = (0.001, 0.9, 0.999, 1e-8, 0.0)
    assert L.qlora_adamw_step(None, 1, *args, 1, None) == 1
    assert L.qlora_adamw_step(good, 0, *args, 1, None) == 1
    assert L.qlora_adamw_step(good, 17, *args, 1, None) == 1
    assert L.qlora_adamw_step(good, 1, *args, 0, None) == 1           # step < 1
    assert L.qlora_adamw_step(good, 1, 0.001, 1.0, 0.999, 1e-8, 0.0, 1, None) == 1
    assert L.qlora_adamw_step(good, 1, 0.001, 0.9, 0.999, 0.0, 0.0, 1, None) == 1
    assert L.qlora_adamw_step(good, 1, -1.0, 0.9, 0.999, 1e-8, 0.0, 1, None) == 1
    nul = (T * 1)(T(16, 0, 0, 48, 64, 8))
    assert L.qlora_adamw_step(nul, 1, *args, 1, None) == 1
    empty = (T * 1)(T(16, 0, 32, 48, 64, 0))
    assert L.qlora_adamw_step(empty, 1, *args, 1, None) == 1
    mis = (T * 1)(T(20, 0, 32, 48, 64, 8))
    assert L.qlora_adamw_step(mis, 1, *args, 1, None) == 3
