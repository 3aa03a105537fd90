"""The C-ABI library: it loads, exports every symbol include/qlora.h declares,
derives the same fp32 NF4 codebook as the oracle, and rejects bad arguments
on the host before any launch.  No GPU is touched: every call here returns
before the library's first CUDA call (fake device pointers are never
dereferenced)."""
import ctypes
import os
import re
import subprocess

import numpy as np
import pytest

from bit_nf4_quantized_qlora_b200 import binding as B
from oracle import codebooks, nf4

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER_DIR = os.path.join(ROOT, "include")


def _declared_functions():
    names = set()
    for fn in os.listdir(HEADER_DIR):
        if not fn.endswith(".h"):
            continue
        text = open(os.path.join(HEADER_DIR, fn)).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        for m in re.finditer(r"^\s*(?:const\s+)?[A-Za-z_][\w\s\*]*?\b(qlora_\w+)\s*\(", text, flags=re.M):
            names.add(m.group(1))
    return sorted(names)


@pytest.fixture(scope="module")
def lib():
    return B.lib()


def test_header_declares_the_five_entry_points():
    names = _declared_functions()
    for n in ("qlora_quantize_nf4_dq", "qlora_dequant", "qlora_linear_fwd", "qlora_linear_bwd_dx",
              "qlora_lora_bwd", "qlora_workspace_bytes"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    names = _declared_functions()
    assert len(names) >= 10
    out = subprocess.run(["nm", "-D", "--defined-only", B.LIB_PATH], capture_output=True, text=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    for n in names:
        assert n in exported, n
        assert hasattr(lib, n)


@pytest.mark.parametrize("name", ["nf4", "fp4", "int4"])
def test_library_baseline_codebooks_equal_the_oracle(lib, name):
    """The library builds each codebook with its own code (FP4 by decoding the
    e2m1 bit patterns); levels equal the oracle's bit for bit, -0 included."""
    got = np.array(B.qlora_codebook_levels(B.CODEBOOKS[name]), dtype=np.float32)
    assert np.array_equal(got.view(np.uint32), codebooks.levels_f32(name).view(np.uint32))


def test_unknown_codebook_is_rejected_on_the_host(lib):
    buf = (ctypes.c_float * 16)()
    assert lib.qlora_codebook_levels(3, buf) == B.QLORA_ERR_CODEBOOK
    assert lib.qlora_codebook_levels(-1, buf) == B.QLORA_ERR_CODEBOOK
    assert lib.qlora_quantize_4bit_dq(P, 64, 64, 3, P, P, P, None, None) == B.QLORA_ERR_CODEBOOK
    w = _w()
    w.codebook = 7
    assert lib.qlora_dequant(ctypes.byref(w), P, None) == B.QLORA_ERR_CODEBOOK
    assert _fwd(lib, w=w) == B.QLORA_ERR_CODEBOOK


def test_merge_rejects_bad_arguments(lib):
    w = _w()
    f = lib.qlora_merge_adapter
    assert f(ctypes.byref(w), P, P, 16, 2.0, None, None, None) == B.QLORA_ERR_NULL       # no output
    assert f(ctypes.byref(w), P, P, 16, 2.0, MIS, None, None) == B.QLORA_ERR_ALIGN
    assert f(ctypes.byref(w), P, P, 16, 2.0, None, MIS, None) == B.QLORA_ERR_ALIGN
    assert f(ctypes.byref(w), P, P, 24, 2.0, P, None, None) == B.QLORA_ERR_SHAPE         # r % 16
    assert f(ctypes.byref(w), P, P, 272, 2.0, P, None, None) == B.QLORA_ERR_SHAPE        # r > 256
    assert f(ctypes.byref(w), P, None, 16, 2.0, P, None, None) == B.QLORA_ERR_NULL       # half an adapter
    assert f(ctypes.byref(w), MIS, P, 16, 2.0, P, None, None) == B.QLORA_ERR_ALIGN
    assert f(ctypes.byref(_w(k=1000)), P, P, 16, 2.0, P, None, None) == B.QLORA_ERR_SHAPE
    w.codebook = 5
    assert f(ctypes.byref(w), P, P, 16, 2.0, P, None, None) == B.QLORA_ERR_CODEBOOK
    w.codebook = 0
    w.dq_format = 2
    assert f(ctypes.byref(w), P, P, 16, 2.0, P, None, None) == B.QLORA_ERR_FORMAT


def test_weight_struct_layout():
    """Three pointers and two int64 sizes (40 bytes), then block, group,
    codebook and dq_format (int32): 56 bytes, the size the struct had before
    dq_format took its tail padding.  Zeroed codebook and dq_format fields
    mean NF4 with linear 8-bit absmax codes."""
    assert ctypes.sizeof(B.NF4WeightC) == 56
    assert B.NF4WeightC.codebook.offset == 48
    assert B.NF4WeightC.dq_format.offset == 52
    w = B.NF4WeightC(0, 0, 0, 1, 64, 64, 256)
    assert w.codebook == B.QLORA_CODEBOOK_NF4 and w.dq_format == B.QLORA_DQ_LINEAR8


def test_library_codebook_equals_oracle_codebook(lib):
    """The library derives its levels with its own inverse-normal routine; the
    fp32 values must equal the oracle's bit for bit."""
    got = np.array(B.qlora_nf4_levels(), dtype=np.float32)
    assert np.array_equal(got.view(np.uint32), nf4.levels_f32().view(np.uint32))


def test_version_and_status_strings(lib):
    assert lib.qlora_version() >> 16 == 1
    for st in (0, -1, -2, -3, -4, -5, -6, -7, -8):
        assert lib.qlora_status_string(st)
    assert b"FORMAT" in lib.qlora_status_string(B.QLORA_ERR_FORMAT)


def test_workspace_bytes(lib):
    f = B.qlora_workspace_bytes
    assert f(B.QLORA_OP_FWD, 4096, 11008, 4096, 0) == 0
    assert f(B.QLORA_OP_FWD, 4096, 11008, 4096, 64) == 4096 * 64 * 2
    assert f(B.QLORA_OP_FWD, 3, 1024, 1024, 16) == 256          # rounded up to 256 B
    assert f(B.QLORA_OP_BWD_DX, 16, 1024, 1024, 16) == 512
    # U and T (2 x 512 B), then the fp32 partials of the one-pass adapter
    # products for r <= 64: U of each n-range (here 8 ranges of one 128-column
    # block: the split that gives the busiest CTA the fewest stages) and dB of
    # each m-slice (one: m fits one 128-row block).
    assert f(B.QLORA_OP_LORA_BWD, 16, 1024, 1024, 16) == 1024 + 8 * 16 * 16 * 4 + 1 * 1024 * 16 * 4
    # r > 64 keeps the separate products: U and T only.
    assert f(B.QLORA_OP_LORA_BWD, 16, 1024, 1024, 128) == 2 * 16 * 128 * 2
    assert f(99, 1, 1, 1, 1) == 2 ** 64 - 1
    assert f(B.QLORA_OP_FWD, -1, 1, 1, 1) == 2 ** 64 - 1


# ---- host-side validation (fake, aligned device addresses) -----------------

P = 0x10000000          # a 16-byte aligned fake address, never dereferenced
MIS = P + 8             # misaligned


def _w(n=1024, k=1024, codes=P, q=P, s=P, block=64, group=256):
    return B.NF4WeightC(codes, q, s, n, k, block, group)


def _fwd(lib, X=P, m=16, w=None, A=P, Bm=P, r=16, Y=P, ws=P, ws_bytes=1 << 20):
    w = w if w is not None else _w()
    return lib.qlora_linear_fwd(X, m, ctypes.byref(w), A, Bm, r, 2.0, Y, ws, ws_bytes, None)


def test_fwd_rejects_bad_arguments(lib):
    assert _fwd(lib, X=None) == B.QLORA_ERR_NULL
    assert _fwd(lib, Y=None) == B.QLORA_ERR_NULL
    assert _fwd(lib, w=_w(codes=0)) == B.QLORA_ERR_NULL
    assert _fwd(lib, w=_w(k=1000)) == B.QLORA_ERR_SHAPE           # k % 64
    assert _fwd(lib, w=_w(n=1020)) == B.QLORA_ERR_SHAPE           # n % 8
    assert _fwd(lib, w=_w(n=0)) == B.QLORA_ERR_SHAPE
    assert _fwd(lib, w=_w(block=32)) == B.QLORA_ERR_SHAPE
    assert _fwd(lib, w=_w(group=128)) == B.QLORA_ERR_SHAPE
    assert _fwd(lib, r=12) == B.QLORA_ERR_SHAPE                    # r % 16
    assert _fwd(lib, r=-16) == B.QLORA_ERR_SHAPE
    assert _fwd(lib, m=-1) == B.QLORA_ERR_SHAPE
    assert _fwd(lib, A=None) == B.QLORA_ERR_NULL                   # one adapter pointer
    assert _fwd(lib, X=MIS) == B.QLORA_ERR_ALIGN
    assert _fwd(lib, Y=MIS) == B.QLORA_ERR_ALIGN
    assert _fwd(lib, A=MIS) == B.QLORA_ERR_ALIGN
    assert _fwd(lib, w=_w(codes=MIS)) == B.QLORA_ERR_ALIGN
    assert _fwd(lib, ws=None) == B.QLORA_ERR_WORKSPACE
    assert _fwd(lib, ws_bytes=16 * 16 * 2 - 1) == B.QLORA_ERR_WORKSPACE
    assert _fwd(lib, ws=MIS) == B.QLORA_ERR_ALIGN


def test_fwd_empty_batch_is_a_no_op(lib):
    assert _fwd(lib, m=0, X=None, Y=None, ws=None) == B.QLORA_OK


def test_bwd_dx_rejects_bad_arguments(lib):
    w = _w()
    f = lambda **kw: lib.qlora_linear_bwd_dx(kw.get("dY", P), kw.get("m", 16), ctypes.byref(kw.get("w", w)),
                                             kw.get("A", P), kw.get("B", P), kw.get("r", 16), 2.0,
                                             kw.get("dX", P), kw.get("ws", P), kw.get("ws_bytes", 1 << 20), None)
    assert f(dY=None) == B.QLORA_ERR_NULL
    assert f(dX=MIS) == B.QLORA_ERR_ALIGN
    assert f(w=_w(k=96)) == B.QLORA_ERR_SHAPE
    assert f(ws_bytes=10) == B.QLORA_ERR_WORKSPACE
    assert f(m=0, dY=None, dX=None) == B.QLORA_OK


def test_lora_bwd_rejects_bad_arguments(lib):
    f = lambda **kw: lib.qlora_lora_bwd(kw.get("X", P), kw.get("dY", P), kw.get("m", 16), kw.get("n", 1024),
                                        kw.get("k", 1024), kw.get("A", P), kw.get("B", P), kw.get("r", 16), 2.0,
                                        kw.get("dA", P), kw.get("dB", P), kw.get("ws", P),
                                        kw.get("ws_bytes", 1 << 20), None)
    assert f(A=None) == B.QLORA_ERR_NULL
    assert f(dB=None) == B.QLORA_ERR_NULL
    assert f(X=None) == B.QLORA_ERR_NULL
    assert f(r=0) == B.QLORA_ERR_SHAPE
    assert f(k=100) == B.QLORA_ERR_SHAPE
    assert f(n=12) == B.QLORA_ERR_SHAPE
    assert f(dA=MIS) == B.QLORA_ERR_ALIGN
    assert f(ws=None) == B.QLORA_ERR_WORKSPACE
    assert f(ws_bytes=1023) == B.QLORA_ERR_WORKSPACE


def test_quantize_and_dequant_reject_bad_arguments(lib):
    q = lambda **kw: lib.qlora_quantize_nf4_dq(kw.get("W", P), kw.get("n", 64), kw.get("k", 64), kw.get("c", P),
                                               kw.get("q", P), kw.get("s", P), kw.get("a", None), None)
    assert q(W=None) == B.QLORA_ERR_NULL
    assert q(k=63) == B.QLORA_ERR_SHAPE
    assert q(n=0) == B.QLORA_ERR_SHAPE
    assert q(c=MIS) == B.QLORA_ERR_ALIGN
    assert q(a=MIS) == B.QLORA_ERR_ALIGN
    w = _w()
    assert lib.qlora_dequant(ctypes.byref(w), None, None) == B.QLORA_ERR_NULL
    assert lib.qlora_dequant(ctypes.byref(w), MIS, None) == B.QLORA_ERR_ALIGN
    w.dq_format = -1
    assert lib.qlora_dequant(ctypes.byref(w), P, None) == B.QLORA_ERR_FORMAT
    qf = lambda fmt, cb=0, W=P: lib.qlora_quantize_4bit_dq_format(W, 64, 64, cb, fmt, P, P, P, None, None)
    assert qf(2) == B.QLORA_ERR_FORMAT
    assert qf(-1) == B.QLORA_ERR_FORMAT
    assert qf(B.QLORA_DQ_FP8_MEAN, cb=9) == B.QLORA_ERR_CODEBOOK
    assert qf(B.QLORA_DQ_FP8_MEAN, W=None) == B.QLORA_ERR_NULL
    assert lib.qlora_dequant(None, P, None) == B.QLORA_ERR_NULL


def test_poll_rejects_null(lib):
    assert lib.qlora_poll_device_error(None, None) == B.QLORA_ERR_NULL


def _noalloc(lib, X=P, m=16, w=None, A=P, Bm=P, r=16, Y=P):
    w = w if w is not None else _w()
    return lib.qlora_linear_fwd_noalloc(X, m, ctypes.byref(w), A, Bm, r, 2.0, Y, None)


def test_noalloc_reports_errors_in_the_order_of_the_workspace_forward(lib):
    """Every host-side check of the forward comes before the built-in
    scratch's size check, so a bad weight or a half adapter is reported as
    such even when m is too large for the scratch."""
    big = (1 << 20) // (2 * 256) + 1                                 # m * r * 2 beyond the scratch at r = 256
    assert _noalloc(lib, m=big, r=256, w=_w(k=1000)) == B.QLORA_ERR_SHAPE
    assert _noalloc(lib, m=big, r=256, A=None) == B.QLORA_ERR_NULL
    assert _noalloc(lib, m=big, r=256, w=_w(codes=0)) == B.QLORA_ERR_NULL
    assert _noalloc(lib, m=big, r=256, X=MIS) == B.QLORA_ERR_ALIGN
    assert _noalloc(lib, m=big, r=256) == B.QLORA_ERR_WORKSPACE
    for kw in (dict(X=None), dict(Y=MIS), dict(w=_w(n=1020)), dict(r=12), dict(m=-1), dict(A=MIS)):
        assert _noalloc(lib, **kw) == _fwd(lib, **kw), kw
    assert _noalloc(lib, m=0, X=None, Y=None) == B.QLORA_OK


def test_selftests_reject_bad_arguments(lib):
    assert lib.qlora_selftest_bounded_wait(0, None, None) == B.QLORA_ERR_SHAPE
    assert lib.qlora_selftest_bounded_wait(3_000_000_000, None, None) == B.QLORA_ERR_SHAPE
    assert lib.qlora_selftest_bounded_wait(1000, MIS + 1, None) == B.QLORA_ERR_ALIGN
    assert lib.qlora_selftest_div255(0x3F800000, 16, None, None) == B.QLORA_ERR_NULL
    assert lib.qlora_selftest_div255(0x3F800000, 16, P + 4, None) == B.QLORA_ERR_ALIGN
    assert lib.qlora_selftest_div255(0x3F800000, 0, P, None) == B.QLORA_ERR_SHAPE
    assert lib.qlora_selftest_div255(0x7F7FFFFF, 2, P, None) == B.QLORA_ERR_SHAPE    # would reach +inf


def test_device_error_bits_match_the_header():
    text = open(os.path.join(HEADER_DIR, "qlora.h")).read()
    for name in ("OPERANDS", "WEIGHT_TILE", "FREE_STAGE", "ACCUMULATOR", "DRAIN", "SELFTEST"):
        m = re.search(r"QLORA_DEVERR_%s\s*=\s*1u\s*<<\s*(\d+)" % name, text)
        assert m and getattr(B, "QLORA_DEVERR_" + name) == 1 << int(m.group(1)), name


def test_dropout_entry_points_reject_bad_arguments(lib):
    d = lambda **kw: lib.qlora_lora_dropout(kw.get("X", P), kw.get("m", 16), kw.get("k", 128), kw.get("p", 0.05),
                                            1, 2, kw.get("Xd", P), None)
    assert d(p=1.0) == B.QLORA_ERR_SHAPE
    assert d(p=-0.1) == B.QLORA_ERR_SHAPE
    assert d(p=float("nan")) == B.QLORA_ERR_SHAPE
    assert d(k=100) == B.QLORA_ERR_SHAPE
    assert d(X=None) == B.QLORA_ERR_NULL
    assert d(Xd=MIS) == B.QLORA_ERR_ALIGN
    assert d(m=0, X=None, Xd=None) == B.QLORA_OK
    w = _w()
    f = lambda **kw: lib.qlora_linear_fwd_dropout(kw.get("X", P), kw.get("m", 16), ctypes.byref(kw.get("w", w)),
                                                  kw.get("A", P), kw.get("B", P), kw.get("r", 16), 2.0,
                                                  kw.get("p", 0.05), 1, 2, kw.get("Xd", P), kw.get("Y", P),
                                                  kw.get("ws", P), kw.get("ws_bytes", 1 << 20), None)
    assert f(A=None, B=None) == B.QLORA_ERR_NULL                  # dropout needs an adapter
    assert f(r=0) == B.QLORA_ERR_SHAPE
    assert f(p=1.5) == B.QLORA_ERR_SHAPE
    assert f(Xd=None) == B.QLORA_ERR_NULL
    assert f(Xd=MIS) == B.QLORA_ERR_ALIGN
    assert f(ws=None) == B.QLORA_ERR_WORKSPACE
    assert f(w=_w(k=1000)) == B.QLORA_ERR_SHAPE
    g = lambda **kw: lib.qlora_linear_bwd_dx_dropout(kw.get("dY", P), kw.get("m", 16), ctypes.byref(kw.get("w", w)),
                                                     kw.get("A", P), kw.get("B", P), kw.get("r", 16), 2.0,
                                                     kw.get("p", 0.05), 1, 2, kw.get("dX", P), kw.get("ws", P),
                                                     kw.get("ws_bytes", 1 << 20), None)
    assert g(B=None) == B.QLORA_ERR_NULL
    assert g(p=1.0) == B.QLORA_ERR_SHAPE
    assert g(dX=MIS) == B.QLORA_ERR_ALIGN
    assert g(ws_bytes=10) == B.QLORA_ERR_WORKSPACE
    assert g(m=0, dY=None, dX=None) == B.QLORA_OK


def test_linear_bwd_rejects_bad_arguments(lib):
    w = _w()
    f = lambda **kw: lib.qlora_linear_bwd(kw.get("dY", P), kw.get("X", P), kw.get("T", None), kw.get("m", 16),
                                          ctypes.byref(kw.get("w", w)), kw.get("A", P), kw.get("B", P),
                                          kw.get("r", 16), 2.0, kw.get("dX", P), kw.get("dA", P), kw.get("dB", P),
                                          kw.get("ws", P), kw.get("ws_bytes", 1 << 20), None)
    assert f(A=None) == B.QLORA_ERR_NULL
    assert f(dB=None) == B.QLORA_ERR_NULL
    assert f(X=None) == B.QLORA_ERR_NULL
    assert f(r=0) == B.QLORA_ERR_SHAPE
    assert f(w=_w(k=1000)) == B.QLORA_ERR_SHAPE
    assert f(dX=MIS) == B.QLORA_ERR_ALIGN
    assert f(T=MIS) == B.QLORA_ERR_ALIGN
    assert f(ws=None) == B.QLORA_ERR_WORKSPACE
    assert f(ws_bytes=100) == B.QLORA_ERR_WORKSPACE
