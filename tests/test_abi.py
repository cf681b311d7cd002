"""The C-ABI library loads, exports what include/w4.h declares, and refuses bad
arguments before touching a device (CPU only: no compute calls here)."""

import ctypes as C
import os
import re
import subprocess

import numpy as np
import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "w4.h")


def _lib():
    from int8_weight_quantized_w4_b200 import _lib as L
    if not os.path.exists(L.LIB_PATH):
        from int8_weight_quantized_w4_b200 import build
        build.build(quiet=True)
    return L.load()


def declared_functions():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"^W4_API\s+[\w\s\*]+?\b(\w+)\(", src, flags=re.M)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for must in ("w4_matmul", "i8_head_logits", "w4_matmul_grouped", "w4_pack_nibbles", "w4_unpack_nibbles",
                 "w4_status_string", "w4_device_error"):
        assert must in names


def test_library_exports_every_declared_symbol():
    lib = _lib()
    from int8_weight_quantized_w4_b200 import _lib as L
    out = subprocess.run(["nm", "-D", "--defined-only", L.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r" T (\w+)$", out, flags=re.M))
    for name in declared_functions():
        assert name in exported, name
        assert getattr(lib, name) is not None
        assert name in L.SIGNATURES, f"binding lacks {name}"


def test_abi_version_and_status_strings():
    lib = _lib()
    from int8_weight_quantized_w4_b200 import _lib as L
    assert lib.w4_abi_version() == L.ABI_VERSION == 6
    assert lib.w4_status_string(0) == b"W4_OK"
    assert lib.w4_status_string(6) == b"W4_ERR_TIMEOUT"
    assert lib.w4_status_string(99) == b"W4_ERR_UNKNOWN"


def test_host_pack_unpack_exhaustive_against_oracle():
    from int8_weight_quantized_w4_b200 import pack_nibbles, unpack_nibbles
    allb = np.arange(256, dtype=np.uint8)
    assert np.array_equal(unpack_nibbles(allb, 512), oracle.unpack_nibbles(allb, 512))
    pairs = np.array([(lo, hi) for hi in range(16) for lo in range(16)], np.uint8).reshape(-1)
    assert np.array_equal(pack_nibbles(pairs), oracle.pack_nibbles(pairs))
    odd = np.arange(15, dtype=np.uint8)
    assert np.array_equal(pack_nibbles(odd), oracle.pack_nibbles(odd))
    assert list(unpack_nibbles(np.array([0x21], np.uint8), 2)) == [1, 2]


def test_host_pack_rejects_values_above_15():
    from int8_weight_quantized_w4_b200 import W4Error, pack_nibbles
    with pytest.raises(W4Error) as e:
        pack_nibbles(np.array([1, 16], np.uint8))
    assert e.value.status == 8


def _matmul(lib, x=0x1000, ldx=64, qw=0x2000, sc=0x3000, zp=0x4000, y=0x5000, ldy=64, M=1, K=64, N=64,
            path=0):
    return lib.w4_matmul_path(x, ldx, qw, sc, zp, y, ldy, M, K, N, None, 0, path, None)


@pytest.mark.parametrize("kw,status", [
    (dict(K=33), 2), (dict(K=-32), 2), (dict(N=63), 2), (dict(M=-1), 2),
    (dict(ldx=32), 2), (dict(ldy=32), 2),
    (dict(y=0), 1), (dict(qw=0), 1), (dict(x=0), 1), (dict(zp=0), 1), (dict(sc=0), 1),
    (dict(qw=0x2008), 3), (dict(sc=0x3004), 3), (dict(zp=0x4001), 3), (dict(x=0x1002), 3), (dict(y=0x5001), 3),
    (dict(path=7), 8),
])
def test_matmul_argument_errors_before_any_launch(kw, status):
    lib = _lib()
    assert _matmul(lib, **kw) == status
    assert lib.w4_last_error()  # a reason is recorded


def test_matmul_noops_need_no_device():
    lib = _lib()
    assert _matmul(lib, M=0) == 0
    assert _matmul(lib, N=0) == 0
    assert _matmul(lib, M=0, x=0, qw=0, sc=0, zp=0, y=0) == 0


@pytest.mark.parametrize("kw,status", [
    (dict(K=-1), 2), (dict(ldl=10), 2), (dict(ldt=10), 2), (dict(ldh=10), 2),
    (dict(table=0x2001), 3), (dict(h=0x1002), 3), (dict(logits=0), 1), (dict(table=0), 1),
])
def test_head_argument_errors(kw, status):
    lib = _lib()
    a = dict(h=0x1000, ldh=32, table=0x2000, ldt=20, scales=0x3000, logits=0x4000, ldl=20, M=1, K=32, V=20)
    a.update(kw)
    st = lib.i8_head_logits(a["h"], a["ldh"], a["table"], a["ldt"], a["scales"], a["logits"], a["ldl"], a["M"],
                            a["K"], a["V"], None, 0, None)
    assert st == status


def test_grouped_argument_errors():
    lib = _lib()
    from int8_weight_quantized_w4_b200._lib import W4Desc
    d = (W4Desc * 2)()
    d[0] = W4Desc(0x1000, 64, 0x2000, 0x3000, 0x4000, 0x5000, 64, 1, 64, 64)
    d[1] = W4Desc(0x1000, 64, 0x2000, 0x3000, 0x4000, 0x5000, 64, 1, 40, 64)
    assert lib.w4_matmul_grouped(d, 2, None, 0, None) == 2
    assert b"descriptor 1" in lib.w4_last_error()
    assert lib.w4_matmul_grouped(d, 0, None, 0, None) == 0
    assert lib.w4_matmul_grouped(None, 3, None, 0, None) == 1


def test_desc_layout_matches_the_c_struct(tmp_path):
    """The ctypes descriptor has the C struct's size and field offsets."""
    from int8_weight_quantized_w4_b200._lib import W4Desc
    src = tmp_path / "layout.c"
    src.write_text('#include <stddef.h>\n#include <stdio.h>\n#include "w4.h"\n'
                   'int main(void) { printf("%zu %zu %zu %zu %zu %zu\\n", sizeof(w4_desc), offsetof(w4_desc, N), '
                   'offsetof(w4_desc, bias), offsetof(w4_desc, residual), offsetof(w4_desc, ldr), '
                   'offsetof(w4_desc, act)); return 0; }\n')
    exe = tmp_path / "layout"
    subprocess.run(["gcc", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)], check=True)
    got = [int(v) for v in subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.split()]
    want = [C.sizeof(W4Desc), W4Desc.N.offset, W4Desc.bias.offset, W4Desc.residual.offset, W4Desc.ldr.offset,
            W4Desc.act.offset]
    assert got == want


def _desc(**kw):
    from int8_weight_quantized_w4_b200._lib import W4Desc
    a = dict(x=0x1000, ldx=64, qw=0x2000, scales=0x3000, zp=0x4000, y=0x5000, ldy=64, M=1, K=64, N=64, bias=0,
             residual=0, ldr=0, act=0, reserved=0)
    a.update(kw)
    return W4Desc(**a)


@pytest.mark.parametrize("kw,status", [
    (dict(act=3), 8), (dict(act=-1), 8), (dict(reserved=1), 8),
    (dict(bias=0x6002), 3), (dict(residual=0x7002, ldr=64), 3),
    (dict(residual=0x7000, ldr=32), 2), (dict(residual=0x5000, ldr=128), 2),
    (dict(K=40), 2), (dict(y=0), 1),
])
def test_epilogue_argument_errors_before_any_launch(kw, status):
    lib = _lib()
    d = _desc(**kw)
    assert lib.w4_matmul_desc(C.byref(d), None, 0, 0, None) == status
    assert lib.w4_last_error()
    g = (type(d) * 1)(d)
    assert lib.w4_matmul_grouped(g, 1, None, 0, None) == status


def test_epilogue_noops_need_no_device():
    lib = _lib()
    assert lib.w4_matmul_desc(C.byref(_desc(M=0, act=1, bias=0x6000)), None, 0, 0, None) == 0
    assert lib.w4_matmul_desc(None, None, 0, 0, None) == 1


@pytest.mark.parametrize("kw,status", [
    (dict(block=48), 8), (dict(block=0), 8), (dict(st=2), 8), (dict(K=96, block=64), 2), (dict(N=63), 2),
    (dict(ldw=32), 2), (dict(w=0), 1), (dict(qw=0), 1), (dict(w=0x1002), 3), (dict(sc=0x3002), 3),
    (dict(sc=0x3001, st=1), 3), (dict(K=-64), 2),
])
def test_quantize_argument_errors_before_any_launch(kw, status):
    lib = _lib()
    a = dict(w=0x1000, ldw=64, K=128, N=64, block=32, st=0, qw=0x2000, sc=0x3000, zp=0x4000)
    a.update(kw)
    assert lib.w4_quantize(a["w"], a["ldw"], a["K"], a["N"], a["block"], a["st"], a["qw"], a["sc"], a["zp"],
                           None) == status
    assert lib.w4_last_error()


def test_quantize_head_argument_errors_before_any_launch():
    lib = _lib()
    assert lib.i8_quantize_head(0x1000, 10, 8, 20, 0x2000, 20, 0x3000, None) == 2   # ldw < V
    assert lib.i8_quantize_head(0x1000, 20, 8, 20, 0x2000, 10, 0x3000, None) == 2   # ldt < V
    assert lib.i8_quantize_head(0x1002, 20, 8, 20, 0x2000, 20, 0x3000, None) == 3
    assert lib.i8_quantize_head(0x1000, 20, 8, 20, 0x2000, 20, 0, None) == 1
    assert lib.i8_quantize_head(0x1000, 20, 8, 0, 0x2000, 20, 0x3000, None) == 0    # V = 0: nothing to do


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    from int8_weight_quantized_w4_b200 import _lib as L
    monkeypatch.setattr(L, "LIB_PATH", str(tmp_path / "nope.so"))
    monkeypatch.setattr(L, "_lib", None)
    with pytest.raises(L.W4LibraryMissing):
        L.load()


# ---------------------------------------------------------------- streaming layout

def test_repacked_bytes_is_the_page_format_total():
    lib = _lib()
    import math
    for K, N in [(768, 768), (768, 2304), (3072, 768), (8192, 3072), (32, 256), (96, 768)]:
        nb = K // 32
        gs = 32 // math.gcd(nb, 32)
        assert N % (8 * gs) == 0
        assert lib.w4_repacked_bytes(K, N) == K * N // 2 + nb * N * 4 + nb * N // 2
    # a last group that is only partly filled is padded to whole strips of the group
    assert lib.w4_repacked_bytes(768, 200) == 7 * 3 * 5248
    for K, N in [(33, 64), (64, 60), (0, 64), (64, 0), (-32, 64)]:
        assert lib.w4_repacked_bytes(K, N) == 0


def _rdesc(**kw):
    from int8_weight_quantized_w4_b200._lib import W4RDesc
    a = dict(x=0x1000, ldx=64, wr=0x2000, y=0x5000, ldy=64, M=1, K=64, N=64, bias=0, residual=0, ldr=0, act=0,
             reserved=0)
    a.update(kw)
    return W4RDesc(**a)


@pytest.mark.parametrize("kw,status", [
    (dict(M=2), 2), (dict(N=60), 2), (dict(K=40), 2), (dict(K=14368), 2), (dict(M=-1), 2),
    (dict(x=0x1004), 3), (dict(wr=0x2008), 3), (dict(y=0x5002), 3), (dict(bias=0x6002), 3),
    (dict(x=0), 1), (dict(wr=0), 1), (dict(y=0), 1), (dict(act=5), 8), (dict(reserved=1), 8),
])
def test_w4r_argument_errors_before_any_launch(kw, status):
    lib = _lib()
    d = _rdesc(**kw)
    assert lib.w4r_matmul(C.byref(d), None) == status
    assert lib.w4_last_error()


def test_decode_step_argument_errors_before_any_launch():
    """The one-launch step checks its body descriptors, its head and the
    aliasing of h with the body's outputs on the host: every refusal here
    comes before the device is touched."""
    lib = _lib()
    from int8_weight_quantized_w4_b200._lib import W4RDesc
    good = (W4RDesc * 1)(_rdesc())
    h, tr, lg, K, V = 0x9000, 0xA000, 0xB000, 64, 100
    step = lib.w4r_decode_step
    assert step(good, 1, h, tr, K, V, 0, None) == 1          # logits NULL
    assert step(good, 1, h, tr, K, V, 0xB002, None) == 3     # logits misaligned
    assert step(good, 1, 0x9004, tr, K, V, lg, None) == 3    # h not 16-byte aligned
    assert step(good, 1, h, 0xA008, K, V, lg, None) == 3     # table not 16-byte aligned
    assert step(good, 1, h, tr, 72, V, lg, None) == 2        # head K % 16 != 0
    assert step(good, 1, 0, tr, K, V, lg, None) == 1         # h NULL
    assert step(good, -1, h, tr, K, V, lg, None) == 2        # negative count
    assert step(None, 1, h, tr, K, V, lg, None) == 1         # descs NULL
    bad = (W4RDesc * 1)(_rdesc(M=2))
    assert step(bad, 1, h, tr, K, V, lg, None) == 2          # a body descriptor's own check
    # h inside the body's output y (0x5000 .. 0x5100): refused
    assert step(good, 1, 0x5040, tr, K, V, lg, None) == 8
    assert b"overlaps" in lib.w4_last_error()
    argmax = lib.w4r_decode_step_argmax
    assert argmax(good, 1, h, tr, K, V, 0xC000, 0, 0, None) == 1        # keys NULL
    assert argmax(good, 1, h, tr, K, V, 0, 0, 0xD000, None) == 1        # token NULL
    assert argmax(good, 1, h, tr, K, V, 0xC000, 0, 0xD004, None) == 3   # keys misaligned


def test_w4r_noops_and_repack_shape_errors_need_no_device():
    lib = _lib()
    assert lib.w4r_matmul(C.byref(_rdesc(M=0)), None) == 0
    assert lib.w4r_matmul(C.byref(_rdesc(N=0, x=0, wr=0)), None) == 0
    assert lib.w4r_matmul(None, None) == 1
    assert lib.w4r_matmul_grouped(None, 0, None) == 0
    assert lib.w4_repack(0x1000, 0x2000, 0x3000, 64, 60, 0x4000, None) == 2
    assert lib.w4_repack(0x1000, 0x2000, 0x3000, 40, 64, 0x4000, None) == 2
    assert lib.w4_repack(0x1000, 0x2004, 0x3000, 64, 64, 0x4000, None) == 3
    assert lib.w4_repack(0, 0x2000, 0x3000, 64, 64, 0x4000, None) == 1
    assert lib.w4_repack_restore(0x4000, 64, 62, 0x1000, 0x2000, 0x3000, None) == 2


def test_rdesc_layout_matches_the_c_struct(tmp_path):
    from int8_weight_quantized_w4_b200._lib import W4RDesc
    src = tmp_path / "rlayout.c"
    src.write_text('#include <stddef.h>\n#include <stdio.h>\n#include "w4.h"\n'
                   'int main(void) { printf("%zu %zu %zu %zu %zu\\n", sizeof(w4r_desc), offsetof(w4r_desc, wr), '
                   'offsetof(w4r_desc, N), offsetof(w4r_desc, ldr), offsetof(w4r_desc, act)); return 0; }\n')
    exe = tmp_path / "rlayout"
    subprocess.run(["gcc", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)], check=True)
    got = [int(v) for v in subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.split()]
    assert got == [C.sizeof(W4RDesc), W4RDesc.wr.offset, W4RDesc.N.offset, W4RDesc.ldr.offset, W4RDesc.act.offset]
