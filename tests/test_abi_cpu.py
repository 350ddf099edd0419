"""The C-ABI library loads, exports every declared symbol, and rejects bad
arguments on the host (no GPU needed: validation happens before any launch)."""

import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    names = []
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names += re.findall(r"^\s*(?:const\s+)?[\w]+\s*\*?\s*(wise_\w+)\s*\(", src, flags=re.M)
    return sorted(set(names))


@pytest.fixture(scope="module")
def lib():
    from recurrent_depth_lm_b200 import _lib
    return _lib


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert len(names) >= 9, names
    raw = ctypes.CDLL(lib.LIB_PATH)
    for n in names:
        assert hasattr(raw, n), n
    assert set(names) == set(lib._SIGNATURES), "binding and header disagree"


def test_version(lib):
    assert "sm_100a" in lib.version()


def shape(lib, b=1, h=2, n=256, d=64, s=0.0):
    return lib.WiseShape(b, h, n, d, s)


@pytest.mark.parametrize("b,h,n,d", [(0, 1, 256, 64), (1, 0, 256, 64), (1, 1, 100, 64),
                                     (1, 1, 0, 64), (1, 1, 32768, 64), (1, 1, 256, 80),
                                     (1, 1, 256, 256)])
def test_bad_shapes_rejected(lib, b, h, n, d):
    L = lib.lib
    fake = 1 << 20
    rc = L.wise_full_attn_mass(fake, fake, fake, fake, None, None, None, 0, shape(lib, b, h, n, d),
                               None)
    assert rc == lib.WISE_ERR_SHAPE, lib.last_error()
    rc = L.wise_sparse_attn(fake, fake, fake, fake, fake, fake, 1, None, shape(lib, b, h, n, d), None)
    assert rc == lib.WISE_ERR_SHAPE
    assert L.wise_schedule_max_nnz(shape(lib, b, h, n, d)) == -1


def test_shape_struct_matches_header(lib):
    """The ctypes mirror of wise_shape_t has the header's fields, in order."""
    src = open(os.path.join(ROOT, "include", "wise.h")).read()
    body = re.search(r"typedef struct wise_shape \{(.*?)\} wise_shape_t;", src, flags=re.S).group(1)
    body = re.sub(r"/\*.*?\*/", "", body, flags=re.S)
    fields = re.findall(r"(?:int32_t|float)\s+(\w+);", body)
    assert fields == [f[0] for f in lib.WiseShape._fields_]
    assert ctypes.sizeof(lib.WiseShape) == 4 * len(fields)


@pytest.mark.parametrize("h,kv", [(6, 4), (8, 3), (4, -1)])
def test_kv_heads_must_divide_heads(lib, h, kv):
    L = lib.lib
    fake = 1 << 20
    s = lib.WiseShape(1, h, 256, 64, 0.0, kv)
    assert L.wise_full_attn_mass(fake, fake, fake, fake, None, None, None, 0, s, None) == \
        lib.WISE_ERR_SHAPE
    assert "kv_heads" in lib.last_error()
    assert L.wise_sparse_attn(fake, fake, fake, fake, fake, fake, 1, None, s, None) == \
        lib.WISE_ERR_SHAPE


def test_null_and_alignment_rejected(lib):
    L = lib.lib
    s = shape(lib)
    assert L.wise_full_attn_mass(None, 16, 16, 16, None, None, None, 0, s, None) == lib.WISE_ERR_ARG
    # mass without lse
    assert L.wise_full_attn_mass(16, 16, 16, 16, None, 16, None, 0, s, None) == lib.WISE_ERR_ARG
    assert L.wise_full_attn_mass(18, 16, 16, 16, None, None, None, 0, s, None) == lib.WISE_ERR_ALIGN
    # workspace given but too small
    assert L.wise_full_attn_mass(16, 16, 16, 16, 16, 16, 16, 8, s, None) == lib.WISE_ERR_WORKSPACE
    assert L.wise_mass_workspace_bytes(s) == 1 * 2 * 8 * 256 * 4
    assert L.wise_sparse_attn(16, 16, 16, 16, None, 16, 1, None, s, None) == lib.WISE_ERR_ARG
    assert L.wise_sparse_attn(16, 16, 16, 16, 16, 16, -1, None, s, None) == lib.WISE_ERR_ARG
    assert L.wise_sparse_attn(16, 16, 24, 16, 16, 16, 1, None, s, None) == lib.WISE_ERR_ALIGN
    assert L.wise_select_union(None, 16, None, 0.95, s, None) == lib.WISE_ERR_ARG
    assert L.wise_select_union(16, 16, None, 0.0, s, None) == lib.WISE_ERR_ARG
    assert L.wise_select_union(16, 16, None, float("nan"), s, None) == lib.WISE_ERR_ARG
    assert "eta" in lib.last_error()


def test_full_attn_mass_b16_checks(lib):
    L = lib.lib
    s = shape(lib)
    a, ws = 1 << 20, L.wise_mass_b16_workspace_bytes(s)
    assert ws == 2 * L.wise_mass_workspace_bytes(s)
    args = [a, a, a, a, a, a, a, ws]
    for i in range(7):                          # q k v o lse mass16 workspace
        bad = list(args)
        bad[i] = None
        assert L.wise_full_attn_mass_b16(*bad, s, None) == lib.WISE_ERR_ARG, i
    for i in (0, 3, 4, 5, 6):
        bad = list(args)
        bad[i] = a + 4
        assert L.wise_full_attn_mass_b16(*bad, s, None) == lib.WISE_ERR_ALIGN, i
    bad = list(args)
    bad[7] = ws - 16
    assert L.wise_full_attn_mass_b16(*bad, s, None) == lib.WISE_ERR_WORKSPACE
    assert L.wise_full_attn_mass_b16(*args, lib.WiseShape(1, 2, 100, 64, 0.0, 0), None) == \
        lib.WISE_ERR_SHAPE


def test_window_step_checks(lib):
    """wise_window_step validates before enqueueing anything: every pointer but step_bits is
    required, eta must be > 0, buffers 16-byte aligned, the workspace large enough."""
    L = lib.lib
    s = shape(lib)
    a, ws = 1 << 20, L.wise_mass_workspace_bytes(s)
    args = [a, a, a, a, a, a, a, None, 0.95, a, ws]
    assert L.wise_window_step(*args, lib.WiseShape(1, 2, 100, 64, 0.0, 0), None) == \
        lib.WISE_ERR_SHAPE
    for i in (0, 1, 2, 3, 4, 5, 6, 9):          # q k v o lse mass union workspace
        bad = list(args)
        bad[i] = None
        assert L.wise_window_step(*bad, s, None) == lib.WISE_ERR_ARG, i
    for eta in (0.0, -0.5, float("nan")):
        bad = list(args)
        bad[8] = eta
        assert L.wise_window_step(*bad, s, None) == lib.WISE_ERR_ARG
    assert "eta" in lib.last_error()
    for i in (0, 3, 4, 5, 9):                  # q, o, lse, mass, workspace misaligned
        bad = list(args)
        bad[i] = a + 4
        assert L.wise_window_step(*bad, s, None) == lib.WISE_ERR_ALIGN, i
    bad = list(args)
    bad[10] = ws - 16
    assert L.wise_window_step(*bad, s, None) == lib.WISE_ERR_WORKSPACE



def test_select_blocks_checks(lib):
    L = lib.lib
    s = shape(lib)
    fake = 1 << 20
    assert L.wise_select_union_blocks(None, fake, None, 0.95, 64, s, None) == lib.WISE_ERR_ARG
    assert L.wise_select_union_blocks(fake, fake, None, -1.0, 64, s, None) == lib.WISE_ERR_ARG
    for bad in (0, 16, 48, 96, 256):
        assert L.wise_select_union_blocks(fake, fake, None, 0.95, bad, s, None) == \
            lib.WISE_ERR_ARG
        assert "block" in lib.last_error()
    odd = lib.WiseShape(1, 2, 96, 64, 0.0, 0)       # 3 blocks of 32: not a multiple of 64
    assert L.wise_select_union_blocks(fake, fake, None, 0.95, 64, odd, None) == lib.WISE_ERR_SHAPE
    odd = lib.WiseShape(1, 2, 192, 64, 0.0, 0)      # 6 blocks of 32: not a multiple of 128
    assert L.wise_select_union_blocks(fake, fake, None, 0.95, 128, odd, None) == \
        lib.WISE_ERR_SHAPE


def test_control_and_support_mass_checks(lib):
    L = lib.lib
    s = shape(lib)
    a, b = 1 << 20, 1 << 21
    for fn in (L.wise_select_size_matched, L.wise_select_mass_matched):
        assert fn(None, a, b, s, None) == lib.WISE_ERR_ARG
        assert fn(a, None, b, s, None) == lib.WISE_ERR_ARG
        assert fn(a, b, None, s, None) == lib.WISE_ERR_ARG
        assert fn(a, b, b, s, None) == lib.WISE_ERR_ARG          # out aliases ref
        assert "alias" in lib.last_error()
        assert fn(a, b, a + 64, lib.WiseShape(1, 2, 100, 64, 0.0, 0), None) == lib.WISE_ERR_SHAPE
    assert L.wise_support_mass(None, a, b, s, None) == lib.WISE_ERR_ARG
    assert L.wise_support_mass(a, b, None, s, None) == lib.WISE_ERR_ARG
    assert L.wise_support_mass(a, b, a + 64, lib.WiseShape(1, 2, 256, 80, 0.0, 0), None) == \
        lib.WISE_ERR_SHAPE


def test_block16_checks(lib):
    L = lib.lib
    s = shape(lib)
    a = 1 << 20
    assert L.wise_block_mass_b16(None, a, a, a, s, None) == lib.WISE_ERR_ARG
    assert L.wise_block_mass_b16(a, a, None, a, s, None) == lib.WISE_ERR_ARG
    assert L.wise_block_mass_b16(a + 8, a, a, a, s, None) == lib.WISE_ERR_ALIGN
    assert L.wise_select_union_b16(None, a, None, 0.95, s, None) == lib.WISE_ERR_ARG
    assert L.wise_select_union_b16(a, a, None, 0.0, s, None) == lib.WISE_ERR_ARG
    ws = L.wise_schedule_b16_workspace_bytes(s)
    assert ws > L.wise_schedule_workspace_bytes(s)      # plus the folded 32-token masks
    assert L.wise_build_schedule_b16(a, a, a, None, 10, None, a, ws, s, None) == lib.WISE_ERR_ARG
    assert L.wise_build_schedule_b16(a, a, a, a, 10, None, a, ws - 1, s, None) == \
        lib.WISE_ERR_WORKSPACE
    assert L.wise_build_schedule_b16(a, a, a, a, 1, None, a, ws, s, None) == lib.WISE_ERR_CAPACITY
    assert L.wise_sparse_attn_b16(a, a, a, a, a, a, None, 1, None, s, None) == lib.WISE_ERR_ARG
    assert L.wise_sparse_attn_b16(a, a, a, a, a, a, a, -1, None, s, None) == lib.WISE_ERR_ARG
    assert L.wise_sparse_attn_b16(a, a, a + 4, a, a, a, a, 1, None, s, None) == lib.WISE_ERR_ALIGN

def test_schedule_sizes_and_checks(lib):
    L = lib.lib
    s = shape(lib, 1, 32, 4096, 128)
    assert L.wise_schedule_max_nnz(s) == 32 * 128 * 129 // 2
    ws = L.wise_schedule_workspace_bytes(s)
    assert ws >= 4 * ((32 * 128 + 1023) // 1024)
    # workspace missing / too small
    rc = L.wise_build_schedule(16, 16, 16, 10 ** 9, None, None, 0, s, None)
    assert rc == lib.WISE_ERR_WORKSPACE
    # capacity below the worst case without nnz_out
    rc = L.wise_build_schedule(16, 16, 16, 10, None, 16, ws, s, None)
    assert rc == lib.WISE_ERR_CAPACITY
    assert L.wise_build_schedule(None, 16, 16, 10, None, 16, ws, s, None) == lib.WISE_ERR_ARG


def test_last_error_is_thread_local(lib):
    import threading
    L = lib.lib
    L.wise_select_union(None, None, None, 0.5, shape(lib), None)
    seen = {}

    def other():
        seen["msg"] = lib.last_error()

    t = threading.Thread(target=other)
    t.start()
    t.join()
    assert seen["msg"] == ""
    assert lib.last_error() != ""


def test_header_is_plain_c_and_links(tmp_path):
    """include/wise.h compiles as C99 (no C++ or torch types), and a C program linked
    against libwise.so calls it: version string, a shape error with its message."""
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    pkg = os.path.join(ROOT, "recurrent_depth_lm_b200")
    src = tmp_path / "use_wise.c"
    src.write_text(r'''
#include <stdio.h>
#include <string.h>
#include "wise.h"
int main(void) {
  wise_shape_t s;
  memset(&s, 0, sizeof s);
  s.batch = 1; s.heads = 2; s.seqlen = 100; s.head_dim = 64;   /* seqlen not a multiple of 32 */
  int rc = wise_select_union((const float*)0x1000, (uint32_t*)0x1000, NULL, 0.95f, s, NULL);
  printf("%s|%d|%s\n", wise_version(), rc, wise_last_error());
  return rc == WISE_ERR_SHAPE ? 0 : 1;
}
''')
    exe = tmp_path / "use_wise"
    subprocess.run([cc, "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                    str(src), "-L", pkg, "-lwise", "-Wl,-rpath," + pkg, "-o", str(exe)],
                   check=True, capture_output=True, text=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True)
    assert out.returncode == 0, out.stdout + out.stderr
    version, rc, msg = out.stdout.strip().split("|")
    assert version and int(rc) < 0 and "seqlen" in msg
