"""wise_build_schedule_static: the schedule build for callers that cannot
allocate device memory (their device memory is owned by a host framework's
pool, or cudaMalloc is off-limits in their serving loop because it can
synchronise the device).  It must produce exactly what wise_build_schedule
produces with a caller-provided workspace.

This file is collected last on purpose (pytest orders files by name), so a
run that stops at the first failure has run every other test before it.
"""

import ctypes

import numpy as np
import pytest

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from recurrent_depth_lm_b200 import _lib
    return _lib


def _bits(bh, nq, seed):
    rng = np.random.default_rng(seed)
    w = rng.integers(0, 2 ** 32, size=(1, bh, nq, (nq + 31) // 32), dtype=np.uint64)
    return torch.from_numpy(w.astype(np.uint32).view(np.int32)).cuda()


def _with_workspace(lib, bits, shape, cap):
    rows = shape.batch * shape.heads * (shape.seqlen // 32)
    ro = torch.full((rows + 1,), -7, dtype=torch.int32, device="cuda")
    ci = torch.full((cap,), -7, dtype=torch.int32, device="cuda")
    ws = torch.empty(max(1, lib.lib.wise_schedule_workspace_bytes(shape)), dtype=torch.uint8,
                     device="cuda")
    nnz = ctypes.c_int64(-1)
    rc = lib.lib.wise_build_schedule(bits.data_ptr(), ro.data_ptr(), ci.data_ptr(), cap,
                                     ctypes.byref(nnz), ws.data_ptr(), ws.numel(), shape,
                                     torch.cuda.current_stream().cuda_stream)
    lib.check(rc, "wise_build_schedule")
    return ro, ci, nnz.value


def _static(lib, bits, shape, cap, with_nnz):
    rows = shape.batch * shape.heads * (shape.seqlen // 32)
    ro = torch.full((rows + 1,), -9, dtype=torch.int32, device="cuda")
    ci = torch.full((cap,), -9, dtype=torch.int32, device="cuda")
    nnz = ctypes.c_int64(-1)
    rc = lib.lib.wise_build_schedule_static(bits.data_ptr(), ro.data_ptr(), ci.data_ptr(), cap,
                                            ctypes.byref(nnz) if with_nnz else None, shape,
                                            torch.cuda.current_stream().cuda_stream)
    lib.check(rc, "wise_build_schedule_static")
    torch.cuda.synchronize()
    return ro, ci, (nnz.value if with_nnz else int(ro[-1].item()))


@pytest.mark.parametrize("bh,n", [(3, 1440), (32, 4096)])
def test_static_schedule_matches_workspace_version_twice(lib, bh, n):
    shape = lib.WiseShape(1, bh, n, 128, 0.0)
    cap = int(lib.lib.wise_schedule_max_nnz(shape))
    # two calls in a row on different inputs: the second must not see the first's scratch
    for call, seed in enumerate((11, 12)):
        bits = _bits(bh, n // 32, seed + bh)
        ro_ref, ci_ref, nnz_ref = _with_workspace(lib, bits, shape, cap)
        ro, ci, nnz = _static(lib, bits, shape, cap, with_nnz=(call == 0))
        assert nnz == nnz_ref
        assert torch.equal(ro, ro_ref)
        assert torch.equal(ci[:nnz], ci_ref[:nnz_ref])


def test_static_schedule_rejects_shapes_beyond_its_scratch(lib):
    # 64 * 32 heads * 512 query blocks = 1,048,576 rows is the limit; one more batch is too many
    shape = lib.WiseShape(65, 32, 16384, 128, 0.0)
    rc = lib.lib.wise_build_schedule_static(16, 16, 16, 1 << 40, None, shape, None)
    assert rc == lib.WISE_ERR_WORKSPACE
    assert "1048576" in lib.last_error()


def test_static_schedule_at_its_row_limit(lib):
    # exactly 1,048,576 schedule rows (64 x 32 heads x 512 query blocks): the last scratch
    # slot is in use; a sparse random bitmask keeps the schedule small
    shape = lib.WiseShape(64, 32, 16384, 128, 0.0)
    rows = 64 * 32 * 512
    g = torch.Generator(device="cuda").manual_seed(5)
    words = [torch.randint(-2 ** 31, 2 ** 31 - 1, (1, 64 * 32, 512, 16), dtype=torch.int32,
                           device="cuda", generator=g) for _ in range(4)]
    bits = words[0] & words[1] & words[2] & words[3]          # ~1/16 of the bits set
    cap = int(lib.lib.wise_schedule_max_nnz(shape))
    ro_ref, ci_ref, nnz_ref = _with_workspace(lib, bits, shape, cap)
    ro, ci, nnz = _static(lib, bits, shape, cap, with_nnz=True)
    assert ro.numel() == rows + 1 and nnz == nnz_ref > 0
    assert torch.equal(ro, ro_ref)
    assert torch.equal(ci[:nnz], ci_ref[:nnz_ref])


# Runs in a child process that holds no torch state: the driver API makes a second CUDA
# context on the device current between calls, and the library, whose runtime picks up
# the current context, must find its scratch array's address in each context.
_CTX_CHILD = r"""
import ctypes, sys
import numpy as np
cu = ctypes.CDLL("libcuda.so.1")
lib = ctypes.CDLL(sys.argv[1])
def ck(r, what):
    if r != 0:
        raise SystemExit(f"{what} failed: {r}")
class Shape(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("heads", ctypes.c_int32), ("seqlen", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("scale", ctypes.c_float), ("kv_heads", ctypes.c_int32)]
vp, i64 = ctypes.c_void_p, ctypes.c_int64
lib.wise_build_schedule.argtypes = [vp, vp, vp, i64, ctypes.POINTER(i64), vp, ctypes.c_size_t, Shape, vp]
lib.wise_build_schedule_static.argtypes = [vp, vp, vp, i64, ctypes.POINTER(i64), Shape, vp]
lib.wise_schedule_workspace_bytes.restype = ctypes.c_size_t
lib.wise_schedule_workspace_bytes.argtypes = [Shape]
lib.wise_schedule_max_nnz.restype = i64
lib.wise_schedule_max_nnz.argtypes = [Shape]
shape = Shape(1, 6, 2048, 128, 0.0, 0)
rows, W = 6 * 64, 2
cap = lib.wise_schedule_max_nnz(shape)
ws_bytes = lib.wise_schedule_workspace_bytes(shape)
ck(cu.cuInit(0), "cuInit")
dev = ctypes.c_int()
ck(cu.cuDeviceGet(ctypes.byref(dev), 0), "cuDeviceGet")

def alloc(nbytes):
    p = ctypes.c_uint64()
    ck(cu.cuMemAlloc_v2(ctypes.byref(p), ctypes.c_size_t(nbytes)), "cuMemAlloc")
    return p.value

def run(seed):
    # both builds in the current context, on its own buffers; returns (ok, nnz)
    rng = np.random.default_rng(seed)
    bits = rng.integers(0, 2 ** 32, size=rows * W, dtype=np.uint64).astype(np.uint32)
    d_bits = alloc(bits.nbytes)
    ck(cu.cuMemcpyHtoD_v2(ctypes.c_uint64(d_bits), bits.ctypes.data, ctypes.c_size_t(bits.nbytes)), "HtoD")
    out = []
    for static in (False, True):
        ro, ci = alloc(4 * (rows + 1)), alloc(4 * cap)
        nnz = i64(-1)
        if static:
            rc = lib.wise_build_schedule_static(d_bits, ro, ci, cap, ctypes.byref(nnz), shape, None)
        else:
            ws = alloc(max(ws_bytes, 16))
            rc = lib.wise_build_schedule(d_bits, ro, ci, cap, ctypes.byref(nnz), ws, ws_bytes, shape, None)
        ck(rc, "static build" if static else "workspace build")
        h_ro = np.empty(rows + 1, np.int32)
        h_ci = np.empty(nnz.value, np.int32)
        ck(cu.cuMemcpyDtoH_v2(h_ro.ctypes.data, ctypes.c_uint64(ro), ctypes.c_size_t(h_ro.nbytes)), "DtoH")
        ck(cu.cuMemcpyDtoH_v2(h_ci.ctypes.data, ctypes.c_uint64(ci), ctypes.c_size_t(h_ci.nbytes)), "DtoH")
        out.append((h_ro, h_ci))
    return all(np.array_equal(a, b) for a, b in zip(*out)), int(out[1][0][-1])

primary = ctypes.c_void_p()
ck(cu.cuDevicePrimaryCtxRetain(ctypes.byref(primary), dev), "retain")
ck(cu.cuCtxSetCurrent(primary), "set primary")
res = [run(1)]
second = ctypes.c_void_p()
ck(cu.cuCtxCreate_v2(ctypes.byref(second), 0, dev), "cuCtxCreate")   # now current
res.append(run(2))
ck(cu.cuCtxSetCurrent(primary), "back to primary")
res.append(run(3))
ck(cu.cuCtxSynchronize(), "sync")
ck(cu.cuCtxDestroy_v2(second), "cuCtxDestroy")
ck(cu.cuCtxSetCurrent(primary), "primary again")
res.append(run(4))
ck(cu.cuCtxSetCurrent(None), "unset")
ck(cu.cuDevicePrimaryCtxRelease_v2(dev), "release")
print("RESULTS", res)
sys.exit(0 if all(ok and nnz > 0 for ok, nnz in res) else 1)
"""


def test_static_schedule_follows_the_current_context(lib):
    """Calls made in the primary context, in a second context on the same device, and back
    in the primary context each use the scratch address of the context they run in, and
    match the workspace build there."""
    import subprocess
    import sys
    r = subprocess.run([sys.executable, "-c", _CTX_CHILD, lib.LIB_PATH], capture_output=True,
                       text=True, timeout=300)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-2000:]
