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
