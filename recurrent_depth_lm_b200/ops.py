"""torch-tensor front end of the C ABI (argument marshalling only).

Tensors are device tensors owned by the caller (or allocated here with torch
when an output is not supplied); the library itself never allocates.  Every
function launches on the current torch CUDA stream unless `stream` is given.
"""

from __future__ import annotations

import ctypes
import math

import torch

from . import _lib
from ._lib import WiseShape, check, lib

BLOCK = 32


def shape_of(q: torch.Tensor, scale: float | None = None, kv_heads: int = 0) -> WiseShape:
    if q.dim() != 4:
        raise ValueError("expected [batch, heads, seqlen, head_dim]")
    b, h, n, d = q.shape
    return WiseShape(b, h, n, d, float(scale) if scale else 0.0, int(kv_heads))


def _ptr(t: torch.Tensor | None) -> int | None:
    return None if t is None else t.data_ptr()


def _stream(stream) -> int:
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


def _check_qkv(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, o: torch.Tensor) -> int:
    """Validate q/o [B, H, n, d] and k/v [B, H_kv, n, d]; returns H_kv (grouped-query
    attention when H_kv < H: query head h reads K/V head h // (H // H_kv))."""
    for t in (q, k, v, o):
        if not t.is_cuda or t.dtype != torch.bfloat16 or not t.is_contiguous():
            raise ValueError("q/k/v/o must be contiguous bf16 CUDA tensors")
    if o.shape != q.shape or v.shape != k.shape:
        raise ValueError("o must match q and v must match k")
    if q.dim() != 4 or k.dim() != 4 or k.shape[0] != q.shape[0] or k.shape[2:] != q.shape[2:]:
        raise ValueError("k/v must be [batch, kv_heads, seqlen, head_dim] matching q")
    if k.shape[1] < 1 or q.shape[1] % k.shape[1] != 0:
        raise ValueError("query heads must be a multiple of k/v heads")
    return int(k.shape[1])


def words_per_row(nq: int) -> int:
    return (nq + 31) // 32


def full_attn_mass(q, k, v, *, with_mass: bool = False, o=None, lse=None, mass=None,
                   workspace=None, one_pass: bool = True, scale=None, stream=None):
    """Dense causal attention (+ block mass).  Returns (o, lse, mass).

    With mass requested and ``one_pass`` (default), the block mass comes from the
    per-key-block log-sum-exps the attention kernel records in ``workspace``
    (allocated here if not given); ``one_pass=False`` uses the two-pass path.
    """
    b, h, n, d = q.shape
    if o is None:
        o = torch.empty_like(q)
    kv = _check_qkv(q, k, v, o)
    if with_mass and mass is None:
        mass = torch.empty(b, h, n // BLOCK, n // BLOCK, dtype=torch.float32, device=q.device)
    if mass is not None and lse is None:
        lse = torch.empty(b, h, n, dtype=torch.float32, device=q.device)
    if mass is not None and one_pass and workspace is None:
        workspace = mass_workspace(b, h, n, d, q.device)
    ws = workspace if (mass is not None and one_pass) else None
    rc = lib.wise_full_attn_mass(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(mass),
                                 _ptr(ws), 0 if ws is None else ws.numel() * ws.element_size(),
                                 shape_of(q, scale, kv), _stream(stream))
    check(rc, "wise_full_attn_mass")
    return o, lse, mass


def window_step(q, k, v, union_bits, eta: float, *, step_bits=None, o=None, lse=None,
                mass=None, workspace=None, scale=None, stream=None):
    """One discovery-window step: dense attention, block mass and the eta-support ORed
    into `union_bits` (in place), in one library call.  Returns (o, lse, mass)."""
    b, h, n, d = q.shape
    if o is None:
        o = torch.empty_like(q)
    kv = _check_qkv(q, k, v, o)
    if mass is None:
        mass = torch.empty(b, h, n // BLOCK, n // BLOCK, dtype=torch.float32, device=q.device)
    if lse is None:
        lse = torch.empty(b, h, n, dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = mass_workspace(b, h, n, d, q.device)
    if mass.dtype != torch.float32 or union_bits.dtype != torch.int32:
        raise ValueError("mass must be float32 and union_bits int32 (uint32 bit patterns)")
    rc = lib.wise_window_step(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(mass),
                              _ptr(union_bits), _ptr(step_bits), float(eta), _ptr(workspace),
                              workspace.numel() * workspace.element_size(),
                              shape_of(q, scale, kv), _stream(stream))
    check(rc, "wise_window_step")
    return o, lse, mass


def mass_workspace(b: int, h: int, n: int, head_dim: int, device) -> torch.Tensor:
    nbytes = lib.wise_mass_workspace_bytes(WiseShape(b, h, n, head_dim, 0.0))
    return torch.empty(max(1, nbytes // 4), dtype=torch.float32, device=device)


def select_union(mass, union_bits, eta: float, *, step_bits=None, head_dim: int = 128,
                 scale=None, block: int = BLOCK, stream=None):
    """OR the cumulative-eta support of `mass` into `union_bits` (in place).

    ``block`` > 32 selects on blocks of that many tokens (64 or 128) and writes the
    result as 32 x 32 subtiles; ``mass`` is always the 32-token block mass.
    """
    b, h, nq, _ = mass.shape
    shp = WiseShape(b, h, nq * BLOCK, head_dim, float(scale) if scale else 0.0)
    if mass.dtype != torch.float32 or union_bits.dtype != torch.int32:
        raise ValueError("mass must be float32 and union_bits int32 (uint32 bit patterns)")
    if block == BLOCK:
        rc = lib.wise_select_union(_ptr(mass), _ptr(union_bits), _ptr(step_bits), float(eta),
                                   shp, _stream(stream))
        check(rc, "wise_select_union")
    else:
        rc = lib.wise_select_union_blocks(_ptr(mass), _ptr(union_bits), _ptr(step_bits),
                                          float(eta), int(block), shp, _stream(stream))
        check(rc, "wise_select_union_blocks")
    return union_bits


def _control(fn, name, mass, ref_bits, out, head_dim, stream):
    b, h, nq, _ = mass.shape
    if mass.dtype != torch.float32 or ref_bits.dtype != torch.int32:
        raise ValueError("mass must be float32 and ref_bits int32 (uint32 bit patterns)")
    out = torch.empty_like(ref_bits) if out is None else out
    shp = WiseShape(b, h, nq * BLOCK, head_dim, 0.0)
    check(fn(_ptr(mass), _ptr(ref_bits), _ptr(out), shp, _stream(stream)), name)
    return out


def select_size_matched(mass, ref_bits, *, out=None, head_dim: int = 128, stream=None):
    """SizeMatched control: per row the |ref row| blocks of largest mass (TopK)."""
    return _control(lib.wise_select_size_matched, "wise_select_size_matched", mass, ref_bits,
                    out, head_dim, stream)


def select_mass_matched(mass, ref_bits, *, out=None, head_dim: int = 128, stream=None):
    """MassMatched control: per row the fewest ranked blocks reaching the ref row's mass."""
    return _control(lib.wise_select_mass_matched, "wise_select_mass_matched", mass, ref_bits,
                    out, head_dim, stream)


def support_mass(mass, bits, *, out=None, head_dim: int = 128, stream=None):
    """Retained attention mass of the support `bits` per (b, h, q): fp32 [B, H, nq]."""
    b, h, nq, _ = mass.shape
    if mass.dtype != torch.float32 or bits.dtype != torch.int32:
        raise ValueError("mass must be float32 and bits int32 (uint32 bit patterns)")
    out = torch.empty(b, h, nq, dtype=torch.float32, device=mass.device) if out is None else out
    shp = WiseShape(b, h, nq * BLOCK, head_dim, 0.0)
    check(lib.wise_support_mass(_ptr(mass), _ptr(bits), _ptr(out), shp, _stream(stream)),
          "wise_support_mass")
    return out


def new_bitmask(b: int, h: int, nq: int, device) -> torch.Tensor:
    return torch.zeros(b, h, nq, words_per_row(nq), dtype=torch.int32, device=device)


def schedule_workspace(b: int, h: int, n: int, head_dim: int, device) -> torch.Tensor:
    nbytes = lib.wise_schedule_workspace_bytes(WiseShape(b, h, n, head_dim, 0.0))
    return torch.empty(max(1, nbytes), dtype=torch.uint8, device=device)


def schedule_max_nnz(b: int, h: int, n: int, head_dim: int = 128) -> int:
    return int(lib.wise_schedule_max_nnz(WiseShape(b, h, n, head_dim, 0.0)))


def build_schedule(union_bits, *, head_dim: int = 128, row_offsets=None, col_idx=None,
                   workspace=None, exact_nnz: bool = True, stream=None):
    """CSR schedule of the working set.  Returns (row_offsets, col_idx, nnz or None)."""
    b, h, nq, _ = union_bits.shape
    n = nq * BLOCK
    dev = union_bits.device
    if row_offsets is None:
        row_offsets = torch.empty(b * h * nq + 1, dtype=torch.int32, device=dev)
    if col_idx is None:
        col_idx = torch.empty(schedule_max_nnz(b, h, n, head_dim), dtype=torch.int32, device=dev)
    if workspace is None:
        workspace = schedule_workspace(b, h, n, head_dim, dev)
    nnz = ctypes.c_int64(-1)
    rc = lib.wise_build_schedule(_ptr(union_bits), _ptr(row_offsets), _ptr(col_idx),
                                 col_idx.numel(), ctypes.byref(nnz) if exact_nnz else None,
                                 _ptr(workspace), workspace.numel(),
                                 WiseShape(b, h, n, head_dim, 0.0), _stream(stream))
    check(rc, "wise_build_schedule")
    return row_offsets, col_idx, (int(nnz.value) if exact_nnz else None)


def sparse_attn(q, k, v, row_offsets, col_idx, col_count: int | None = None, *, o=None,
                lse=None, scale=None, stream=None):
    """Block-sparse causal attention over a CSR schedule.  Returns (o, lse)."""
    if o is None:
        o = torch.empty_like(q)
    kv = _check_qkv(q, k, v, o)
    if col_count is None:
        col_count = col_idx.numel()
    rc = lib.wise_sparse_attn(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(row_offsets),
                              _ptr(col_idx), int(col_count), _ptr(lse), shape_of(q, scale, kv),
                              _stream(stream))
    check(rc, "wise_sparse_attn")
    return o, lse


# ------------------------------------------------------------------ block size 16

def block_mass_b16(q, k, lse, *, out=None, scale=None, stream=None):
    """Block mass of 16-token blocks from the dense pass's lse: fp32 [B, H, n/16, n/16]."""
    b, h, n, _ = q.shape
    if out is None:
        out = torch.empty(b, h, n // 16, n // 16, dtype=torch.float32, device=q.device)
    kv = _check_qkv(q, k, k, q)
    rc = lib.wise_block_mass_b16(_ptr(q), _ptr(k), _ptr(lse), _ptr(out), shape_of(q, scale, kv),
                                 _stream(stream))
    check(rc, "wise_block_mass_b16")
    return out


def mass_b16_workspace(b: int, h: int, n: int, head_dim: int, device) -> torch.Tensor:
    nbytes = lib.wise_mass_b16_workspace_bytes(WiseShape(b, h, n, head_dim, 0.0))
    return torch.empty(max(1, nbytes // 4), dtype=torch.float32, device=device)


def full_attn_mass_b16(q, k, v, *, o=None, lse=None, mass16=None, workspace=None, scale=None,
                       stream=None):
    """Dense causal attention plus the 16-token block mass in one pass.  Returns
    (o, lse, mass16); the mass equals block_mass_b16's without recomputing QK^T."""
    b, h, n, d = q.shape
    if o is None:
        o = torch.empty_like(q)
    kv = _check_qkv(q, k, v, o)
    if lse is None:
        lse = torch.empty(b, h, n, dtype=torch.float32, device=q.device)
    if mass16 is None:
        mass16 = torch.empty(b, h, n // 16, n // 16, dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = mass_b16_workspace(b, h, n, d, q.device)
    rc = lib.wise_full_attn_mass_b16(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(mass16),
                                     _ptr(workspace), workspace.numel() * workspace.element_size(),
                                     shape_of(q, scale, kv), _stream(stream))
    check(rc, "wise_full_attn_mass_b16")
    return o, lse, mass16


def new_bitmask_b16(b: int, h: int, n: int, device) -> torch.Tensor:
    """Zeroed 16-token working-set masks [B, H, n/16, ceil(n/16/32)]."""
    return new_bitmask(b, h, n // 16, device)


def select_union_b16(mass16, union16, eta: float, *, step_bits=None, head_dim: int = 128,
                     stream=None):
    """OR the cumulative-eta support over 16-token blocks into `union16` (in place)."""
    b, h, n16, _ = mass16.shape
    if mass16.dtype != torch.float32 or union16.dtype != torch.int32:
        raise ValueError("mass16 must be float32 and union16 int32 (uint32 bit patterns)")
    rc = lib.wise_select_union_b16(_ptr(mass16), _ptr(union16), _ptr(step_bits), float(eta),
                                   WiseShape(b, h, n16 * 16, head_dim, 0.0), _stream(stream))
    check(rc, "wise_select_union_b16")
    return union16


def schedule_b16_workspace(b: int, h: int, n: int, head_dim: int, device) -> torch.Tensor:
    nbytes = lib.wise_schedule_b16_workspace_bytes(WiseShape(b, h, n, head_dim, 0.0))
    return torch.empty(max(1, nbytes), dtype=torch.uint8, device=device)


def build_schedule_b16(union16, *, head_dim: int = 128, row_offsets=None, col_idx=None,
                       sub=None, workspace=None, exact_nnz: bool = True, stream=None):
    """32-token CSR schedule plus 16 x 16 sub-masks.  Returns (row_offsets, col_idx, sub, nnz)."""
    b, h, n16, _ = union16.shape
    n = n16 * 16
    nq = n // BLOCK
    dev = union16.device
    if row_offsets is None:
        row_offsets = torch.empty(b * h * nq + 1, dtype=torch.int32, device=dev)
    if col_idx is None:
        col_idx = torch.empty(schedule_max_nnz(b, h, n, head_dim), dtype=torch.int32, device=dev)
    if sub is None:
        sub = torch.empty(col_idx.numel(), dtype=torch.uint8, device=dev)
    if sub.numel() < col_idx.numel():
        raise ValueError("sub must hold one byte per col_idx entry")
    if workspace is None:
        workspace = schedule_b16_workspace(b, h, n, head_dim, dev)
    nnz = ctypes.c_int64(-1)
    rc = lib.wise_build_schedule_b16(_ptr(union16), _ptr(row_offsets), _ptr(col_idx), _ptr(sub),
                                     col_idx.numel(), ctypes.byref(nnz) if exact_nnz else None,
                                     _ptr(workspace), workspace.numel(),
                                     WiseShape(b, h, n, head_dim, 0.0), _stream(stream))
    check(rc, "wise_build_schedule_b16")
    return row_offsets, col_idx, sub, (int(nnz.value) if exact_nnz else None)


def sparse_attn_b16(q, k, v, row_offsets, col_idx, sub, col_count: int | None = None, *,
                    o=None, lse=None, scale=None, stream=None):
    """Block-sparse causal attention whose entries carry 16 x 16 sub-masks.  Returns (o, lse)."""
    if o is None:
        o = torch.empty_like(q)
    kv = _check_qkv(q, k, v, o)
    if col_count is None:
        col_count = col_idx.numel()
    rc = lib.wise_sparse_attn_b16(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(row_offsets),
                                  _ptr(col_idx), _ptr(sub), int(col_count), _ptr(lse),
                                  shape_of(q, scale, kv), _stream(stream))
    check(rc, "wise_sparse_attn_b16")
    return o, lse


def device_status(clear: bool = True) -> int:
    st = ctypes.c_uint32(0)
    check(lib.wise_device_status(ctypes.byref(st), 1 if clear else 0), "wise_device_status")
    return int(st.value)


def causal_flops(n: int, d: int, bh: int) -> float:
    """Useful FLOPs of dense causal attention: 4*d per admissible (i, j) pair."""
    return 4.0 * d * bh * n * (n + 1) / 2


def default_scale(d: int) -> float:
    return 1.0 / math.sqrt(d)
