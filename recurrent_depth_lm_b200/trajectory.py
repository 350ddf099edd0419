"""WISE trajectory driver for one attention layer (the user-facing API).

Wan & Chen, "Attention Routing Stabilizes Early: Working-Set Inference for
Recurrent-Depth Language Models", section 5 and appendix B: steps
t <= t_d run unrestricted (dense) causal attention; steps t_d-3 .. t_d also
select each query block's cumulative-eta key-block support and union it;
after step t_d the union is compacted once into a CSR schedule; every later
step runs block-sparse attention over that schedule with fresh Q, K, V.
Appendix C.6's block-size variants (block = 64 or 128) select on coarser blocks
and run the result as exact 32 x 32 subtiles; block = 16 selects on 16-token
blocks (masses recomputed from the dense pass's lse) and runs 32 x 32 tiles that
carry 16 x 16 sub-masks.

The selection-only controls of appendix B ("Intervention controls") replace the
frozen support: "static95" is the eta-support of step 1 alone, "size_matched"
the |W_q| blocks of largest step-1 mass, "mass_matched" the fewest step-1-ranked
blocks reaching the step-1 mass of W_q; steps up to t_d are unchanged.  With
track_retained, every late step also runs dense attention with block mass
(analysis only) and records the retained future mass of the frozen support
("Evaluation metrics").

All buffers are allocated once here with torch; the library calls only
enqueue kernels on the current stream (no host synchronisation inside a
trajectory).
"""

from __future__ import annotations

import torch

from . import ops

SUPPORTS = ("wise", "static95", "size_matched", "mass_matched")


class WiseTrajectory:
    def __init__(self, batch: int, heads: int, seqlen: int, head_dim: int, *, t_d: int = 12,
                 window=(9, 12), eta: float = 0.95, scale: float | None = None,
                 block: int = ops.BLOCK, support: str = "wise", track_retained: bool = False,
                 device="cuda", keep_step_bits: bool = False):
        if support not in SUPPORTS:
            raise ValueError(f"support must be one of {SUPPORTS}")
        if support in ("size_matched", "mass_matched") and block != ops.BLOCK:
            raise ValueError("the size- and mass-matched controls are defined for block = 32")
        if block not in (16, 32, 64, 128):
            raise ValueError("block must be 16, 32, 64 or 128")
        if block == 16 and (support != "wise" or track_retained):
            raise ValueError("block 16 runs the WISE support without retained-mass tracking")
        if seqlen % block:
            raise ValueError(f"seqlen must be a multiple of the block size {block}")
        self.block = block
        self.b, self.h, self.n, self.d = batch, heads, seqlen, head_dim
        self.nq = seqlen // ops.BLOCK
        self.t_d, self.window, self.eta = t_d, tuple(window), float(eta)
        self.scale = scale
        dev = torch.device(device)
        self.lse = torch.empty(batch, heads, seqlen, dtype=torch.float32, device=dev)
        self.mass16 = self.sub = self.mass = self.mass_ws = None
        if block == 16:   # 16-token masses and working set; sub-masks of the schedule
            self.mass16 = torch.empty(batch, heads, seqlen // 16, seqlen // 16,
                                      dtype=torch.float32, device=dev)
            self.union = ops.new_bitmask_b16(batch, heads, seqlen, dev)
            # per-(row, 16-key block) log-sum-exps of the one-pass 16-token mass
            self.mass_ws = ops.mass_b16_workspace(batch, heads, seqlen, head_dim, dev)
        else:
            self.mass = torch.empty(batch, heads, self.nq, self.nq, dtype=torch.float32,
                                    device=dev)
            self.union = ops.new_bitmask(batch, heads, self.nq, dev)
            # per-(row, key block) log-sum-exps of the one-pass block mass (window steps)
            self.mass_ws = ops.mass_workspace(batch, heads, seqlen, head_dim, dev)
        self.step_bits = {}
        self.keep_step_bits = keep_step_bits
        self.row_offsets = torch.empty(batch * heads * self.nq + 1, dtype=torch.int32, device=dev)
        self.col_idx = torch.empty(ops.schedule_max_nnz(batch, heads, seqlen, head_dim),
                                   dtype=torch.int32, device=dev)
        self.workspace = ops.schedule_workspace(batch, heads, seqlen, head_dim, dev)
        if block == 16:
            self.sub = torch.empty(self.col_idx.numel(), dtype=torch.uint8, device=dev)
            self.workspace = ops.schedule_b16_workspace(batch, heads, seqlen, head_dim, dev)
        self.scheduled = False
        self.support = support
        # step-1 block masses and the control support (selection-only controls)
        self.mass1 = (torch.empty_like(self.mass) if support != "wise" else None)
        self.control = ops.new_bitmask(batch, heads, self.nq, dev) if support != "wise" else None
        self.track_retained = track_retained
        self.retained = {}
        self.o_scratch = None
        if track_retained:
            self.o_scratch = torch.empty(batch, heads, seqlen, head_dim, dtype=torch.bfloat16,
                                         device=dev)

    def reset(self) -> None:
        self.union.zero_()
        if self.control is not None:
            self.control.zero_()
        self.step_bits.clear()
        self.retained.clear()
        self.scheduled = False

    @property
    def frozen(self):
        """The support the late steps run on (the WISE union or the control)."""
        return self.union if self.support == "wise" else self.control

    def in_window(self, t: int) -> bool:
        return self.window[0] <= t <= self.window[1]

    def step(self, t: int, q, k, v, o=None, lse=None, stream=None):
        """Attention of recurrent step t (1-based).  Returns O."""
        if t <= self.t_d:
            first = t == 1 and self.mass1 is not None   # step-1 masses for the controls
            if self.block == 16 and self.in_window(t):
                o, _, _ = ops.full_attn_mass_b16(q, k, v, o=o, lse=self.lse, mass16=self.mass16,
                                                 workspace=self.mass_ws, scale=self.scale,
                                                 stream=stream)
                sb = None
                if self.keep_step_bits:
                    sb = torch.empty_like(self.union)
                    self.step_bits[t] = sb
                ops.select_union_b16(self.mass16, self.union, self.eta, step_bits=sb,
                                     head_dim=self.d, stream=stream)
            elif self.in_window(t) or first:
                m = self.mass1 if first else self.mass
                sb = None
                if self.in_window(t) and self.keep_step_bits:
                    sb = torch.empty_like(self.union)
                    self.step_bits[t] = sb
                if self.in_window(t) and self.block == ops.BLOCK:
                    # attention, block mass and selection in one library call
                    o, _, _ = ops.window_step(q, k, v, self.union, self.eta, step_bits=sb, o=o,
                                              lse=self.lse, mass=m, workspace=self.mass_ws,
                                              scale=self.scale, stream=stream)
                else:
                    o, _, _ = ops.full_attn_mass(q, k, v, o=o, lse=self.lse, mass=m,
                                                 workspace=self.mass_ws, scale=self.scale,
                                                 stream=stream)
                    if self.in_window(t):
                        ops.select_union(m, self.union, self.eta, step_bits=sb,
                                         head_dim=self.d, scale=self.scale, block=self.block,
                                         stream=stream)
                if first and self.support == "static95":
                    ops.select_union(m, self.control, self.eta, head_dim=self.d,
                                     scale=self.scale, block=self.block, stream=stream)
            else:
                o, _, _ = ops.full_attn_mass(q, k, v, o=o, lse=lse, scale=self.scale,
                                             stream=stream)
            if t == self.t_d:
                self.build_schedule(stream=stream)
            return o
        if not self.scheduled:
            raise RuntimeError("late step before the schedule was built (t <= t_d never reached)")
        if self.block == 16:
            o, _ = ops.sparse_attn_b16(q, k, v, self.row_offsets, self.col_idx, self.sub,
                                       self.col_idx.numel(), o=o, lse=lse, scale=self.scale,
                                       stream=stream)
        else:
            o, _ = ops.sparse_attn(q, k, v, self.row_offsets, self.col_idx,
                                   self.col_idx.numel(), o=o, lse=lse, scale=self.scale,
                                   stream=stream)
        if self.track_retained:
            ops.full_attn_mass(q, k, v, o=self.o_scratch, lse=self.lse, mass=self.mass,
                               workspace=self.mass_ws, scale=self.scale, stream=stream)
            self.retained[t] = ops.support_mass(self.mass, self.frozen, head_dim=self.d,
                                                stream=stream)
        return o

    def build_schedule(self, stream=None) -> None:
        if self.support == "size_matched":
            ops.select_size_matched(self.mass1, self.union, out=self.control, head_dim=self.d,
                                    stream=stream)
        elif self.support == "mass_matched":
            ops.select_mass_matched(self.mass1, self.union, out=self.control, head_dim=self.d,
                                    stream=stream)
        if self.block == 16:
            ops.build_schedule_b16(self.union, head_dim=self.d, row_offsets=self.row_offsets,
                                   col_idx=self.col_idx, sub=self.sub, workspace=self.workspace,
                                   exact_nnz=False, stream=stream)
        else:
            ops.build_schedule(self.frozen, head_dim=self.d, row_offsets=self.row_offsets,
                               col_idx=self.col_idx, workspace=self.workspace, exact_nnz=False,
                               stream=stream)
        self.scheduled = True

    def retained_future_mass(self) -> float:
        """Mean over late steps, heads and query blocks of the retained attention mass."""
        if not self.retained:
            raise RuntimeError("no late step ran with track_retained=True")
        return float(torch.stack(list(self.retained.values())).mean().item())

    # ------------------------------------------------------------ save / replay
    def state(self) -> dict:
        """The frozen working set and its schedule as host arrays.  Late steps depend on
        nothing else, so a loaded state replays them without the exploration steps."""
        import numpy as np
        if not self.scheduled:
            raise RuntimeError("no schedule yet: run the steps up to t_d first")
        nnz = self.nnz()
        st = {
            "shape": np.array([self.b, self.h, self.n, self.d, self.block], np.int64),
            "t_d": np.array(self.t_d), "window": np.array(self.window), "eta": np.array(self.eta),
            "support": np.array(self.support),
            "frozen": self.frozen.cpu().numpy(),
            "row_offsets": self.row_offsets.cpu().numpy(),
            "col_idx": self.col_idx[:nnz].cpu().numpy(),
        }
        if self.sub is not None:
            st["sub"] = self.sub[:nnz].cpu().numpy()
        return st

    def save(self, path) -> None:
        import numpy as np
        np.savez(path, **self.state())

    def load(self, path_or_state) -> None:
        """Restore a saved working set and schedule; the next step may be any t > t_d."""
        import numpy as np
        st = path_or_state if isinstance(path_or_state, dict) else dict(np.load(path_or_state))
        want = np.array([self.b, self.h, self.n, self.d, self.block], np.int64)
        if not np.array_equal(np.asarray(st["shape"]), want):
            raise ValueError(f"saved shape/block {st['shape'].tolist()} != {want.tolist()}")
        col = np.asarray(st["col_idx"], np.int32)
        ro = np.asarray(st["row_offsets"], np.int32)
        if ro.shape != tuple(self.row_offsets.shape) or col.size > self.col_idx.numel() or \
                (ro.size and int(ro[-1]) != col.size):
            raise ValueError("saved schedule does not fit this trajectory")
        self.frozen.copy_(torch.from_numpy(np.asarray(st["frozen"], np.int32)))
        self.row_offsets.copy_(torch.from_numpy(ro))
        self.col_idx[:col.size].copy_(torch.from_numpy(col))
        if self.sub is not None:
            self.sub[:col.size].copy_(torch.from_numpy(np.asarray(st["sub"], np.uint8)))
        self.scheduled = True

    def nnz(self) -> int:
        return int(self.row_offsets[-1].item())

    def density(self) -> float:
        """Fraction of admissible (causal) query-key blocks retained, counted at the
        selection's block size (16-token blocks for block = 16)."""
        if self.block != 16:
            return self.nnz() / (self.b * self.h * self.nq * (self.nq + 1) / 2)
        import numpy as np
        n16 = self.n // 16
        words = self.union.cpu().numpy().view(np.uint32).reshape(-1, n16, self.union.shape[-1])
        bits = np.unpackbits(words.view(np.uint8), axis=-1, bitorder="little")[..., :n16]
        return float(np.tril(bits.astype(bool)).sum()) / (self.b * self.h * n16 * (n16 + 1) / 2)
