"""Sign-Muon with one process per GPU and a real sign exchange.

The SignMuon summary's distributed flow (section 2 "Algorithmic flow
(distributed)", steps 1-5, and "Communication efficiency"): every worker
computes its sign matrices locally, the signs are exchanged -- a 1-bit
all-gather of the packed words, or an integer SUM all-reduce of the int8
signs -- and every worker applies the same majority vote to its own replica
of W, so the replicas stay identical without exchanging W.

Here each process (rank) holds `local_workers` workers as buffers on its GPU,
so the vote covers world_size * local_workers workers.  The exchange is one
collective per group of matrices, issued on a dedicated stream as soon as the
group's Newton-Schulz iterations have written its signs, so that it overlaps
the iterations of the next group.  Only the collective is a library call
(NCCL through torch.distributed); momentum, Newton-Schulz, sign packing and
the vote are the kernels of libsignmuon.so, called exactly as in SignMuonStep.

Exchange layouts (per group g of consecutive matrices, per local unit (i, m)
in matrix-major, worker-minor order, each unit's block a multiple of 16
bytes):
  pack1: local[g]    = the units' packed words back to back;
         gathered[g] = all ranks' local[g] in rank order (all_gather), so the
         vote reads global worker r * local_workers + m of matrix i at
         gathered[g] + r * len(local[g]) + offset(i, m).
  int8:  local[g]    = the units' int8 signs back to back, summed in place
         over the ranks (all_reduce SUM); the vote then sums the
         local_workers partial sums of matrix i and takes the sign, which is
         sign(sum over all world_size * local_workers workers).
"""
from __future__ import annotations

import dataclasses
from typing import List, Optional, Sequence, Tuple

import torch

from . import _lib as L
from .step import NS_QUINTIC, _check_buf, _dtype_code


@dataclasses.dataclass
class ExchangeLayout:
    """Where every local unit's signs sit in the per-group exchange buffers.

    groups[g]      = (first matrix, end matrix) of group g
    offsets[u]     = element offset of local unit u = i * local_workers + m in
                     its group's buffer (int32 words for pack1, bytes for int8)
    group_len[g]   = elements of group g's local buffer
    group_of[i]    = the group of matrix i
    """
    variant: str
    local_workers: int
    groups: List[Tuple[int, int]]
    offsets: List[int]
    group_len: List[int]
    group_of: List[int]


def _unit_elems(shape, variant: str) -> int:
    r, c = shape
    if variant == "pack1":
        return int(L.signmuon_packed_words((r, c)))     # a multiple of 4 words
    return (r * c + 15) // 16 * 16                       # int8, padded to 16 bytes


def exchange_layout(shapes: Sequence[Tuple[int, int]], local_workers: int, n_groups: int,
                    variant: str) -> ExchangeLayout:
    """Splits the matrices into at most n_groups consecutive, non-empty groups
    of about equal parameter count (group g closes at the first matrix where
    the running count reaches g/n_groups of the total) and lays out every
    local unit's signs in them."""
    if variant not in ("pack1", "int8"):
        raise ValueError("variant must be 'pack1' or 'int8'")
    if local_workers < 1 or n_groups < 1:
        raise ValueError("local_workers and n_groups must be >= 1")
    shapes = [(int(r), int(c)) for r, c in shapes]
    total = sum(r * c for r, c in shapes)
    bounds, cum = [0], 0
    for i, (r, c) in enumerate(shapes):
        cum += r * c
        if len(bounds) < n_groups and cum * n_groups >= total * len(bounds) and i + 1 < len(shapes):
            bounds.append(i + 1)
    bounds.append(len(shapes))
    groups = [(bounds[j], bounds[j + 1]) for j in range(len(bounds) - 1)]
    offsets, group_len, group_of = [], [], [0] * len(shapes)
    for g, (a, b) in enumerate(groups):
        off = 0
        for i in range(a, b):
            group_of[i] = g
            n = _unit_elems(shapes[i], variant)
            for _ in range(local_workers):
                offsets.append(off)
                off += n
        group_len.append(off)
    return ExchangeLayout(variant, local_workers, groups, offsets, group_len, group_of)


def vote_sign_offsets(layout: ExchangeLayout, world_size: int) -> List[Tuple[int, int]]:
    """(group, element offset) of every sign buffer the vote reads, in the
    vote's (matrix-major, worker-minor) order.  pack1: world_size *
    local_workers workers per matrix in the gathered buffers; int8:
    local_workers (already summed over ranks) in the local buffers."""
    out = []
    n_mats = len(layout.group_of)
    Ml = layout.local_workers
    for i in range(n_mats):
        g = layout.group_of[i]
        if layout.variant == "pack1":
            for r in range(world_size):
                for m in range(Ml):
                    out.append((g, r * layout.group_len[g] + layout.offsets[i * Ml + m]))
        else:
            for m in range(Ml):
                out.append((g, layout.offsets[i * Ml + m]))
    return out


def exchange(kind: str, local: torch.Tensor, gathered: Optional[torch.Tensor], group=None) -> None:
    """The collective of one group: all_gather of the packed words (pack1)
    into `gathered`, or in-place SUM all_reduce of the int8 signs."""
    import torch.distributed as dist
    if kind == "pack1":
        dist.all_gather_into_tensor(gathered, local, group=group)
    else:
        dist.all_reduce(local, op=dist.ReduceOp.SUM, group=group)


class SignMuonDistStep:
    """One Sign-Muon step per call with local_workers workers on this rank
    and the signs exchanged over `group` (torch.distributed, NCCL on GPUs).

    world_size / rank default to the group's; they may be given explicitly to
    drive the phases without a process group (local_phase, then filling
    `gathered` / `local`, then vote_phase).
    """

    def __init__(self, shapes: Sequence[Tuple[int, int]], local_workers: int, k: int, variant: str,
                 beta: float, eta: float, w_dtype: torch.dtype, polar: bool = False,
                 coeffs=NS_QUINTIC, device: Optional[torch.device] = None, group=None,
                 world_size: Optional[int] = None, rank: Optional[int] = None, n_groups: Optional[int] = None,
                 ns_workspace_cap: int = 16 << 30):
        if world_size is None or rank is None:
            import torch.distributed as dist
            world_size = dist.get_world_size(group) if world_size is None else world_size
            rank = dist.get_rank(group) if rank is None else rank
        self.world_size, self.rank, self.group = int(world_size), int(rank), group
        L.load()
        self.shapes = [(int(r), int(c)) for r, c in shapes]
        self.local_workers = Ml = int(local_workers)
        self.vote_workers = self.world_size * Ml if variant == "pack1" else Ml
        if self.world_size * Ml > L.SIGNMUON_MAX_WORKERS:
            raise ValueError(f"world_size * local_workers must be <= {L.SIGNMUON_MAX_WORKERS}")
        self.k, self.variant = int(k), variant
        self.beta, self.eta, self.w_dtype = float(beta), float(eta), w_dtype
        self.polar, self.coeffs = bool(polar), tuple(float(x) for x in coeffs)
        self.device = dev = torch.device(device or "cuda")
        # Several groups let the exchange of one overlap the Newton-Schulz
        # iterations of the next; a single rank has nothing to overlap.
        if n_groups is None:
            n_groups = 1 if self.world_size == 1 else 4
        self.layout = lay = exchange_layout(self.shapes, Ml, n_groups, variant)
        n_mats = len(self.shapes)
        self.units = n_mats * Ml
        self.mom = [torch.zeros(self.shapes[u // Ml], dtype=torch.float32, device=dev) for u in range(self.units)]
        self.x = [torch.empty((self.shapes[u // Ml][0], L.signmuon_x_ld(self.shapes[u // Ml][1])),
                              dtype=torch.bfloat16, device=dev) for u in range(self.units)]
        self.inv_norm = torch.empty(self.units, dtype=torch.float32, device=dev)
        self.ws_mom = torch.empty(L.signmuon_momentum_workspace_bytes(self.shapes, Ml), dtype=torch.uint8,
                                  device=dev)
        elt = torch.int32 if variant == "pack1" else torch.int8
        esz = 4 if variant == "pack1" else 1
        self.local = [torch.zeros(n, dtype=elt, device=dev) for n in lay.group_len]
        self.gathered = ([torch.zeros(self.world_size * n, dtype=elt, device=dev) for n in lay.group_len]
                         if variant == "pack1" else None)
        # Newton-Schulz: one workspace and one plan per group (a plan's unit
        # table lives in its workspace), outputs straight into local[g].
        self.ws_ns, self._plans = [], [None] * len(lay.groups)
        for (a, b) in lay.groups:
            gs = self.shapes[a:b]
            full = L.signmuon_newton_schulz_workspace_bytes(gs, Ml)
            minimal = L.signmuon_newton_schulz_workspace_bytes(gs, Ml, minimal=True)
            self.ws_ns.append(torch.empty(max(minimal, min(full, ns_workspace_cap)), dtype=torch.uint8,
                                          device=dev))
        self.ws_vote = torch.empty(L.signmuon_vote_workspace_bytes(self.shapes, self.vote_workers),
                                   dtype=torch.uint8, device=dev)
        src = self.gathered if variant == "pack1" else self.local
        self._vote_ptrs = [src[g].data_ptr() + off * esz for g, off in vote_sign_offsets(lay, self.world_size)]
        self._esz = esz
        self.comm_stream = torch.cuda.Stream(device=dev)
        self._events = [torch.cuda.Event() for _ in lay.groups]
        if self.polar:
            self.vote = [torch.empty((r, L.signmuon_x_ld(c)), dtype=torch.bfloat16, device=dev)
                         for (r, c) in self.shapes]
            self.nnz = torch.zeros(max(n_mats, 2), dtype=torch.int64, device=dev)
            self.vote_inv = torch.zeros(max(n_mats, 4), dtype=torch.float32, device=dev)
            full1 = L.signmuon_newton_schulz_workspace_bytes(self.shapes, 1)
            min1 = L.signmuon_newton_schulz_workspace_bytes(self.shapes, 1, minimal=True)
            self.ws_polar = torch.empty(max(min1, min(full1, ns_workspace_cap)), dtype=torch.uint8, device=dev)
            self._polar_plan, self._polar_key = None, None

    # ------------------------------------------------------------------
    def state_dict(self):
        return {"mom": [m.clone() for m in self.mom]}

    def load_state_dict(self, sd):
        for dst, src in zip(self.mom, sd["mom"]):
            dst.copy_(src)

    def _ns_group(self, g: int, stream: int) -> None:
        a, b = self.layout.groups[g]
        Ml = self.local_workers
        if self._plans[g] is None:
            u0, u1 = a * Ml, b * Ml
            outs = [self.local[g].data_ptr() + self.layout.offsets[u] * self._esz for u in range(u0, u1)]
            mode = L.SIGNMUON_OUT_PACK1 if self.variant == "pack1" else L.SIGNMUON_OUT_INT8
            self._plans[g] = L.signmuon_newton_schulz_plan(
                self.shapes[a:b], Ml, [x.data_ptr() for x in self.x[u0:u1]], self.inv_norm.data_ptr() + 4 * u0,
                mode, outs, L.SIGNMUON_F32, None, self.ws_ns[g].data_ptr(), self.ws_ns[g].numel(), stream)
        ca, cb, cc = self.coeffs
        L.signmuon_newton_schulz_run(self._plans[g], self.k, ca, cb, cc, 0.0, stream)

    def local_phase(self, grads: Sequence[torch.Tensor], stream: Optional[int] = None) -> None:
        """Momentum, normalisation, Newton-Schulz and the signs of this rank's
        workers, into the local exchange buffers (no exchange)."""
        stream = self._stream(stream)
        self._momentum(grads, stream)
        for g in range(len(self.layout.groups)):
            self._ns_group(g, stream)

    def _momentum(self, grads, stream):
        Ml = self.local_workers
        if len(grads) != self.units:
            raise ValueError("expected one gradient per (matrix, local worker)")
        gptr = [_check_buf(gr, self.shapes[u // Ml], self.w_dtype, f"grad[{u}]") for u, gr in enumerate(grads)]
        L.signmuon_momentum_norm(self.shapes, Ml, _dtype_code(self.w_dtype), gptr,
                                 [m.data_ptr() for m in self.mom], self.beta, [x.data_ptr() for x in self.x],
                                 self.inv_norm.data_ptr(), self.ws_mom.data_ptr(), self.ws_mom.numel(), stream)

    def vote_phase(self, weights: Sequence[torch.Tensor], stream: Optional[int] = None) -> None:
        """Majority vote over every worker's signs (from the exchange buffers)
        and the update of this rank's replica of W (+ the local polar step)."""
        stream = self._stream(stream)
        wptr = [_check_buf(w, s, self.w_dtype, f"weight[{i}]") for i, (w, s) in enumerate(zip(weights, self.shapes))]
        int8_in = self.variant == "int8"
        if not self.polar:
            L.signmuon_vote_update(self.shapes, self.vote_workers, int8_in, self._vote_ptrs,
                                   _dtype_code(self.w_dtype), wptr, self.eta, None, 0, 0, self.ws_vote.data_ptr(),
                                   self.ws_vote.numel(), stream)
            return
        L.signmuon_vote_update(self.shapes, self.vote_workers, int8_in, self._vote_ptrs,
                               _dtype_code(self.w_dtype), None, self.eta, [v.data_ptr() for v in self.vote],
                               self.nnz.data_ptr(), self.vote_inv.data_ptr(), self.ws_vote.data_ptr(),
                               self.ws_vote.numel(), stream)
        if self._polar_key != tuple(wptr):
            self._polar_plan = L.signmuon_newton_schulz_plan(
                self.shapes, 1, [v.data_ptr() for v in self.vote], self.vote_inv.data_ptr(),
                L.SIGNMUON_OUT_UPDATE_W, None, _dtype_code(self.w_dtype), wptr, self.ws_polar.data_ptr(),
                self.ws_polar.numel(), stream, plan=self._polar_plan)
            self._polar_key = tuple(wptr)
        ca, cb, cc = self.coeffs
        L.signmuon_newton_schulz_run(self._polar_plan, 1, ca, cb, cc, self.eta, stream)

    # The three phases under the names SignMuonStep uses.
    def momentum_norm(self, grads: Sequence[torch.Tensor], stream: int) -> None:
        self._momentum(grads, stream)

    def newton_schulz(self, stream: int) -> None:
        """Newton-Schulz + signs of each group, each group's exchange issued
        on comm_stream as soon as its signs exist (overlapping the next
        group's iterations); `stream` (the current stream of the device)
        then waits for the last exchange."""
        main = torch.cuda.current_stream(self.device)
        if main.cuda_stream != stream:
            raise ValueError("newton_schulz must run on the device's current stream")
        for g in range(len(self.layout.groups)):
            self._ns_group(g, stream)
            self._events[g].record(main)
            self.comm_stream.wait_event(self._events[g])
            with torch.cuda.stream(self.comm_stream):
                exchange(self.variant, self.local[g], self.gathered[g] if self.gathered else None, self.group)
        main.wait_stream(self.comm_stream)

    def vote_update(self, weights: Sequence[torch.Tensor], stream: int) -> None:
        self.vote_phase(weights, stream)

    def step(self, weights: Sequence[torch.Tensor], grads: Sequence[torch.Tensor]) -> None:
        """One step: momentum, then Newton-Schulz with the pipelined exchange,
        then the vote and the update, on the current stream."""
        stream = torch.cuda.current_stream(self.device).cuda_stream
        self._momentum(grads, stream)
        self.newton_schulz(stream)
        self.vote_phase(weights, stream)

    def kernel_launches_per_step(self) -> int:
        """libsignmuon kernels per step once the plans exist (the collectives
        are NCCL's, not counted)."""
        def uploads(nbytes):
            return max(1, -(-nbytes // (32768 - 512)))
        n_mats = len(self.shapes)
        mom = uploads(self.units * 56) + 2
        ns = 0
        for g, (a, b) in enumerate(self.layout.groups):
            ns += (3 * self.k if self.k > 0 else 1) * self._waves(self.shapes[a:b], self.local_workers,
                                                                  self.ws_ns[g].numel())
        vote = uploads(-(-n_mats * 64 // 256) * 256 + n_mats * self.vote_workers * 8) + 1
        total = mom + ns + vote
        if self.polar:
            total += 1 + 3 * self._waves(self.shapes, 1, self.ws_polar.numel())
        return total

    @staticmethod
    def _waves(shapes, M, ws_bytes) -> int:
        from .step import SignMuonStep
        return SignMuonStep._waves(shapes, M, ws_bytes)

    def exchange_bytes_per_step(self) -> int:
        """Bytes this rank contributes to the exchange per step."""
        return sum(self.layout.group_len) * self._esz

    def _stream(self, stream):
        return torch.cuda.current_stream(self.device).cuda_stream if stream is None else stream
