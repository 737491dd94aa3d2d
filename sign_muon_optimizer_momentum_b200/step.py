"""SignMuonStep: one Sign-Muon optimizer step over M simulated workers.

The step follows the SignMuon summary's "Algorithmic flow (distributed)"
(section 2), with the M workers held as M gradient and momentum buffers on
one GPU, so that the exchange of step 3 becomes the local M-way reduction of
the vote kernel:

  1. signmuon_momentum_norm          momentum, bf16 copy, Frobenius norm
  2. signmuon_newton_schulz_run      k iterations, sign fused into the last
                                     (planned once by signmuon_newton_schulz_plan)
  3-4. signmuon_vote_update          majority vote + W <- W - eta * vote
  5. (polar) vote matrix -> one Newton-Schulz iteration -> W update

PyTorch is used only to allocate device buffers and to pick the stream; all
arithmetic runs in libsignmuon.so.
"""
from __future__ import annotations

from typing import List, Optional, Sequence, Tuple

import torch

from . import _lib as L

NS_QUINTIC = (3.4445, -4.7750, 2.0315)


def _dtype_code(dt: torch.dtype) -> int:
    if dt == torch.float32:
        return L.SIGNMUON_F32
    if dt == torch.bfloat16:
        return L.SIGNMUON_BF16
    raise TypeError(f"unsupported dtype {dt} (fp32 or bf16)")


def _check_buf(t: torch.Tensor, shape, dtype, what: str) -> int:
    if not t.is_cuda:
        raise ValueError(f"{what} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{what}: expected {dtype}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape) or not t.is_contiguous():
        raise ValueError(f"{what}: expected a contiguous tensor of shape {tuple(shape)}")
    p = t.data_ptr()
    if p % 16:
        raise ValueError(f"{what}: data pointer must be 16-byte aligned")
    return p


class SignMuonStep:
    """Holds the optimizer state (one fp32 momentum buffer per worker and
    matrix) and the scratch buffers of the step.

    shapes:    list of (rows, cols) weight matrices
    n_workers: M, the number of simulated data-parallel workers
    k:         Newton-Schulz iterations
    variant:   "pack1" (1-bit packed signs) or "int8" (integer-sum vote)
    polar:     run the optional local polar step on the voted matrix
    norm:      "frobenius" (X0 = M / ||M||_F) or "spectral" (X0 = M / sigma_est,
               sigma_est from `spectral_iters` power iterations)
    """

    def __init__(self, shapes: Sequence[Tuple[int, int]], n_workers: int, k: int, variant: str,
                 beta: float, eta: float, w_dtype: torch.dtype, polar: bool = False,
                 coeffs=NS_QUINTIC, device: Optional[torch.device] = None,
                 ns_workspace_cap: int = 16 << 30, norm: str = "frobenius", spectral_iters: int = 5):
        if variant not in ("pack1", "int8"):
            raise ValueError("variant must be 'pack1' or 'int8'")
        if norm not in ("frobenius", "spectral"):
            raise ValueError("norm must be 'frobenius' or 'spectral'")
        self.norm = norm
        self.spectral_iters = int(spectral_iters)
        L.load()
        self.shapes = [(int(r), int(c)) for r, c in shapes]
        self.n_workers = int(n_workers)
        self.k = int(k)
        self.variant = variant
        self.beta = float(beta)
        self.eta = float(eta)
        self.w_dtype = w_dtype
        self.polar = bool(polar)
        self.coeffs = tuple(float(x) for x in coeffs)
        self.device = torch.device(device or "cuda")
        dev = self.device
        M = self.n_workers
        self.units = len(self.shapes) * M
        # k = 0 with the Frobenius scale: sign(X0) = sign(M) (all +1 for a
        # non-finite norm), so the momentum kernel writes the signs directly
        # (no bf16 copy of M, no Newton-Schulz call).  Packed signs need whole
        # 32-column words per row.
        self.fused_sign = (self.k == 0 and norm == "frobenius" and
                           (variant == "int8" or all(c % 32 == 0 for _, c in self.shapes)))
        self.mom: List[torch.Tensor] = []
        self.x: List[torch.Tensor] = []
        self.signs: List[torch.Tensor] = []
        for (r, c) in self.shapes:
            for _ in range(M):
                self.mom.append(torch.zeros((r, c), dtype=torch.float32, device=dev))
                if not self.fused_sign:
                    self.x.append(torch.empty((r, L.signmuon_x_ld(c)), dtype=torch.bfloat16, device=dev))
                if variant == "pack1":
                    self.signs.append(torch.empty(L.signmuon_packed_words((r, c)), dtype=torch.int32,
                                                  device=dev))
                else:
                    self.signs.append(torch.empty((r, c), dtype=torch.int8, device=dev))
        self.inv_norm = torch.empty(self.units, dtype=torch.float32, device=dev)
        self.ws_mom = torch.empty(L.signmuon_momentum_workspace_bytes(self.shapes, M), dtype=torch.uint8,
                                  device=dev)
        self._ns_plan = self._polar_plan = None
        self._ns_plan_key = self._polar_plan_key = None
        full = L.signmuon_newton_schulz_workspace_bytes(self.shapes, M)
        minimal = L.signmuon_newton_schulz_workspace_bytes(self.shapes, M, minimal=True)
        # (No Newton-Schulz workspace when k = 0 runs fused.)
        self.ws_ns = torch.empty(0 if self.fused_sign else max(minimal, min(full, ns_workspace_cap)),
                                 dtype=torch.uint8, device=dev)
        self.ws_vote = torch.empty(L.signmuon_vote_workspace_bytes(self.shapes, M), dtype=torch.uint8,
                                   device=dev)
        if self.norm == "spectral":
            self.ws_spec = torch.empty(L.signmuon_spectral_workspace_bytes(self.shapes, M), dtype=torch.uint8,
                                       device=dev)
        if self.polar:
            self.vote = [torch.empty((r, L.signmuon_x_ld(c)), dtype=torch.bfloat16, device=dev)
                         for (r, c) in self.shapes]
            n = len(self.shapes)
            self.nnz = torch.zeros(max(n, 2), dtype=torch.int64, device=dev)
            self.vote_inv = torch.zeros(max(n, 4), dtype=torch.float32, device=dev)
            full1 = L.signmuon_newton_schulz_workspace_bytes(self.shapes, 1)
            min1 = L.signmuon_newton_schulz_workspace_bytes(self.shapes, 1, minimal=True)
            self.ws_polar = torch.empty(max(min1, min(full1, ns_workspace_cap)), dtype=torch.uint8,
                                        device=dev)

    # ------------------------------------------------------------------
    def state_dict(self):
        return {"mom": [m.clone() for m in self.mom]}

    def load_state_dict(self, sd):
        for dst, src in zip(self.mom, sd["mom"]):
            dst.copy_(src)

    # ------------------------------------------------------------------
    def momentum_norm(self, grads: Sequence[torch.Tensor], stream: int) -> None:
        gdt = self.w_dtype
        gptr = []
        for u, g in enumerate(grads):
            r, c = self.shapes[u // self.n_workers]
            gptr.append(_check_buf(g, (r, c), gdt, f"grad[{u}]"))
        if self.fused_sign:
            L.signmuon_momentum_sign(self.shapes, self.n_workers, _dtype_code(gdt), gptr,
                                     [m.data_ptr() for m in self.mom], self.beta, self.variant == "int8",
                                     [x.data_ptr() for x in self.signs], self.inv_norm.data_ptr(),
                                     self.ws_mom.data_ptr(), self.ws_mom.numel(), stream)
            return
        L.signmuon_momentum_norm(self.shapes, self.n_workers, _dtype_code(gdt), gptr,
                                 [m.data_ptr() for m in self.mom], self.beta,
                                 [x.data_ptr() for x in self.x], self.inv_norm.data_ptr(),
                                 self.ws_mom.data_ptr(), self.ws_mom.numel(), stream)
        if self.norm == "spectral":
            L.signmuon_spectral_norm(self.shapes, self.n_workers, [x.data_ptr() for x in self.x],
                                     self.spectral_iters, self.inv_norm.data_ptr(), self.ws_spec.data_ptr(),
                                     self.ws_spec.numel(), stream)

    def newton_schulz(self, stream: int, out_mode: Optional[int] = None, outs=None) -> None:
        if self.fused_sign:
            if out_mode is not None or outs is not None:
                raise RuntimeError("k = 0 runs fused into the momentum call: there is no separate output")
            return                      # the signs were written by momentum_norm
        self._ns_plan_for(stream, out_mode, outs)
        a, b, c = self.coeffs
        L.signmuon_newton_schulz_run(self._ns_plan, self.k, a, b, c, 0.0, stream)

    def _ns_plan_for(self, stream: int, out_mode: Optional[int], outs) -> None:
        if self.fused_sign:
            return
        # The unit table (tensor maps, buffer addresses) is built once per set
        # of output buffers; every later call only launches the iterations.
        if out_mode is None:
            out_mode = L.SIGNMUON_OUT_PACK1 if self.variant == "pack1" else L.SIGNMUON_OUT_INT8
        optrs = [o.data_ptr() for o in (self.signs if outs is None else outs)]
        key = (out_mode, tuple(optrs))
        if self._ns_plan_key != key:
            self._ns_plan = L.signmuon_newton_schulz_plan(
                self.shapes, self.n_workers, [x.data_ptr() for x in self.x], self.inv_norm.data_ptr(),
                out_mode, optrs, L.SIGNMUON_F32, None, self.ws_ns.data_ptr(), self.ws_ns.numel(), stream,
                plan=self._ns_plan)
            self._ns_plan_key = key

    def _polar_plan_for(self, wptr, stream: int) -> None:
        key = tuple(wptr)
        if self._polar_plan_key != key:
            self._polar_plan = L.signmuon_newton_schulz_plan(
                self.shapes, 1, [v.data_ptr() for v in self.vote], self.vote_inv.data_ptr(),
                L.SIGNMUON_OUT_UPDATE_W, None, _dtype_code(self.w_dtype), wptr, self.ws_polar.data_ptr(),
                self.ws_polar.numel(), stream, plan=self._polar_plan)
            self._polar_plan_key = key

    def vote_update(self, weights: Sequence[torch.Tensor], stream: int) -> None:
        wptr = [_check_buf(w, s, self.w_dtype, f"weight[{i}]")
                for i, (w, s) in enumerate(zip(weights, self.shapes))]
        sptr = [s.data_ptr() for s in self.signs]
        int8_in = self.variant == "int8"
        if not self.polar:
            L.signmuon_vote_update(self.shapes, self.n_workers, int8_in, sptr, _dtype_code(self.w_dtype),
                                   wptr, self.eta, None, 0, 0, self.ws_vote.data_ptr(),
                                   self.ws_vote.numel(), stream)
            return
        L.signmuon_vote_update(self.shapes, self.n_workers, int8_in, sptr, _dtype_code(self.w_dtype),
                               None, self.eta, [v.data_ptr() for v in self.vote], self.nnz.data_ptr(),
                               self.vote_inv.data_ptr(), self.ws_vote.data_ptr(), self.ws_vote.numel(),
                               stream)
        self._polar_plan_for(wptr, stream)
        a, b, c = self.coeffs
        L.signmuon_newton_schulz_run(self._polar_plan, 1, a, b, c, self.eta, stream)

    def prepare(self, weights: Sequence[torch.Tensor]) -> None:
        """Builds the Newton-Schulz plans (and the local polar step's plan for
        these weight tensors) without running a step, on the current stream."""
        stream = torch.cuda.current_stream(self.device).cuda_stream
        self._ns_plan_for(stream, None, None)
        if self.polar:
            wptr = [_check_buf(w, s, self.w_dtype, f"weight[{i}]")
                    for i, (w, s) in enumerate(zip(weights, self.shapes))]
            self._polar_plan_for(wptr, stream)

    def capture(self, weights: Sequence[torch.Tensor], grads: Sequence[torch.Tensor]) -> "torch.cuda.CUDAGraph":
        """Captures one step over these weight and gradient tensors into a CUDA
        graph: graph.replay() then runs a whole step (every kernel of it, the
        descriptor uploads included) with one launch from the host, on the
        values the tensors hold at that time.  The tensors must stay allocated
        and in place while the graph is used.  Capturing runs nothing."""
        if len(weights) != len(self.shapes) or len(grads) != self.units:
            raise ValueError("expected one weight per matrix and one gradient per (matrix, worker)")
        self.prepare(weights)
        cur = torch.cuda.current_stream(self.device)
        side = torch.cuda.Stream(self.device)
        side.wait_stream(cur)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=side):
            self.step(weights, grads)
        cur.wait_stream(side)
        return graph

    def step(self, weights: Sequence[torch.Tensor], grads: Sequence[torch.Tensor]) -> None:
        """One optimizer step: updates `weights` (one tensor per matrix) in place
        from `grads` (n_mats * n_workers tensors, index i * n_workers + m)."""
        if len(weights) != len(self.shapes) or len(grads) != self.units:
            raise ValueError("expected one weight per matrix and one gradient per (matrix, worker)")
        stream = torch.cuda.current_stream(self.device).cuda_stream
        self.momentum_norm(grads, stream)
        self.newton_schulz(stream)
        self.vote_update(weights, stream)

    def kernel_launches_per_step(self) -> int:
        """Number of libsignmuon kernels one step enqueues once the Newton-Schulz
        plans exist (from the second step on; the momentum and vote unit tables
        are still uploaded every step)."""
        def uploads(nbytes):
            return max(1, -(-nbytes // (32768 - 512)))
        M = self.n_workers
        n_mats = len(self.shapes)
        mom = uploads(self.units * 56) + 2
        if self.norm == "spectral":
            # Unit table + segment tables in one upload; per iteration the
            # segment pass (widths that are multiples of 8 up to 4096), the
            # row-block pass (other widths) and the reduction.
            def al(x):
                return -(-x // 256) * 256
            seg_w = [(-(-r // 128)) * M for (r, c) in self.shapes if c % 8 == 0 and c <= 4096]
            n_seg, has_rb = sum(seg_w), len(seg_w) < n_mats
            mom += uploads(al(self.units * 48) + al(n_seg * 4) + al(513 * 4)) + 1
            mom += self.spectral_iters * (int(n_seg > 0) + int(has_rb) + 1)
        ns_waves = 0 if self.fused_sign else self._waves(self.shapes, M, self.ws_ns.numel())
        ns = 0 if self.fused_sign else (3 * self.k if self.k > 0 else 1) * ns_waves
        vote = uploads(-(-n_mats * 64 // 256) * 256 + self.units * 8) + 1
        total = mom + ns + vote
        if self.polar:
            total += 1  # 1/sqrt(nnz) kernel (the nnz clear is a memset, not a kernel)
            total += 3 * self._waves(self.shapes, 1, self.ws_polar.numel())
        return total

    @staticmethod
    def _waves(shapes, M, ws_bytes) -> int:
        """Waves the library splits the units into for this workspace size
        (its buffers per unit: A, B' and an X copy, 1 KB aligned)."""
        def al(x, a):
            return (x + a - 1) // a * a

        def unit_bytes(r, c):
            s = min(r, c)
            return 2 * al(s * al(s, 8) * 2, 1024) + al(r * al(c, 8) * 2, 1024)
        # The minimal workspace is the tables plus the largest unit's buffers.
        tables = (L.signmuon_newton_schulz_workspace_bytes(shapes, M, minimal=True)
                  - max(unit_bytes(r, c) for r, c in shapes))
        arena = ws_bytes - tables
        waves, used = 0, arena
        for (r, c) in shapes:
            b = unit_bytes(r, c)
            for _ in range(M):
                if used + b > arena:
                    waves += 1
                    used = 0
                used += b
        return waves
