"""One step of the path -- rollout capture, guided forward, straight-through
backward, round-to-nearest comparator -- fed from host memory and returned
to it, with the host<->device copies overlapped with the kernels.

The rows are cut into chunks.  The rollout chunks go up first: each one's
maxima are max-accumulated into the per-group amax as soon as it lands
(``trace_capture_amax`` on the first, ``trace_capture_amax_accumulate`` on the
rest), so the global scales are exact before any chunk is quantised.  Then
every chunk is captured with that amax and run through the forwards and the
backward while the training activations and gradients of later chunks are
still arriving, and each finished chunk's outputs go back down on their own
stream while later chunks compute.  Upload, compute and download run on
three streams ordered by events, so both directions of the host link and
the GPU work at the same time.

Plumbing only (buffers, streams, events, copies); every step of the method
runs in libtrace_fp4.so.
"""
from __future__ import annotations

import math

import torch

from . import ops


def _row_quantum(cols: int) -> int:
    """Smallest row count whose slices keep every array's alignment: x 32 B,
    codes 16 B, mantissa bits / mask 16 B, scales 16 B."""
    return 256 // math.gcd(cols, 256)


def row_chunks(rows: int, cols: int, chunks: int) -> list[tuple[int, int]]:
    """Row ranges [a, b) covering 0..rows in about `chunks` pieces, every
    start a multiple of the row quantum (so each chunk's slices of every
    array keep the alignment the calls require); no empty range."""
    q = _row_quantum(cols)
    per = max(q, -(-rows // max(1, chunks)) // q * q)
    cuts = list(range(0, rows, per)) + [rows]
    return [(a, b) for a, b in zip(cuts[:-1], cuts[1:]) if b > a]


class HostStep:
    """The step for one site of shape [rows, cols] (groups by host int64
    offsets, or None), in `chunks` row chunks."""

    OUT_KEYS = ("codes", "mbits", "scales", "gscale", "out", "mask", "grad_in", "out_rtn",
                "mask_rtn")

    def __init__(self, rows: int, cols: int, offsets=None, chunks: int = 8, device="cuda"):
        if cols % 32 or rows < 0:
            raise ops.TraceError("rows >= 0 and cols % 32 == 0 are required")
        self.rows, self.cols = rows, cols
        self.device = torch.device(device)
        self.offsets_h = None if offsets is None else torch.as_tensor(offsets, dtype=torch.int64)
        self.G = 1 if offsets is None else int(self.offsets_h.numel()) - 1
        self.cuts = row_chunks(rows, cols, chunks)
        # chunk-local group offsets (the group ids stay global)
        self.chunk_offs = []
        for a, b in self.cuts:
            if self.offsets_h is None:
                self.chunk_offs.append(None)
            else:
                lo = (self.offsets_h - a).clamp(0, b - a)
                self.chunk_offs.append(lo.to(self.device))
        n, dev = rows * cols, self.device
        bf = torch.bfloat16
        self.xr = torch.empty(rows, cols, dtype=bf, device=dev)
        self.xt = torch.empty(rows, cols, dtype=bf, device=dev)
        self.g = torch.empty(rows, cols, dtype=bf, device=dev)
        self.d = {"codes": torch.empty(n // 2, dtype=torch.uint8, device=dev),
                  "mbits": torch.empty(n // 32, dtype=torch.int32, device=dev),
                  "scales": torch.empty(rows, cols // 16, dtype=torch.uint8, device=dev),
                  "gscale": torch.empty(self.G, dtype=torch.float32, device=dev),
                  "out": torch.empty(rows, cols, dtype=bf, device=dev),
                  "mask": torch.empty(n // 32, dtype=torch.int32, device=dev),
                  "grad_in": torch.empty(rows, cols, dtype=bf, device=dev),
                  "out_rtn": torch.empty(rows, cols, dtype=bf, device=dev),
                  "mask_rtn": torch.empty(n // 32, dtype=torch.int32, device=dev)}
        self.amax = torch.empty(self.G, dtype=torch.int32, device=dev)
        self.up = torch.cuda.Stream(dev)
        self.comp = torch.cuda.Stream(dev)
        self.down = torch.cuda.Stream(dev)

    def alloc_host(self) -> dict:
        """Pinned host tensors for the outputs, shaped like the device ones."""
        return {k: torch.empty(v.shape, dtype=v.dtype, pin_memory=True) for k, v in self.d.items()}

    def _slices(self, a: int, b: int):
        c = self.cols
        return {"codes": slice(a * c // 2, b * c // 2), "mbits": slice(a * c // 32, b * c // 32),
                "scales": slice(a, b), "out": slice(a, b), "mask": slice(a * c // 32, b * c // 32),
                "grad_in": slice(a, b), "out_rtn": slice(a, b),
                "mask_rtn": slice(a * c // 32, b * c // 32)}

    def run(self, x_roll_h: torch.Tensor, x_train_h: torch.Tensor, grad_h: torch.Tensor,
            out_h: dict, stream: torch.cuda.Stream | None = None) -> None:
        """Enqueue the step: inputs from pinned host tensors [rows, cols] bf16,
        outputs into `out_h` (see alloc_host).  Ordered after the work already
        on `stream` (default: the current stream), and `stream` waits for the
        last download, so an event recorded on it afterwards marks the end."""
        caller = torch.cuda.current_stream(self.device) if stream is None else stream
        start = torch.cuda.Event()
        start.record(caller)
        self.up.wait_event(start)
        self.comp.wait_event(start)
        self.down.wait_event(start)
        G, C = self.G, self.cols
        have_roll, have_train, done = [], [], []
        with torch.cuda.stream(self.up):
            for a, b in self.cuts:
                self.xr[a:b].copy_(x_roll_h[a:b], non_blocking=True)
                e = torch.cuda.Event()
                e.record(self.up)
                have_roll.append(e)
            for a, b in self.cuts:
                self.xt[a:b].copy_(x_train_h[a:b], non_blocking=True)
                self.g[a:b].copy_(grad_h[a:b], non_blocking=True)
                e = torch.cuda.Event()
                e.record(self.up)
                have_train.append(e)
        s = self.comp
        for i, (a, b) in enumerate(self.cuts):
            s.wait_event(have_roll[i])
            fn = ops.trace_capture_amax if i == 0 else ops.trace_capture_amax_accumulate
            fn(self.xr[a:b], b - a, C, G, self.chunk_offs[i], self.amax, s)
        d = self.d
        captured = []
        for i, (a, b) in enumerate(self.cuts):
            sl = self._slices(a, b)
            o = self.chunk_offs[i]
            ops.trace_capture_with_amax(self.xr[a:b], b - a, C, G, o, self.amax,
                                        d["codes"][sl["codes"]], d["mbits"][sl["mbits"]],
                                        d["scales"][sl["scales"]], d["gscale"],
                                        ops.TRACE_SCALES_ROW_MAJOR, s)
            e = torch.cuda.Event()
            e.record(s)
            captured.append(e)
            s.wait_event(have_train[i])
            ops.trace_guided_fq_fwd(self.xt[a:b], b - a, C, G, o, d["mbits"][sl["mbits"]],
                                    d["scales"][sl["scales"]], d["gscale"], d["out"][a:b],
                                    d["mask"][sl["mask"]], s)
            ops.trace_fq_bwd(self.g[a:b], d["mask"][sl["mask"]], (b - a) * C, d["grad_in"][a:b], s)
            ops.trace_rtn_fq_fwd(self.xt[a:b], b - a, C, G, o, d["scales"][sl["scales"]],
                                 d["gscale"], d["out_rtn"][a:b], d["mask_rtn"][sl["mask_rtn"]], s)
            e = torch.cuda.Event()
            e.record(s)
            done.append(e)
        # each chunk's capture outputs go down as soon as it is captured (they
        # need only the rollout side), the forward / backward outputs after
        early = ("codes", "mbits", "scales")
        with torch.cuda.stream(self.down):
            for i, (a, b) in enumerate(self.cuts):
                sls = self._slices(a, b)
                self.down.wait_event(captured[i])
                for k in early:
                    out_h[k][sls[k]].copy_(d[k][sls[k]], non_blocking=True)
                self.down.wait_event(done[i])
                for k, sl in sls.items():
                    if k not in early:
                        out_h[k][sl].copy_(d[k][sl], non_blocking=True)
            out_h["gscale"].copy_(d["gscale"], non_blocking=True)
        end = torch.cuda.Event()
        end.record(self.down)
        caller.wait_event(end)
