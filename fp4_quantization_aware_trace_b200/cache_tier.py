"""Cache tier: carries each site's compact cache from the rollout to the
trainer through pinned host memory.

The TRACE post (rcap.io, "TRACE: Rollout-Guided Quantization-Aware Training
for FP4") keeps, per capture site, one mantissa bit per element plus the
scales, and only for the deeper half of the layers (compact-cache paragraph;
the ablation keeps the latter 20 of 40 layers); its stack-and-caveats list
asks for a rollout engine that emits these per-site records, a tier that
holds them and a trainer that reads them back.  This module is that tier on
one GPU:

* ``CacheTier.capture`` runs the library's capture with the mantissa bits,
  block scales and global scales written into ONE device record
  (``trace_cache_record_bytes`` lays it out), then queues a single
  device-to-host copy of the record on a dedicated copy stream, ordered
  after the capture by an event, so the copy overlaps whatever the compute
  stream does next.  Device records come from a small ring per shape; a slot
  is reused only after its previous copy has finished (stream-side wait, no
  host sync).
* ``CacheTier.fetch`` brings a record back (one host-to-device copy on the
  caller's stream, after the device-to-host copy that filled it) and returns
  a ``Capture`` view for ``ops.guided_fq_fwd``.
* Layers outside the kept set are captured without a record: the trainer
  rounds them to nearest with its own scales (plain QAT).

Only plumbing lives here (buffers, streams, events, copies); every step of
the method runs in libtrace_fp4.so.
"""
from __future__ import annotations

import dataclasses
from typing import Hashable

import torch

from . import ops


def kept_layers(num_layers: int, keep: int | None = None) -> range:
    """The deepest `keep` layers (default: the deeper half, as the post's
    ablation keeps layers 20..39 of 40)."""
    if num_layers < 0:
        raise ValueError("num_layers must be >= 0")
    keep = (num_layers + 1) // 2 if keep is None else keep
    if not 0 <= keep <= num_layers:
        raise ValueError("keep must lie in [0, num_layers]")
    return range(num_layers - keep, num_layers)


@dataclasses.dataclass(frozen=True)
class RecordLayout:
    rows: int
    cols: int
    num_groups: int
    nbytes: int
    mbits_offset: int
    scales_offset: int
    gscale_offset: int

    @staticmethod
    def of(rows: int, cols: int, num_groups: int = 1) -> "RecordLayout":
        key = (rows, cols, num_groups)
        lay = _LAYOUTS.get(key)
        if lay is None:
            nb, om, os_, og = ops.trace_cache_record_bytes(rows, cols, num_groups)
            if nb == 0:
                raise ops.TraceError(f"invalid record shape [{rows}, {cols}] x {num_groups} groups")
            lay = _LAYOUTS[key] = RecordLayout(rows, cols, num_groups, nb, om, os_, og)
        return lay

    def view(self, record: torch.Tensor, offsets: torch.Tensor | None = None,
             codes: torch.Tensor | None = None) -> ops.Capture:
        """A Capture whose mbits / scales / gscale alias `record` (uint8)."""
        n = self.rows * self.cols
        if record.dtype != torch.uint8 or record.numel() < self.nbytes:
            raise ops.TraceError("record must be a uint8 tensor of at least nbytes")
        return ops.Capture(
            codes=codes,
            mbits=record[self.mbits_offset:self.mbits_offset + n // 8].view(torch.int32),
            scales=record[self.scales_offset:self.scales_offset + n // 16].view(
                self.rows, self.cols // 16),
            gscale=record[self.gscale_offset:self.gscale_offset + 4 * self.num_groups].view(
                torch.float32),
            offsets=offsets)


_LAYOUTS: dict = {}  # (rows, cols, groups) -> RecordLayout (pure host arithmetic, cached)


@dataclasses.dataclass
class _Held:
    layout: RecordLayout
    host: torch.Tensor           # pinned uint8 [nbytes]
    copied: torch.cuda.Event     # device-to-host copy finished
    offsets: torch.Tensor | None
    fetched: torch.cuda.Event | None = None  # last host-to-device copy of it finished


class CacheTier:
    """Per-site compact-cache records in pinned host memory.

    keys are any hashable (e.g. (trajectory batch, layer, site)); `layer`
    decides whether a site is kept."""

    def __init__(self, num_layers: int, keep: int | None = None, device="cuda",
                 ring: int = 2):
        self.layers = frozenset(kept_layers(num_layers, keep))
        self.device = torch.device(device)
        self.copy_stream = torch.cuda.Stream(self.device)
        self.ring = max(1, int(ring))
        self._slots: dict[RecordLayout, list] = {}
        self._next: dict[RecordLayout, int] = {}
        self._held: dict[Hashable, _Held] = {}
        self._ws: dict[int, torch.Tensor] = {}
        self.d2h_bytes = 0
        self.h2d_bytes = 0

    # -- rollout side -------------------------------------------------------
    def is_kept(self, layer: int) -> bool:
        return layer in self.layers

    def _slot(self, lay: RecordLayout):
        slots = self._slots.setdefault(lay, [])
        i = self._next.get(lay, 0)
        self._next[lay] = (i + 1) % self.ring
        if i == len(slots):
            rec = torch.empty(lay.nbytes, dtype=torch.uint8, device=self.device)
            slots.append([rec, None, {}])  # record, event of its last copy, cached views
        return slots[i]

    def _workspace(self, G: int, rows: int, cols: int) -> torch.Tensor:
        nb = max(ops.trace_capture_workspace_bytes(rows, cols, G), 256)
        ws = self._ws.get(nb)
        if ws is None:
            ws = self._ws[nb] = torch.zeros(nb, dtype=torch.uint8, device=self.device)
        return ws

    def capture(self, key: Hashable, layer: int, x: torch.Tensor,
                offsets: torch.Tensor | None = None, codes: torch.Tensor | None = None,
                stream: torch.cuda.Stream | None = None) -> ops.Capture:
        """Capture one rollout site.  For a kept layer the compact cache goes
        into a device record and is queued for the host under `key`.  Returns
        the Capture (its codes are the rollout's own FP4 codes).  The record
        view it returns is valid until `ring` more captures of the same shape
        have been made."""
        rows, cols = int(x.shape[0]), int(x.shape[1])
        G = 1 if offsets is None else int(offsets.numel()) - 1
        stream = torch.cuda.current_stream(self.device) if stream is None else stream
        if codes is None:
            codes = torch.empty(rows * cols // 2, dtype=torch.uint8, device=self.device)
        if not self.is_kept(layer):
            cap, ws = ops.alloc_capture(rows, cols, G, self.device, offsets)
            cap.codes = codes
            return ops.capture(x, offsets, cap, ws, stream)
        lay = RecordLayout.of(rows, cols, G)
        slot = self._slot(lay)
        if slot[1] is not None:
            stream.wait_event(slot[1])        # the slot's previous copy is done
        views = slot[2]
        vkey = (id(offsets), id(codes))
        cap = views.get(vkey)
        if cap is None or cap.offsets is not offsets or cap.codes is not codes:
            views.clear()
            cap = views[vkey] = lay.view(slot[0], offsets, codes)
        ops.capture(x, offsets, cap, self._workspace(G, rows, cols), stream)
        ready = torch.cuda.Event()
        ready.record(stream)
        held = self._held.get(key)
        if held is None or held.layout != lay:
            if held is not None:
                self.drop(key)
            host = torch.empty(lay.nbytes, dtype=torch.uint8, pin_memory=True)
        else:
            # the same host buffer again: the copy stream runs in order after
            # the copy that filled it; a fetch still reading it must finish
            host = held.host
            if held.fetched is not None:
                self.copy_stream.wait_event(held.fetched)
        copied = torch.cuda.Event()
        self.copy_stream.wait_event(ready)
        with torch.cuda.stream(self.copy_stream):
            host.copy_(slot[0], non_blocking=True)
            copied.record(self.copy_stream)
        slot[1] = copied
        self._held[key] = _Held(lay, host, copied,
                                None if offsets is None else offsets.detach().clone())
        self.d2h_bytes += lay.nbytes
        return cap

    # -- trainer side -------------------------------------------------------
    def has(self, key: Hashable) -> bool:
        return key in self._held

    def fetch(self, key: Hashable, stream: torch.cuda.Stream | None = None,
              out: torch.Tensor | None = None) -> ops.Capture:
        """Bring the record of `key` to the device (one copy on `stream`,
        after the copy that filled it) and return its Capture view (codes
        None: the 1-bit guided forward does not read them)."""
        held = self._held[key]
        stream = torch.cuda.current_stream(self.device) if stream is None else stream
        stream.wait_event(held.copied)
        with torch.cuda.stream(stream):
            rec = (torch.empty(held.layout.nbytes, dtype=torch.uint8, device=self.device)
                   if out is None else out)
            rec.copy_(held.host, non_blocking=True)
            held.fetched = torch.cuda.Event()
            held.fetched.record(stream)
        self.h2d_bytes += held.layout.nbytes
        offs = None if held.offsets is None else held.offsets.to(self.device, non_blocking=True)
        return held.layout.view(rec, offs)

    def host_record(self, key: Hashable) -> torch.Tensor:
        """The pinned host record of `key` (waits for its copy)."""
        held = self._held[key]
        held.copied.synchronize()
        return held.host

    def drop(self, key: Hashable) -> None:
        """Forget `key` and release its host buffer (after its copies)."""
        held = self._held.pop(key)
        held.copied.synchronize()
        if held.fetched is not None:
            held.fetched.synchronize()

    def host_nbytes(self) -> int:
        return sum(h.layout.nbytes for h in self._held.values())

    def synchronize(self) -> None:
        self.copy_stream.synchronize()
