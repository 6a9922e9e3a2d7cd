"""Per-layer hot-set manager (DynaExq, arXiv 2511.15015, abstract): expert
hotness from router traces, a budget-feasible hot set per layer, promotion and
demotion by swapping stable handles to fully materialised versions, without
putting the copies on the critical path.

The arithmetic and the decisions run on the device, in the library:
  - every forward adds its per-expert selection counts to a device counter
    (moe_layer_set_hotness_counter);
  - at the end of a counting window, moe_select_hot_experts picks the n hottest
    experts (ties to the lower id) on the compute stream and clears the counts;
  - moe_apply_hot_set swaps the layer's handle table to BF16 slots for the hot
    experts and to the base (INT8/INT4) versions for every other expert.
This module only orders the work: it issues the host->device copies of the
newly hot experts' BF16 weights into the idle set of slots on a side stream,
once the selection's event has completed (checked with a non-blocking query,
so the host never waits), and enqueues the swap on the compute stream once the
copies' event has completed.  The compute stream never waits on a copy in
flight; a promotion simply takes effect at the first step after its copies
are done.  Two sets of slots alternate: forwards keep reading the active set
while the other one is filled.
"""
from __future__ import annotations

import numpy as np
import torch

from . import binding as B


class PrecisionManager:
    """Hot-set management of one MoELayer whose experts all have a base
    (INT8/INT4) version installed.

    masters: per expert (w13, w2) bf16 CPU tensors in pinned memory (the BF16
        versions a promotion copies in).
    n_hot: hot-set size, e.g. layer.hot_set_size(budget_bytes).
    """

    def __init__(self, layer: B.MoELayer, masters, n_hot: int, device, copy_stream=None):
        self.layer, self.masters, self.n = layer, masters, int(n_hot)
        self.dev = torch.device(device)
        E, H, I = layer.E, layer.H, layer.I
        self.copy = copy_stream if copy_stream is not None else torch.cuda.Stream(self.dev)
        self.counts = torch.zeros(E, dtype=torch.int32, device=self.dev)
        layer.set_hotness_counter(self.counts)
        self.slots = [[(torch.empty((2 * I, H), dtype=torch.bfloat16, device=self.dev),
                        torch.empty((H, I), dtype=torch.bfloat16, device=self.dev))
                       for _ in range(self.n)] for _ in range(2)]
        layer.set_bf16_slots(self.slots[0] + self.slots[1])   # set s: slots [s n, (s + 1) n)
        self.hot_dev = [torch.zeros(max(1, self.n), dtype=torch.int32, device=self.dev)
                        for _ in range(2)]
        self.hot_host = [torch.zeros(max(1, self.n), dtype=torch.int32).pin_memory()
                         for _ in range(2)]
        self.resident = [dict(), dict()]   # per set: expert -> slot index
        self.active = None                 # set the handles point to (None: base versions)
        self.free_ev = [None, None]        # per set: no forward reads it after this event
        self.sel_ev = None                 # selection of the pending promotion
        self.copy_ev = None                # its copies
        self.target = None                 # set being filled
        self.log = []                      # (step, event, details); swaps carry the hot ids
        self.h2d_bytes = 0

    # -- set-up: an initial hot set (not timed) ------------------------------
    def bootstrap(self, hot_ids, compute):
        """Promote `hot_ids` (host ints, n of them) through slot set 0 before
        the first step, e.g. from a popularity estimate."""
        hot = np.sort(np.asarray(hot_ids, np.int32))[:self.n]
        self.hot_host[0][:len(hot)].copy_(torch.from_numpy(hot))
        with torch.cuda.stream(compute):
            self.hot_dev[0][:len(hot)].copy_(self.hot_host[0][:len(hot)], non_blocking=True)
            for i, e in enumerate(hot.tolist()):
                self.slots[0][i][0].copy_(self.masters[e][0], non_blocking=True)
                self.slots[0][i][1].copy_(self.masters[e][1], non_blocking=True)
        self.layer.apply_hot_set(self.hot_dev[0], len(hot), 0, stream=compute)
        self.resident[0] = {e: i for i, e in enumerate(hot.tolist())}
        self.active, self.applied_hot = 0, hot
        self.log.append((0, "bootstrap", hot.copy()))

    # -- one counting window ends: select on the device ---------------------
    def end_window(self, step: int, compute):
        """Select the hot set from the counts of the window that just ended
        (and start a new one), unless a promotion is still in flight."""
        if self.target is not None:
            self.log.append((step, "skip", "promotion in flight"))
            return False
        t = 0 if self.active is None else 1 - self.active
        B.moe_select_hot_experts(self.counts, self.n, zero_counts=True, hot_ids=self.hot_dev[t],
                                 stream=compute)
        with torch.cuda.stream(compute):
            self.hot_host[t].copy_(self.hot_dev[t], non_blocking=True)
            self.sel_ev = torch.cuda.Event()
            self.sel_ev.record(compute)
        self.target = t
        self.log.append((step, "select", t))
        return True

    # -- every step: advance the pipeline without blocking ------------------
    def poll(self, step: int, compute):
        """Issue the copies once the selection is known, and the swap once the
        copies are done.  Returns True if a swap was enqueued at this step."""
        if self.target is None:
            return False
        t = self.target
        if self.copy_ev is None:
            if not self.sel_ev.query():
                return False
            hot = self.hot_host[t][:self.n].numpy().copy()
            src_set = self.active
            with torch.cuda.stream(self.copy):
                if self.free_ev[t] is not None:
                    self.copy.wait_event(self.free_ev[t])
                new_res = {}
                for i, e in enumerate(hot.tolist()):
                    d13, d2 = self.slots[t][i]
                    if src_set is not None and e in self.resident[src_set]:
                        j = self.resident[src_set][e]      # already BF16 on the device
                        s13, s2 = self.slots[src_set][j]
                        d13.copy_(s13, non_blocking=True)
                        d2.copy_(s2, non_blocking=True)
                    else:
                        m13, m2 = self.masters[e]
                        d13.copy_(m13, non_blocking=True)
                        d2.copy_(m2, non_blocking=True)
                        self.h2d_bytes += (m13.numel() + m2.numel()) * 2
                    new_res[e] = i
                self.copy_ev = torch.cuda.Event()
                self.copy_ev.record(self.copy)
            self.resident[t] = new_res
            self.pending_hot = hot
            self.log.append((step, "copies", len(hot)))
            return False
        if not self.copy_ev.query():
            return False
        compute.wait_event(self.copy_ev)   # complete: orders the swap after the copies
        self.layer.apply_hot_set(self.hot_dev[t], self.n, t * self.n, stream=compute)
        if self.active is not None:
            ev = torch.cuda.Event()
            ev.record(compute)             # forwards enqueued before this read the old set
            self.free_ev[self.active] = ev
        self.active = t
        self.applied_hot = self.pending_hot
        self.target, self.sel_ev, self.copy_ev = None, None, None
        self.log.append((step, "swap", np.sort(self.applied_hot)))
        return True

    def hot_experts(self):
        """Sorted expert ids the handles point to BF16 slots for (host view)."""
        return np.array([]) if self.active is None else np.sort(self.applied_hot)

    def close(self):
        self.layer.set_hotness_counter(None)
