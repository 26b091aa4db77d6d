"""The production form of DSpark's scheduler across a sequence of rounds.

paperlayer.ai summary of DSpark, §5.2 Production Scheduler: the scheduler
runs asynchronously; the capacity limit comes from historical predictions,
the current candidates are ranked by their latest cumulative confidence, and
a dynamic top-K selection keeps the confidence ordering while hiding the
scheduling latency; the capacity's global search copes with irregular
hardware-capacity curves.  The same page (its note on production scheduling)
asks that this fit discrete hardware capacity and continuous CUDA-graph
replay.

Here, per round t:
  * capacity step (side stream, enqueued when the round starts, so it overlaps
    drafting): ``dspark_schedule`` in the global-search mode on round t-1's
    survivals writes its admitted count into a device int32, the capacity;
  * selection step (the round's stream, after confidence):
    ``dspark_schedule_topk`` admits the first K of round t's candidates in the
    stable order by survival, K read from that device int32 when the kernel
    runs (one captured graph serves every capacity);
  * the round's survivals are kept for the next round's capacity step.
The first round has no history: its capacity is Algorithm 1's own admitted
count on its survivals (early stop), computed on the round's stream.
Every step runs in libdspark's kernels; this module only orders them.
"""
from __future__ import annotations

import torch

from . import _lib


class ProductionScheduler:
    def __init__(self, B: int, G: int, knots_n, knots_t, budget: int = -1, device="cuda"):
        dev = torch.device(device)
        self.B, self.G, self.budget, self.device = B, G, int(budget), dev
        self.knots_n = torch.as_tensor(knots_n, dtype=torch.int32).to(dev)
        self.knots_t = torch.as_tensor(knots_t, dtype=torch.float64).to(dev)
        n = _lib.dspark_schedule_workspace_size(B, G)
        if n == 0:
            raise ValueError("batch outside the scheduler's limits")
        # Two workspaces: the capacity step and the selection may run at once.
        self.ws_cap = torch.zeros((n + 255) // 256 * 256, dtype=torch.uint8, device=dev)
        self.ws_sel = torch.zeros_like(self.ws_cap)
        i32 = dict(dtype=torch.int32, device=dev)
        self.capacity = torch.zeros(1, **i32)
        self.S_hist = torch.zeros((B, G), dtype=torch.float32, device=dev)
        self._ell_cap = torch.zeros(B, **i32)
        self._theta = torch.zeros(1, dtype=torch.float64, device=dev)
        self.side = torch.cuda.Stream(device=dev)
        self.cap_ready = torch.cuda.Event()
        self.has_history = False

    def start_round(self, stream):
        """Enqueue the capacity step for this round on the side stream (after
        everything already on `stream`, so the kept survivals are final)."""
        if not self.has_history:
            return
        self.side.wait_stream(stream)
        _lib.dspark_schedule(self.S_hist, self.knots_n, self.knots_t, self.budget, _lib.SCHED_GLOBAL_ARGMAX,
                             self.ws_cap, self._ell_cap, self.capacity, self._theta, None, self.side)
        self.cap_ready.record(self.side)

    def select(self, S, ell_out, n_adm_out, order_out=None, stream=None):
        """Admit this round's candidates (top-K of S by the capacity) and keep
        S for the next round's capacity step."""
        stream = torch.cuda.current_stream(self.device) if stream is None else stream
        if self.has_history:
            stream.wait_event(self.cap_ready)
        else:
            _lib.dspark_schedule(S, self.knots_n, self.knots_t, self.budget, _lib.SCHED_GREEDY_EARLY_STOP,
                                 self.ws_sel, self._ell_cap, self.capacity, self._theta, None, stream)
        _lib.dspark_schedule_topk(S, self.capacity, self.budget, self.ws_sel, ell_out, n_adm_out, order_out,
                                  stream)
        with torch.cuda.stream(stream):
            self.S_hist.copy_(S)
        self.has_history = True

    def device_status(self) -> int:
        return _lib.dspark_get_device_status(self.ws_sel) | _lib.dspark_get_device_status(self.ws_cap)


class ProductionRound:
    """A DeviceRound whose scheduling stage is the production scheduler."""

    def __init__(self, dr, sched: ProductionScheduler):
        self.dr, self.sched = dr, sched

    def run(self, stream=None):
        dr, t, o = self.dr, self.dr.t, self.dr.o
        st = torch.cuda.current_stream(dr.device) if stream is None else stream
        self.sched.start_round(st)
        _lib.dspark_draft_markov(t["L"], t["U"], t["Wt"], t["x0"], t["temp"], t["u_draft"], dr.ws,
                                 o["x"], o["pd_x"], o["rowmax"], o["rowsum"], st)
        _lib.dspark_confidence(t["h"], t["w"], float(dr.inp.bias), t["tau"], o["c"], o["S"], st)
        self.sched.select(o["S"], o["ell"], o["n_adm"], o["order"], st)
        _lib.dspark_verify(t["Tlog"], t["L"], t["U"], t["Wt"], t["x0"], o["x"], o["pd_x"], o["rowmax"],
                           o["rowsum"], t["temp"], t["u_accept"], t["u_final"], o["ell"], dr.ws, o["acc"],
                           o["tokens"], o["nout"], o["pt_x"], st)
