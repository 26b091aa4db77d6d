"""One DSpark round on the device: buffers plus the four library calls.

``DeviceRound`` owns the device copies of a round's inputs, its outputs and
one workspace, and enqueues drafting, confidence, scheduling and
verification on a stream (all four run in libdspark's kernels).  The same
object can refresh its inputs from pinned host memory for end-to-end timing.
"""
from __future__ import annotations

import numpy as np
import torch

from . import _lib, synth
from .synth import RoundInputs


def _dev(arr: np.ndarray, dtype: str, device) -> torch.Tensor:
    """fp32 numpy array (or bf16 bit patterns) -> device tensor."""
    if dtype == "bf16":
        t = torch.from_numpy(np.ascontiguousarray(arr).view(np.int16)).view(torch.bfloat16)
    else:
        t = torch.from_numpy(np.ascontiguousarray(arr, dtype=np.float32))
    return t.to(device)


class DeviceRound:
    def __init__(self, inp: RoundInputs, knots_n, knots_t, budget: int, mode: int, device="cuda",
                 tau=None, pinned_host: bool = False, Arec=None):
        """Arec: the RNN head's recurrent matrix [r, r] (fp32 values, sent in
        the round's dtype); None drafts with the Markov head."""
        self.inp = inp
        self.B, self.G, self.V, self.r, self.d = inp.B, inp.G, inp.V, inp.r, inp.d
        self.dt = inp.dtype
        dev = torch.device(device)
        self.device = dev
        bits = inp.bits
        src = (lambda k, a: bits[k]) if self.dt == "bf16" else (lambda k, a: a)
        Wt = np.ascontiguousarray(src("W", inp.W).T)  # transition factor stored [V, r]
        host = {
            "L": src("L", inp.L), "Tlog": src("Tlog", inp.Tlog), "U": src("U", inp.U), "Wt": Wt,
            "h": src("h", inp.h), "w": src("w", inp.w),
        }
        if Arec is not None:
            Ar = np.asarray(Arec, np.float32)
            host["Arec"] = synth.bf16_bits(Ar) if self.dt == "bf16" else Ar
        self.rnn = Arec is not None
        self.t = {k: _dev(v, self.dt, dev) for k, v in host.items()}
        small = {"x0": inp.x0.astype(np.int32), "temp": inp.temp.astype(np.float32),
                 "u_draft": inp.u_draft.astype(np.float32), "u_accept": inp.u_accept.astype(np.float32),
                 "u_final": inp.u_final.astype(np.float32)}
        for k, v in small.items():
            self.t[k] = torch.from_numpy(np.ascontiguousarray(v)).to(dev)
        self.t["knots_n"] = torch.from_numpy(np.asarray(knots_n, np.int32)).to(dev)
        self.t["knots_t"] = torch.from_numpy(np.asarray(knots_t, np.float64)).to(dev)
        self.t["tau"] = None if tau is None else torch.from_numpy(np.asarray(tau, np.float32)).to(dev)
        self.budget, self.mode = int(budget), int(mode)
        B, G = self.B, self.G
        f32 = dict(dtype=torch.float32, device=dev)
        i32 = dict(dtype=torch.int32, device=dev)
        self.o = {
            "x": torch.zeros(B, G, **i32), "pd_x": torch.zeros(B, G, **f32),
            "rowmax": torch.zeros(B, G, **f32), "rowsum": torch.zeros(B, G, **f32),
            "c": torch.zeros(B, G, **f32), "S": torch.zeros(B, G, **f32),
            "ell": torch.zeros(B, **i32), "n_adm": torch.zeros(1, **i32),
            "theta": torch.zeros(1, dtype=torch.float64, device=dev), "order": torch.zeros(B * G, **i32),
            "acc": torch.zeros(B, **i32), "tokens": torch.zeros(B, G + 1, **i32), "nout": torch.zeros(B, **i32),
            "pt_x": torch.zeros(B, G, **f32),
        }
        if self.rnn:
            self.o["H"] = torch.zeros(B, G, self.r, **f32)
        dcode = _lib.DSPARK_BF16 if self.dt == "bf16" else _lib.DSPARK_F32
        need = max(_lib.dspark_draft_workspace_size(B, G, self.V, self.r, dcode),
                   _lib.dspark_schedule_workspace_size(B, G),
                   _lib.dspark_verify_workspace_size(B, G, self.V, self.r, dcode))
        if need == 0:
            raise ValueError("round shape outside the library's limits")
        self.ws = torch.zeros((need + 255) // 256 * 256, dtype=torch.uint8, device=dev)
        self._side = None
        self.host = None
        if pinned_host:
            self.host = {k: (v.cpu().pin_memory() if v is not None else None) for k, v in self.t.items()}
            self.host_out = {k: torch.zeros(v.shape, dtype=v.dtype).pin_memory()
                             for k, v in self.o.items() if k in ("tokens", "nout", "ell")}

    # -------------------------------------------------------------- running
    def run(self, stream=None, overlap_confidence: bool = True, verify: bool = True):
        """Enqueue one round on `stream` (default: the current stream).  The
        confidence stage does not depend on the drafted tokens, so by default
        it runs on a side stream forked from `stream` at the start of the
        round and joined before the scheduler (a fork and a join when the
        round is captured in a graph).  verify=False stops after scheduling."""
        t, o = self.t, self.o
        main = torch.cuda.current_stream(self.device) if stream is None else stream
        conf = lambda st: _lib.dspark_confidence(t["h"], t["w"], float(self.inp.bias), t["tau"], o["c"], o["S"], st)
        if overlap_confidence:
            if self._side is None:
                self._side = torch.cuda.Stream(device=self.device)
                self._fork = torch.cuda.Event()
                self._join = torch.cuda.Event()
            self._fork.record(main)
            self._side.wait_event(self._fork)
            conf(self._side)
            self._join.record(self._side)
        self.draft(main)
        if overlap_confidence:
            main.wait_event(self._join)
        else:
            conf(main)
        _lib.dspark_schedule(o["S"], t["knots_n"], t["knots_t"], self.budget, self.mode, self.ws, o["ell"],
                             o["n_adm"], o["theta"], o["order"], main)
        if verify:
            self.verify(main)

    # Inputs that change every round and feed drafting, confidence and the
    # draws; the target logits follow once the admitted lengths are known.
    ROUND_INPUTS = ("L", "h", "x0", "temp", "u_draft", "u_accept", "u_final")

    def run_from_host(self, stream=None, overlap_confidence: bool = True):
        """Enqueue one round fed from pinned host memory, the way a serving
        loop drives it: the round's draft-side inputs are copied in, drafting,
        confidence and scheduling run, one kernel pulls in the target rows
        that verification reads -- rows 0..ell_b of request b, what a target
        forward over the admitted tokens produces -- reading ell on the
        device, verification runs, and the emitted tokens, counts and lengths
        go to pinned host memory (``host_out``).  Nothing waits on the host;
        synchronise `stream` before reading ``host_out`` or calling
        ``host_round_bytes``."""
        if self.host is None:
            raise RuntimeError("run_from_host needs DeviceRound(..., pinned_host=True)")
        main = torch.cuda.current_stream(self.device) if stream is None else stream
        with torch.cuda.stream(main):
            for k in self.ROUND_INPUTS:
                self.t[k].copy_(self.host[k], non_blocking=True)
            self.run(main, overlap_confidence, verify=False)
            _lib.dspark_gather_admitted_targets(self.host["Tlog"], self.t["Tlog"], self.o["ell"], main)
            self.verify(main)
        self.download(main)

    def host_round_bytes(self):
        """(host-to-device, device-to-host) bytes of the last run_from_host,
        from the admitted lengths it brought back (synchronise first)."""
        ell = self.host_out["ell"].numpy().astype(np.int64)
        tl = self.host["Tlog"]
        h2d = sum(self.host[k].numel() * self.host[k].element_size() for k in self.ROUND_INPUTS)
        h2d += int((ell + 1).sum()) * tl.shape[2] * tl.element_size()
        return h2d, self.d2h_bytes()

    def draft(self, stream=None):
        """The drafting stage alone (Markov or RNN head)."""
        t, o = self.t, self.o
        if self.rnn:
            _lib.dspark_draft_rnn(t["L"], t["U"], t["Arec"], t["Wt"], t["x0"], t["temp"], t["u_draft"], self.ws,
                                  o["x"], o["pd_x"], o["rowmax"], o["rowsum"], o["H"], stream)
        else:
            _lib.dspark_draft_markov(t["L"], t["U"], t["Wt"], t["x0"], t["temp"], t["u_draft"], self.ws,
                                     o["x"], o["pd_x"], o["rowmax"], o["rowsum"], stream)

    def verify(self, stream=None):
        """The verification stage alone, on the admitted lengths in o["ell"]."""
        t, o = self.t, self.o
        if self.rnn:
            _lib.dspark_verify_rnn(t["Tlog"], t["L"], o["H"], t["Wt"], o["x"], o["pd_x"], o["rowmax"],
                                   o["rowsum"], t["temp"], t["u_accept"], t["u_final"], o["ell"], self.ws,
                                   o["acc"], o["tokens"], o["nout"], o["pt_x"], stream)
        else:
            _lib.dspark_verify(t["Tlog"], t["L"], t["U"], t["Wt"], t["x0"], o["x"], o["pd_x"], o["rowmax"],
                               o["rowsum"], t["temp"], t["u_accept"], t["u_final"], o["ell"], self.ws, o["acc"],
                               o["tokens"], o["nout"], o["pt_x"], stream)

    def upload(self, stream=None):
        """Copy every input from pinned host memory (end-to-end timing)."""
        with torch.cuda.stream(stream) if stream is not None else _null():
            for k, v in self.host.items():
                if v is not None:
                    self.t[k].copy_(v, non_blocking=True)

    def download(self, stream=None):
        """Copy the emitted tokens and counts to pinned host memory."""
        with torch.cuda.stream(stream) if stream is not None else _null():
            for k, v in self.host_out.items():
                v.copy_(self.o[k], non_blocking=True)

    def h2d_bytes(self) -> int:
        return sum(v.numel() * v.element_size() for v in self.host.values() if v is not None)

    def d2h_bytes(self) -> int:
        return sum(v.numel() * v.element_size() for v in self.host_out.values())

    def outputs(self) -> dict:
        return {k: v.cpu().numpy() for k, v in self.o.items()}

    def device_status(self) -> int:
        return _lib.dspark_get_device_status(self.ws)


class _null:
    def __enter__(self):
        return None

    def __exit__(self, *a):
        return False
