"""Request-sharded DSpark round across ranks (one process per GPU).

Drafting, confidence and verification are independent per request, so each
rank runs them on its own shard of the batch.  The scheduler's admission is
global -- one budget, one sorted list of every request's candidates (menfem.com
KB entry on DSpark, "Key Contributions": a greedy global sort of candidate
tokens) -- so the round has one exchange: every rank all-gathers the B_local x
G survivals, runs the same deterministic scheduler over the whole batch (the
gathered rows in rank order are the global requests b = rank * B_local + b_local)
and keeps its own requests' admitted lengths.  Every step runs in the
library's kernels; the collective is torch.distributed (NCCL over NVLink on
GPUs, gloo on CPU for tests).
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import _lib


def gather_survivals(S_local: torch.Tensor, group=None) -> torch.Tensor:
    """All-gather the [B_local, G] survivals of every rank into one
    [world * B_local, G] tensor, rank-major, on S_local's device."""
    world = dist.get_world_size(group)
    out = torch.empty((world * S_local.shape[0], S_local.shape[1]), dtype=S_local.dtype, device=S_local.device)
    if dist.get_backend(group) == "nccl":
        dist.all_gather_into_tensor(out, S_local.contiguous(), group=group)
    else:
        dist.all_gather(list(out.chunk(world, dim=0)), S_local.contiguous(), group=group)
    return out


def local_slice(ell_all: torch.Tensor, rank: int, B_local: int) -> torch.Tensor:
    """This rank's requests' admitted lengths from the global ones."""
    return ell_all[rank * B_local:(rank + 1) * B_local]


class ShardedRound:
    """A DeviceRound on this rank's requests plus the global scheduler state.

    knots_n / knots_t / budget describe the whole batch's verify step (the
    admission is one decision over world * B_local requests)."""

    def __init__(self, local, knots_n, knots_t, budget: int, mode: int, group=None):
        self.local = local
        self.group = group
        self.rank = dist.get_rank(group)
        self.world = dist.get_world_size(group)
        dev = local.device
        B, G = local.B, local.G
        self.B_all = self.world * B
        ws_bytes = _lib.dspark_schedule_workspace_size(self.B_all, G)
        if ws_bytes == 0:
            raise ValueError("global batch outside the scheduler's limits")
        self.ws = torch.zeros((ws_bytes + 255) // 256 * 256, dtype=torch.uint8, device=dev)
        self.knots_n = torch.as_tensor(knots_n, dtype=torch.int32).to(dev)
        self.knots_t = torch.as_tensor(knots_t, dtype=torch.float64).to(dev)
        self.budget, self.mode = int(budget), int(mode)
        i32 = dict(dtype=torch.int32, device=dev)
        self.ell_all = torch.zeros(self.B_all, **i32)
        self.n_adm = torch.zeros(1, **i32)
        self.theta = torch.zeros(1, dtype=torch.float64, device=dev)
        self.order = torch.zeros(self.B_all * G, **i32)
        self.S_all = None

    def run(self, stream=None):
        lr = self.local
        t, o = lr.t, lr.o
        _lib.dspark_draft_markov(t["L"], t["U"], t["Wt"], t["x0"], t["temp"], t["u_draft"], lr.ws,
                                 o["x"], o["pd_x"], o["rowmax"], o["rowsum"], stream)
        _lib.dspark_confidence(t["h"], t["w"], float(lr.inp.bias), t["tau"], o["c"], o["S"], stream)
        with torch.cuda.stream(stream) if stream is not None else _null():
            self.S_all = gather_survivals(o["S"], self.group)
        _lib.dspark_schedule(self.S_all, self.knots_n, self.knots_t, self.budget, self.mode, self.ws,
                             self.ell_all, self.n_adm, self.theta, self.order, stream)
        with torch.cuda.stream(stream) if stream is not None else _null():
            o["ell"].copy_(local_slice(self.ell_all, self.rank, lr.B))
        _lib.dspark_verify(t["Tlog"], t["L"], t["U"], t["Wt"], t["x0"], o["x"], o["pd_x"], o["rowmax"],
                           o["rowsum"], t["temp"], t["u_accept"], t["u_final"], o["ell"], lr.ws, o["acc"],
                           o["tokens"], o["nout"], o["pt_x"], stream)


class _null:
    def __enter__(self):
        return None

    def __exit__(self, *a):
        return False
