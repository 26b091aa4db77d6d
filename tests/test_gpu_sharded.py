"""The request-sharded round on the GPU: with one rank (an NCCL group of
size 1, the only size a one-GPU run can hold) it must reproduce the plain
round exactly -- same draft tokens, admitted lengths and emitted tokens --
since the survival all-gather then returns this rank's own survivals."""
import datetime
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist

from speculative_decoding_draft_rank_b200 import synth, workloads as wl

pytestmark = pytest.mark.gpu


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_sharded_round_one_rank_matches_plain_round():
    from speculative_decoding_draft_rank_b200.round import DeviceRound
    from speculative_decoding_draft_rank_b200.sharded import ShardedRound
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60), device_id=torch.device("cuda", 0))
    try:
        w = wl.headline()
        B, G, V, r, d = 64, 5, 20000, 256, 512
        temps = np.tile(np.float32([1.0, 0.0, 0.6, 1.2]), B)[:B]
        inp = synth.generate(B, G, V, r, d, "bf16", seed=3, hot=8, temps=temps)
        plain = DeviceRound(inp, w.knots_n, w.knots_t, -1, 1)
        plain.run()
        sh_local = DeviceRound(inp, w.knots_n, w.knots_t, -1, 1)
        sh = ShardedRound(sh_local, w.knots_n, w.knots_t, -1, 1)
        sh.run()
        torch.cuda.synchronize()
        a, b = plain.outputs(), sh_local.outputs()
        for k in ("x", "pd_x", "S", "ell", "acc", "tokens", "nout"):
            assert np.array_equal(a[k], b[k]), k
        assert int(sh.n_adm.item()) == int(a["n_adm"][0])
        assert plain.device_status() == 0 and sh_local.device_status() == 0
    finally:
        dist.destroy_process_group()
