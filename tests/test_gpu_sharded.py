"""The sharded Muon step (whole matrices per rank, LPT partition, one
all-gather per dtype) on the GPU with the library's real C-ABI step.  A
one-rank NCCL process group runs the ownership, the local step and the
gather path exactly as on N GPUs: the collective copies the rank's own slot
in place.  Multi-rank ownership and unpacking are covered with gloo on CPU."""
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist

import matrix_orthogonalizing_optimizer_step_b200 as mo
from matrix_orthogonalizing_optimizer_step_b200 import sharded
from matrix_orthogonalizing_optimizer_step_b200 import workloads as wl
from oracle import muon_oracle as orc
from tests._util import TOL_BF16_RELF, relF, to64

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda", 0)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_sharded_step_one_rank_nccl_matches_step_and_oracle():
    mo.muon_reset_config()
    shapes = [(768, 2304), (768, 768), (3072, 768), (200, 712), (37, 91)]
    G = [wl.make_single(r, c, 5000 + 3 * i, "student_t3", DEV, "bf16", 0.01) for i, (r, c) in enumerate(shapes)]
    M = [wl.make_single(r, c, 5001 + 3 * i, "student_t3", DEV, "bf16", 0.01) for i, (r, c) in enumerate(shapes)]
    W = [wl.make_single(r, c, 5002 + 3 * i, "params", DEV, "f32") for i, (r, c) in enumerate(shapes)]
    Wr, Mr = [t.clone() for t in W], [t.clone() for t in M]
    W64, G64, M64 = [to64(t) for t in W], [to64(t) for t in G], [to64(t) for t in M]
    lr = 0.05
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0, world_size=1,
                            device_id=DEV)
    try:
        owner = sharded.sharded_step(W, G, M, mu=0.95, nesterov=True, lr=lr, sync_momentum=True,
                                     owner=[0] * len(shapes))
        torch.cuda.synchronize()
        assert owner == [0] * len(shapes)
        assert sharded.partition(shapes, 1) == [0] * len(shapes)
    finally:
        dist.destroy_process_group()
    mo.muon_step(Wr, G, Mr, mu=0.95, nesterov=True, lr=lr)
    torch.cuda.synchronize()
    for x, y in zip(W + M, Wr + Mr):
        assert torch.equal(x, y)
    for i, (r, c) in enumerate(shapes):
        _, _, O = orc.muon_step(W64[i], G64[i], M64[i], 0.95, True, lr, form="standard")
        assert relF((W64[i] - to64(W[i])) / lr, O) <= TOL_BF16_RELF, shapes[i]
    st, _ = mo.muon_device_status()
    assert st == mo.MUON_OK
    assert np.all(np.isfinite(to64(W[0])))
