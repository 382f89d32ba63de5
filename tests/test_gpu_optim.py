"""One step of the hybrid optimizer (Muon + AdamW lanes) on GPU against the
fp64 oracle."""
import numpy as np
import pytest
import torch

import matrix_orthogonalizing_optimizer_step_b200 as mo
from matrix_orthogonalizing_optimizer_step_b200 import workloads as wl
from matrix_orthogonalizing_optimizer_step_b200.optim import MuonHybrid, split_params
from oracle import muon_oracle as orc
from tests._util import TOL_BF16_RELF, relF, to64

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda", 0)


class Tiny(torch.nn.Module):
    def __init__(self):
        super().__init__()
        self.wte = torch.nn.Embedding(500, 128)
        self.attn = torch.nn.Linear(128, 384)
        self.mlp = torch.nn.Linear(128, 512, bias=False)
        self.ln = torch.nn.LayerNorm(128)
        self.conv = torch.nn.Conv2d(16, 64, 3)
        self.lm_head = torch.nn.Linear(128, 500, bias=False)


def test_hybrid_step_matches_oracle():
    mo.muon_reset_config()
    torch.manual_seed(0)
    model = Tiny().to(DEV)
    for i, p in enumerate(model.parameters()):
        p.grad = wl.make_single(1, p.numel(), 700 + i, "student_t3", DEV, "f32", 0.01).view(p.shape)
    muon_p, adamw_p = split_params(model.named_parameters())
    before = {n: to64(p) for n, p in model.named_parameters()}
    grads = {n: to64(p.grad) for n, p in model.named_parameters()}
    lr = 0.02
    opt = MuonHybrid(muon_p, adamw_p, lr=lr, adamw_lr=1e-3)
    opt.step()
    torch.cuda.synchronize()
    after = {n: to64(p) for n, p in model.named_parameters()}
    for name, p in muon_p:
        W0 = before[name].reshape(p.shape[0], -1)
        G0 = grads[name].reshape(p.shape[0], -1)
        r, c = W0.shape
        n, m = min(r, c), max(r, c)
        form = "gram" if orc.ns_flops(n, m, 5, "gram") < orc.ns_flops(n, m, 5, "standard") else "standard"
        _, _, O = orc.muon_step(W0, G0, np.zeros_like(W0), 0.95, True, lr, form=form)
        O_gpu = (W0 - after[name].reshape(W0.shape)) / lr
        assert relF(O_gpu, O) <= TOL_BF16_RELF, name
    for name, p in adamw_p:
        p1, _, _ = orc.adamw_step(before[name].ravel(), grads[name].ravel(), np.zeros(p.numel()),
                                  np.zeros(p.numel()), 1, lr=1e-3, beta1=0.9, beta2=0.95, eps=1e-8,
                                  weight_decay=0.1)
        assert np.max(np.abs(after[name].ravel() - p1)) <= 1e-6 * 1e-3 + 2e-7 * np.max(np.abs(p1)), name
    st, bad = mo.muon_device_status()
    assert st == mo.MUON_OK
