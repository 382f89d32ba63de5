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


def _lanes(seed):
    shapes = [(768, 2304), (768, 768), (3072, 768), (200, 712)]
    G = [wl.make_single(r, c, seed + 3 * i, "student_t3", DEV, "bf16", 0.01) for i, (r, c) in enumerate(shapes)]
    M = [wl.make_single(r, c, seed + 3 * i + 1, "student_t3", DEV, "bf16", 0.01) for i, (r, c) in enumerate(shapes)]
    W = [wl.make_single(r, c, seed + 3 * i + 2, "params", DEV, "f32") for i, (r, c) in enumerate(shapes)]
    numels = [50257 * 768, 1024 * 768, 768, 768, 2304, 5, 4099]
    P = [wl.make_single(1, n, seed + 100 + i, "params", DEV, "f32").view(-1) for i, n in enumerate(numels)]
    AG = [wl.make_single(1, n, seed + 200 + i, "student_t3", DEV, "bf16", 0.01).view(-1) for i, n in enumerate(numels)]
    M1 = [torch.zeros(n, device=DEV) for n in numels]
    M2 = [torch.zeros(n, device=DEV) for n in numels]
    return (W, G, M), (P, AG, M1, M2)


def test_hybrid_call_equals_separate_calls_and_is_one_elementwise_launch():
    """muon_hybrid_step = muon_step + muon_adamw_step bit for bit, with the
    AdamW lane inside the momentum launch: one elementwise launch, no AdamW
    launch, plus the Newton-Schulz launches."""
    mo.muon_reset_config()
    (W, G, M), (P, AG, M1, M2) = _lanes(4000)
    (Wb, _, Mb), (Pb, _, M1b, M2b) = _lanes(4000)
    for t in (1, 2):
        mo.muon_step(Wb, G, Mb, mu=0.95, nesterov=True, lr=0.02)
        mo.muon_adamw_step(Pb, AG, M1b, M2b, t, lr=1e-3)
    mo.muon_hybrid_step(W, G, M, P, AG, M1, M2, 1, lr=0.02, adam_lr=1e-3)  # builds the plan
    torch.cuda.synchronize()
    mo.muon_profile_reset()
    mo.muon_profile_enable(True)
    n0 = mo.muon_launch_count()
    mo.muon_hybrid_step(W, G, M, P, AG, M1, M2, 2, lr=0.02, adam_lr=1e-3)
    prof = mo.muon_profile_read()
    mo.muon_profile_enable(False)
    launched = mo.muon_launch_count() - n0
    assert prof["momentum_norm"]["launches"] == 1
    assert prof["adamw"]["launches"] == 0
    assert launched == 1 + prof["gemm_tc"]["launches"]
    for x, y in zip(W + M + P + M1 + M2, Wb + Mb + Pb + M1b + M2b):
        assert torch.equal(x, y)
    st, _ = mo.muon_device_status()
    assert st == mo.MUON_OK


def test_hybrid_optimizer_issues_one_hybrid_call():
    mo.muon_reset_config()
    torch.manual_seed(1)
    model = Tiny().to(DEV)
    for i, p in enumerate(model.parameters()):
        p.grad = wl.make_single(1, p.numel(), 900 + i, "student_t3", DEV, "f32", 0.01).view(p.shape)
    opt = MuonHybrid(*split_params(model.named_parameters()))
    opt.step()  # first step builds the plan
    torch.cuda.synchronize()
    mo.muon_profile_reset()
    mo.muon_profile_enable(True)
    opt.step()
    prof = mo.muon_profile_read()
    mo.muon_profile_enable(False)
    assert prof["momentum_norm"]["launches"] == 1
    assert prof["adamw"]["launches"] == 0


def test_hybrid_argument_error_enqueues_nothing():
    mo.muon_reset_config()
    (W, G, M), (P, AG, M1, M2) = _lanes(4100)
    W0 = [w.clone() for w in W]
    n0 = mo.muon_launch_count()
    with pytest.raises(mo.MuonError):
        mo.muon_hybrid_step(W, G, M, P, AG, M1, M2, 0)  # step 0: invalid AdamW step
    torch.cuda.synchronize()
    assert mo.muon_launch_count() == n0
    assert all(torch.equal(a, b) for a, b in zip(W, W0))


@pytest.mark.parametrize("grad_dt,par_dt,mom_dt,lam", [
    ("bf16", "f32", "bf16", 0.0), ("f32", "f32", "bf16", 0.0), ("bf16", "bf16", "bf16", 0.0),
    ("bf16", "f32", "f32", 0.0), ("f32", "bf16", "f32", 0.0), ("bf16", "f32", "bf16", 0.06),
    ("f32", "f32", "f32", 0.06)])
def test_hybrid_instances_equal_separate_calls(grad_dt, par_dt, mom_dt, lam):
    """Every instance of the hybrid momentum launch (gradient dtype x momentum
    dtype x soft-threshold split, with fp32 or bf16 parameters) gives the
    same bits as muon_step followed by muon_adamw_step."""
    code = {"f32": mo.MUON_DTYPE_F32, "bf16": mo.MUON_DTYPE_BF16}
    mo.muon_reset_config()
    mo.muon_set_config(grad_dtype=code[grad_dt], param_dtype=code[par_dt], momentum_dtype=code[mom_dt],
                       soft_threshold=lam)
    shapes = [(256, 768), (768, 256), (200, 712), (37, 91)]
    numels = [1024 * 768, 768, 2304, 5, 4099]

    def lanes():
        G = [wl.make_single(r, c, 4300 + i, "student_t3_outl", DEV, grad_dt, 0.01) for i, (r, c) in enumerate(shapes)]
        M = [wl.make_single(r, c, 4400 + i, "student_t3", DEV, mom_dt, 0.01) for i, (r, c) in enumerate(shapes)]
        W = [wl.make_single(r, c, 4500 + i, "params", DEV, par_dt) for i, (r, c) in enumerate(shapes)]
        P = [wl.make_single(1, n, 4600 + i, "params", DEV, par_dt).view(-1) for i, n in enumerate(numels)]
        AG = [wl.make_single(1, n, 4700 + i, "student_t3", DEV, grad_dt, 0.01).view(-1) for i, n in enumerate(numels)]
        M1 = [torch.zeros(n, device=DEV) for n in numels]
        M2 = [torch.zeros(n, device=DEV) for n in numels]
        return W, G, M, P, AG, M1, M2

    W, G, M, P, AG, M1, M2 = lanes()
    Wb, _, Mb, Pb, _, M1b, M2b = lanes()
    for t in (1, 2):
        mo.muon_hybrid_step(W, G, M, P, AG, M1, M2, t, lr=0.02, adam_lr=1e-3)
        mo.muon_step(Wb, G, Mb, mu=0.95, nesterov=True, lr=0.02)
        mo.muon_adamw_step(Pb, AG, M1b, M2b, t, lr=1e-3)
    torch.cuda.synchronize()
    for x, y in zip(W + M + P + M1 + M2, Wb + Mb + Pb + M1b + M2b):
        assert torch.equal(x, y)
    st, _ = mo.muon_device_status()
    assert st == mo.MUON_OK
    mo.muon_reset_config()
