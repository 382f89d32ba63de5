"""GPU parity of the AdamW lane (embeddings, head, 1-D parameters) against
the fp64 oracle over several steps."""
import numpy as np
import pytest
import torch

import matrix_orthogonalizing_optimizer_step_b200 as mo
from matrix_orthogonalizing_optimizer_step_b200 import workloads as wl
from oracle import muon_oracle as orc
from tests._util import to64

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda", 0)

# GPT-2 124M's AdamW parameters: token and position embeddings, LayerNorm
# gains/biases and the linear biases (flat), plus odd sizes for the scalar path
NUMELS = [50257 * 768, 1024 * 768] + [768] * 10 + [2304, 3072, 5, 4099]


@pytest.fixture(autouse=True)
def _fresh():
    mo.muon_reset_config()
    yield
    mo.muon_reset_config()


def _state(numels, par_dt, seed):
    P = [wl.make_single(1, n, seed + i, "params", DEV, par_dt).view(-1) for i, n in enumerate(numels)]
    M = [torch.zeros(n, device=DEV) for n in numels]
    V = [torch.zeros(n, device=DEV) for n in numels]
    return P, M, V


@pytest.mark.parametrize("par_dt,grad_dt", [("f32", "bf16"), ("bf16", "bf16"), ("f32", "f32"), ("bf16", "f32")])
def test_adamw_matches_oracle(par_dt, grad_dt):
    mo.muon_set_config(param_dtype=mo.MUON_DTYPE_F32 if par_dt == "f32" else mo.MUON_DTYPE_BF16,
                       grad_dtype=mo.MUON_DTYPE_F32 if grad_dt == "f32" else mo.MUON_DTYPE_BF16)
    numels = NUMELS if par_dt == "f32" else NUMELS[1:]
    P, M, V = _state(numels, par_dt, 40)
    ref = [(to64(p), np.zeros(p.numel()), np.zeros(p.numel())) for p in P]
    lr, b1, b2, eps, wd = 6e-4, 0.9, 0.95, 1e-8, 0.1
    for step in range(1, 4):
        G = [wl.make_single(1, n, 1000 * step + i, "student_t3", DEV, grad_dt, 0.01).view(-1)
             for i, n in enumerate(numels)]
        if par_dt == "bf16":
            # bf16 parameters: the oracle restarts every step from the GPU's
            # stored parameters, so each step is checked as ONE bf16 rounding
            # of that step's update (no rounding compounded over steps)
            ref = [(to64(P[i]), m, v) for i, (_, m, v) in enumerate(ref)]
        mo.muon_adamw_step(P, G, M, V, step, lr=lr, betas=(b1, b2), eps=eps, weight_decay=wd)
        torch.cuda.synchronize()
        ref = [orc.adamw_step(p, to64(g), m, v, step, lr, b1, b2, eps, wd)
               for (p, m, v), g in zip(ref, G)]
        for i, (p, m, v) in enumerate(ref):
            gm, gv = to64(M[i]), to64(V[i])
            # fp32 rounding of the terms (beta m and (1 - beta) g) bounds the
            # error where they cancel: scale by the tensor's magnitude
            assert np.max(np.abs(gm - m)) <= 1e-6 * np.max(np.abs(m)), i
            assert np.max(np.abs(gv - v)) <= 1e-6 * np.max(np.abs(v)), i
            gp = to64(P[i])
            # fp32 arithmetic of the step: a few fp32 ulps of p, and the moments'
            # 1e-6 relative error seen through lr (|m_hat / (sqrt(v_hat) + eps)|
            # is at most about 1 / sqrt(1 - beta2) for these betas, < 5)
            arith = 1e-6 * 5 * lr + 2.0 ** -21 * np.abs(p)
            if par_dt == "f32":
                assert np.max(np.abs(gp - p)) <= 1e-6 * lr + 2e-7 * np.max(np.abs(p)), i
            else:
                # one round-to-nearest-even bf16 rounding of the fp32 result:
                # half an ulp, at most 2^-8 of its magnitude (8 significant bits)
                assert np.all(np.abs(gp - p) <= 2.0 ** -8 * (np.abs(p) + arith) + arith), i


def test_adamw_zero_gradient_is_pure_decay():
    P, M, V = _state([1000, 4096], "f32", 70)
    P0 = [to64(p) for p in P]
    G = [torch.zeros(p.numel(), dtype=torch.bfloat16, device=DEV) for p in P]
    for step in range(1, 4):
        mo.muon_adamw_step(P, G, M, V, step, lr=0.1, weight_decay=0.2)
    torch.cuda.synchronize()
    for p, p0 in zip(P, P0):
        assert np.allclose(to64(p), p0 * (1 - 0.1 * 0.2) ** 3, rtol=1e-6)


def test_adamw_argument_errors():
    P, M, V = _state([16], "f32", 80)
    G = [torch.zeros(16, dtype=torch.bfloat16, device=DEV)]
    for bad in [dict(step=0), dict(step=1, betas=(1.0, 0.9)), dict(step=1, eps=-1.0),
                dict(step=1, lr=float("nan"))]:
        step = bad.pop("step")
        with pytest.raises(mo.MuonError):
            mo.muon_adamw_step(P, G, M, V, step, **bad)
