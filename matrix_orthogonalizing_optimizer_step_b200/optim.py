"""Hybrid Muon + AdamW optimizer over a model's parameters.

[NanoGPT-Muon] "从 SGD 到 Muon": Muon only handles 2-D parameters (linear
weights, and convolution kernels once flattened to 2-D); scalar and vector
parameters stay with AdamW, and AdamW is also used for the embedding and the
output classification head.  "工程复现清单": AdamW lr 6e-4, betas
(0.9, 0.95), weight decay 0.1; Muon lr 6e-4, momentum 0.95, Nesterov,
five Newton-Schulz steps.

This class only keeps the per-parameter state buffers and hands device
pointers to the library; all arithmetic runs in CUDA.  When both groups use
one gradient dtype and one parameter dtype, the whole step is ONE hybrid
call (muon_hybrid_step): the AdamW elements ride in the same grouped
elementwise launch as the Muon momentum pass, followed by the Newton-Schulz
launches.  Otherwise each group takes its own call (muon_step,
muon_adamw_step).  Gradients may be fp32 or bf16; the installed config's
gradient and parameter dtypes are set to match.
"""
from __future__ import annotations

import torch

from . import MUON_DTYPE_BF16, MUON_DTYPE_F32, muon_adamw_step, muon_hybrid_step, muon_set_config, muon_step

_CODE = {torch.float32: MUON_DTYPE_F32, torch.bfloat16: MUON_DTYPE_BF16}

_ADAMW_NAME_HINTS = ("embed", "wte", "wpe", "lm_head", "head", "classifier")


def split_params(named_params):
    """(muon, adamw) lists of (name, parameter) by the page's rule: Muon for
    parameters of >= 2 dimensions that are not an embedding or output head,
    AdamW for everything else."""
    muon, adamw = [], []
    for name, p in named_params:
        if not p.requires_grad:
            continue
        lname = name.lower()
        if p.dim() >= 2 and not any(h in lname for h in _ADAMW_NAME_HINTS):
            muon.append((name, p))
        else:
            adamw.append((name, p))
    return muon, adamw


class MuonHybrid(torch.optim.Optimizer):
    """Muon for hidden matrices, AdamW for the rest (see module docstring).

    Pass the output of split_params (or two explicit lists of parameters)."""

    def __init__(self, muon_params, adamw_params, lr=6e-4, momentum=0.95, nesterov=True,
                 adamw_lr=6e-4, adamw_betas=(0.9, 0.95), adamw_eps=1e-8, adamw_weight_decay=0.1):
        mp = [p for _, p in muon_params] if muon_params and isinstance(muon_params[0], tuple) else list(muon_params)
        ap = [p for _, p in adamw_params] if adamw_params and isinstance(adamw_params[0], tuple) else list(adamw_params)
        groups = []
        if mp:
            groups.append(dict(params=mp, kind="muon", lr=lr, momentum=momentum, nesterov=nesterov))
        if ap:
            groups.append(dict(params=ap, kind="adamw", lr=adamw_lr, betas=adamw_betas, eps=adamw_eps,
                               weight_decay=adamw_weight_decay))
        super().__init__(groups, {})

    @torch.no_grad()
    def step(self, closure=None):
        loss = closure() if closure is not None else None
        lanes = {}
        for g in self.param_groups:
            ps = [p for p in g["params"] if p.grad is not None]
            if not ps:
                continue
            gdt = {p.grad.dtype for p in ps}
            pdt = {p.dtype for p in ps}
            if len(gdt) != 1 or len(pdt) != 1 or not (gdt | pdt) <= set(_CODE):
                raise TypeError("one gradient dtype and one parameter dtype per group, each fp32 or bf16")
            dts = (gdt.pop(), pdt.pop())
            if g["kind"] == "muon":
                lanes["muon"] = (g, dts, self._muon_lane(ps))
            else:
                lanes["adamw"] = (g, dts, self._adamw_lane(ps))
        if "muon" in lanes and "adamw" in lanes and lanes["muon"][1] == lanes["adamw"][1] \
                and len(lanes["adamw"][2]) == 1:
            # one hybrid call: both lanes in one elementwise launch
            gm, (gd, pd), (W, G, M) = lanes["muon"]
            ga, _, by_step = lanes["adamw"]
            (t, (P, AG, M1, M2)), = by_step.items()
            muon_set_config(grad_dtype=_CODE[gd], param_dtype=_CODE[pd])
            muon_hybrid_step(W, G, M, P, AG, M1, M2, t, mu=gm["momentum"], nesterov=gm["nesterov"],
                             lr=gm["lr"], adam_lr=ga["lr"], betas=ga["betas"], eps=ga["eps"],
                             weight_decay=ga["weight_decay"])
            return loss
        if "muon" in lanes:
            gm, (gd, pd), (W, G, M) = lanes["muon"]
            muon_set_config(grad_dtype=_CODE[gd], param_dtype=_CODE[pd])
            muon_step(W, G, M, mu=gm["momentum"], nesterov=gm["nesterov"], lr=gm["lr"])
        if "adamw" in lanes:
            ga, (gd, pd), by_step = lanes["adamw"]
            muon_set_config(grad_dtype=_CODE[gd], param_dtype=_CODE[pd])
            for t in sorted(by_step):  # normally one step count for the whole group
                P, AG, M1, M2 = by_step[t]
                muon_adamw_step(P, AG, M1, M2, t, lr=ga["lr"], betas=ga["betas"], eps=ga["eps"],
                                weight_decay=ga["weight_decay"])
        return loss

    def _muon_lane(self, ps):
        W, G, M = [], [], []
        for p in ps:
            st = self.state[p]
            if "momentum" not in st:
                st["momentum"] = torch.zeros_like(p, dtype=torch.bfloat16)
            # conv kernels and other >2-D weights are flattened to 2-D views
            W.append(p.view(p.shape[0], -1))
            G.append(p.grad.view(p.shape[0], -1))
            M.append(st["momentum"].view(p.shape[0], -1))
        return W, G, M

    def _adamw_lane(self, ps):
        """{step count: (params, grads, exp_avg, exp_avg_sq)} after advancing
        every parameter's step count."""
        by_step = {}
        for p in ps:
            st = self.state[p]
            if "exp_avg" not in st:
                st["exp_avg"] = torch.zeros(p.numel(), dtype=torch.float32, device=p.device)
                st["exp_avg_sq"] = torch.zeros(p.numel(), dtype=torch.float32, device=p.device)
                st["step"] = 0
            st["step"] += 1
            lists = by_step.setdefault(st["step"], ([], [], [], []))
            lists[0].append(p.view(-1))
            lists[1].append(p.grad.view(-1))
            lists[2].append(st["exp_avg"])
            lists[3].append(st["exp_avg_sq"])
        return by_step
