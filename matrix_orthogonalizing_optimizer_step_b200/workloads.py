"""Seeded synthetic workloads for the Muon step.

This module holds shapes and random draws only -- none of the method's
arithmetic -- so that both the CUDA path and the fp64 oracle can be fed the
same inputs.  Every matrix is drawn from its own generator, seeded by
(workload id, matrix index, role), so any single matrix can be regenerated on
its own.  Roles: 0 = gradient (or the matrix to orthogonalise), 1 = initial
momentum, 2 = parameter.

Distributions (the shapes are the model families'; no dataset is involved):

* gaussian          N(0, 1)
* student_t3        Z / sqrt(chi2_3 / 3), chi2_3 the sum of three squared
                    standard normals (Student-t, nu = 3)
* student_t3_outl   student_t3 with 0.1 % of the entries, drawn uniformly
                    without replacement, multiplied by 100
* normal_1e-4       N(0, 1e-4): variance 1e-4, standard deviation 0.01
* params            N(0, 0.02^2)

Values are drawn in fp32 and rounded to the storage dtype (round to nearest
even) by torch's dtype conversion.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch

ROLE_GRAD, ROLE_MOMENTUM, ROLE_PARAM = 0, 1, 2


@dataclass(frozen=True)
class Workload:
    wid: int
    name: str
    shapes: tuple            # ((rows, cols), ...) one entry per matrix
    grad_dist: str
    grad_scale: float = 1.0
    dtype: str = "bf16"      # storage dtype of grads / the matrices
    momentum_dtype: str = "bf16"
    param_dtype: str = "f32"
    full_step: bool = True   # momentum + NS + update, else NS only
    forms: tuple = ("gram",)
    notes: str = ""
    meta: dict = field(default_factory=dict)
    # element counts of the model's AdamW parameters (embeddings, output
    # head, 1-D parameters), empty when the set has no model around it
    adamw_numels: tuple = ()

    @property
    def count(self):
        return len(self.shapes)

    @property
    def elements(self):
        return sum(r * c for r, c in self.shapes)


def _gpt2_shapes():
    per_layer = ((768, 2304), (768, 768), (768, 3072), (3072, 768))
    return tuple(s for _ in range(12) for s in per_layer)


def _llama8b_shapes():
    per_layer = ((4096, 4096), (4096, 4096), (4096, 1024), (4096, 1024),
                 (4096, 14336), (4096, 14336), (14336, 4096))
    return tuple(s for _ in range(32) for s in per_layer)


def _gpt2_adamw_numels():
    # token / position embeddings (the output head is tied to wte), per layer
    # ln_1 (w, b), qkv bias, attn-out bias, ln_2 (w, b), fc bias, proj bias,
    # final ln_f (w, b)
    per_layer = (768, 768, 2304, 768, 768, 768, 3072, 768)
    return (50257 * 768, 1024 * 768) + per_layer * 12 + (768, 768)


def _llama8b_adamw_numels():
    # token embedding and untied output head (vocabulary 128256), per layer
    # two RMSNorm gains, final norm
    return (128256 * 4096, 128256 * 4096) + (4096, 4096) * 32 + (4096,)


def _moe_shapes():
    return tuple(s for _ in range(64) for s in ((2048, 7168), (7168, 2048)))


WORKLOADS = {
    1: Workload(1, "single-256x1024-f32", ((256, 1024),), "gaussian",
                dtype="f32", full_step=False, forms=("standard", "gram"),
                notes="fp32 N(0,1), seed 0; also the fp32 check path"),
    2: Workload(2, "gpt2-124m-muon-set", _gpt2_shapes(), "student_t3", 0.01,
                notes="12 layers x {qkv 768x2304, attn-out 768x768, "
                      "fc 768x3072, proj 3072x768}; momentum 0.95 Nesterov",
                adamw_numels=_gpt2_adamw_numels()),
    3: Workload(3, "aspect-sweep-b16",
                tuple([(2048, 2048)] * 16 + [(2048, 8192)] * 16
                      + [(1024, 16384)] * 16),
                "gaussian", full_step=False, forms=("standard", "gram")),
    4: Workload(4, "moe-64-experts", _moe_shapes(), "student_t3_outl", 0.01,
                notes="64 experts x {up 2048x7168, down 7168x2048}; "
                      "Gram NS with restart"),
    5: Workload(5, "llama-8b-muon-set", _llama8b_shapes(), "normal_1e-4",
                notes="32 layers x {q,o 4096x4096; k,v 4096x1024; "
                      "gate,up 4096x14336; down 14336x4096}",
                adamw_numels=_llama8b_adamw_numels()),
}

_TORCH_DTYPE = {"bf16": torch.bfloat16, "f32": torch.float32,
                "f16": torch.float16}


def torch_dtype(name):
    return _TORCH_DTYPE[name]


def _generator(wid, idx, role, device):
    g = torch.Generator(device=device)
    if wid == 1:
        # the single 256x1024 matrix is specified with seed 0
        g.manual_seed(role)
    else:
        # one seed per (workload, matrix, role), independent of the device
        g.manual_seed((wid * 1_000_003 + idx) * 16 + role)
    return g


def draw(dist, shape, gen, device, scale=1.0):
    """fp32 draw of one matrix from the named distribution."""
    if dist == "gaussian":
        x = torch.randn(shape, generator=gen, device=device)
    elif dist in ("student_t3", "student_t3_outl"):
        z = torch.randn(shape, generator=gen, device=device)
        chi = torch.randn((3,) + tuple(shape), generator=gen, device=device)
        x = z / torch.sqrt(chi.square().sum(0) / 3.0)
        if dist == "student_t3_outl":
            numel = x.numel()
            k = max(1, numel // 1000)
            pick = torch.randperm(numel, generator=gen, device=device)[:k]
            x.view(-1)[pick] *= 100.0
    elif dist == "normal_1e-4":
        x = torch.randn(shape, generator=gen, device=device) * 0.01
    elif dist == "params":
        x = torch.randn(shape, generator=gen, device=device) * 0.02
    else:
        raise ValueError(dist)
    return x * scale if scale != 1.0 else x


def make_matrix(w: Workload, idx, role, device="cpu", dtype=None):
    """One seeded matrix of workload ``w``: index ``idx``, role ``role``."""
    rows, cols = w.shapes[idx]
    gen = _generator(w.wid, idx, role, device)
    if role == ROLE_PARAM:
        x = draw("params", (rows, cols), gen, device)
        dt = dtype or w.param_dtype
    else:
        x = draw(w.grad_dist, (rows, cols), gen, device, w.grad_scale)
        dt = dtype or (w.momentum_dtype if role == ROLE_MOMENTUM else w.dtype)
    return x.to(_TORCH_DTYPE[dt])


def make_single(rows, cols, seed, dist="gaussian", device="cpu", dtype="bf16",
                scale=1.0):
    """A free-standing seeded matrix (tests of ragged and edge shapes)."""
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return draw(dist, (rows, cols), g, device, scale).to(_TORCH_DTYPE[dtype])
