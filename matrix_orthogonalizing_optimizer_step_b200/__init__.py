"""B200 (sm_100a) Muon optimizer step: Python binding of libmuon.so.

The functions here carry the C ABI's names and only marshal arguments: torch
tensors supply device pointers, and the current torch CUDA stream is bound
before every call.  All arithmetic runs in the library's CUDA kernels; there
is no CPU or PyTorch fallback.  If libmuon.so is missing, the first call
raises ImportError.
"""
from __future__ import annotations

import ctypes

from . import _lib
from ._lib import (  # noqa: F401
    MUON_DTYPE_BF16, MUON_DTYPE_F32, MUON_ERR_CUDA, MUON_ERR_GUARD, MUON_ERR_INVALID_ARG,
    MUON_ERR_NO_MEMORY, MUON_ERR_NONFINITE, MUON_ERR_TIMEOUT,
    MUON_ERR_UNSUPPORTED, MUON_MAX_SHAPE_SCHEDULES, MUON_MAX_STEPS, MUON_NS_AUTO, MUON_NS_GRAM,
    MUON_NS_STANDARD, MUON_OK, MUON_PREC_FP32, STATUS_NAMES,
)

TUNED_COEFFS = (3.4445, -4.7750, 2.0315)

_FORMS = {"standard": MUON_NS_STANDARD, "gram": MUON_NS_GRAM,
          "auto": MUON_NS_AUTO}


class MuonError(RuntimeError):
    def __init__(self, code, msg):
        super().__init__(f"{STATUS_NAMES.get(code, code)}: {msg}")
        self.code = code


def lib():
    return _lib.load()


def _check(rc):
    if rc != MUON_OK:
        raise MuonError(rc, lib().muon_last_error().decode(errors="replace"))
    return rc


def _bind_stream(device):
    import torch
    s = torch.cuda.current_stream(device)
    lib().muon_set_stream(ctypes.c_void_p(s.cuda_stream))


def _coeff_array(coeffs, steps):
    flat = []
    c = list(coeffs)
    if c and not isinstance(c[0], (tuple, list)):
        c = [tuple(c)] * max(steps, 1)
    for t in c[:steps]:
        flat.extend(float(x) for x in t)
    if len(flat) < 3 * steps:
        raise ValueError("need one (a, b, c) triple per step")
    arr = (ctypes.c_float * max(len(flat), 1))(*flat)
    return arr


def _form_bits(mode):
    if isinstance(mode, str):
        return _FORMS[mode]
    return int(mode)


def muon_orthogonalize(X, coeffs=TUNED_COEFFS, steps=5, mode="auto", fp32=False):
    """In place: X <- NS_steps(X / (||X||_F + eps)) for each matrix of X.

    X: contiguous CUDA tensor of shape (m, n) or (batch, m, n); bf16, or fp32
    with fp32=True (the fp32 SIMT check path).  Returns X.
    """
    import torch
    if not X.is_cuda:
        raise ValueError("X must be a CUDA tensor")
    if not X.is_contiguous():
        raise ValueError("X must be contiguous")
    want = torch.float32 if fp32 else torch.bfloat16
    if X.dtype != want:
        raise ValueError(f"X must be {want}")
    if X.dim() == 2:
        batch, m, n = 1, X.shape[0], X.shape[1]
    elif X.dim() == 3:
        batch, m, n = X.shape
    else:
        raise ValueError("X must be 2D or 3D")
    bits = _form_bits(mode) | (MUON_PREC_FP32 if fp32 else 0)
    arr = _coeff_array(coeffs, steps)
    _bind_stream(X.device)
    _check(lib().muon_orthogonalize(batch, m, n, ctypes.c_void_p(X.data_ptr()),
                                    arr, steps, bits))
    return X


def _muon_lane(params, grads, momentum):
    count = len(params)
    if not (len(grads) == len(momentum) == count) or count == 0:
        raise ValueError("params, grads and momentum must be non-empty lists of equal length")
    vp = ctypes.c_void_p
    P = (vp * count)(*[t.data_ptr() for t in params])
    G = (vp * count)(*[t.data_ptr() for t in grads])
    M = (vp * count)(*[t.data_ptr() for t in momentum])
    shapes = []
    for p, g, m in zip(params, grads, momentum):
        if p.dim() != 2 or tuple(g.shape) != tuple(p.shape) or tuple(m.shape) != tuple(p.shape):
            raise ValueError("each param, grad and momentum must be 2D of one shape")
        if not (p.is_contiguous() and g.is_contiguous() and m.is_contiguous()):
            raise ValueError("tensors must be contiguous")
        shapes.extend(p.shape)
    S = (ctypes.c_int * len(shapes))(*shapes)
    return P, G, M, S, count


def _adamw_lane(params, grads, exp_avg, exp_avg_sq):
    count = len(params)
    if not (len(grads) == len(exp_avg) == len(exp_avg_sq) == count) or count == 0:
        raise ValueError("params, grads, exp_avg and exp_avg_sq must be non-empty lists of equal length")
    for ts in zip(params, grads, exp_avg, exp_avg_sq):
        if any(t.numel() != ts[0].numel() or not t.is_contiguous() for t in ts):
            raise ValueError("each param, grad and moment must be contiguous with one element count")
    vp = ctypes.c_void_p
    arr = lambda ts: (vp * count)(*[t.data_ptr() for t in ts])  # noqa: E731
    N = (ctypes.c_longlong * count)(*[t.numel() for t in params])
    return arr(params), arr(grads), arr(exp_avg), arr(exp_avg_sq), N, count


def muon_step(params, grads, momentum, mu=0.95, nesterov=True, lr=6e-4):
    """One Muon step over lists of 2D CUDA tensors (updated in place).

    grads, momentum and params use the installed config's dtypes.
    """
    P, G, M, S, count = _muon_lane(params, grads, momentum)
    _bind_stream(params[0].device)
    _check(lib().muon_step(P, G, M, float(mu), 1 if nesterov else 0, float(lr), S, count))


def _host_lane(host, dev, name):
    """Pointers of the pinned host tensors that mirror the device tensors
    `dev` (same shapes and dtypes), or None."""
    if host is None:
        return None
    if len(host) != len(dev):
        raise ValueError(f"{name} must have one tensor per parameter")
    for h, d in zip(host, dev):
        if h.is_cuda or not h.is_pinned():
            raise ValueError(f"{name} must hold pinned (page-locked) host tensors")
        if tuple(h.shape) != tuple(d.shape) or h.dtype != d.dtype or not h.is_contiguous():
            raise ValueError(f"{name} tensors must be contiguous, with their device tensor's shape and dtype")
    return (ctypes.c_void_p * len(host))(*[t.data_ptr() for t in host])


def muon_step_offload(params, grads, momentum, grads_host=None, params_host=None, mu=0.95, nesterov=True,
                      lr=6e-4, chunks=8):
    """muon_step with the gradients copied in from pinned host tensors
    (grads_host, into the device tensors grads) and the updated parameters
    copied out to pinned host tensors (params_host), pipelined over `chunks`
    groups of matrices so that the copies overlap the step."""
    P, G, M, S, count = _muon_lane(params, grads, momentum)
    GH = _host_lane(grads_host, grads, "grads_host")
    PH = _host_lane(params_host, params, "params_host")
    _bind_stream(params[0].device)
    _check(lib().muon_step_offload(P, GH, G, M, PH, float(mu), 1 if nesterov else 0, float(lr), S, count,
                                   int(chunks)))


def muon_offload_chunks(weights, chunks):
    """The grouping muon_step_offload uses: group bounds [0, ..., len(weights)]
    of consecutive matrices with about equal total weight."""
    count = len(weights)
    W = (ctypes.c_longlong * max(count, 1))(*[int(w) for w in weights])
    B = (ctypes.c_int * (max(min(chunks, count), 0) + 1))()
    g = lib().muon_offload_chunks(W, count, int(chunks), B)
    _check(min(g, 0))
    return list(B[:g + 1])


def muon_hybrid_step(params, grads, momentum, adam_params, adam_grads, exp_avg, exp_avg_sq, step,
                     mu=0.95, nesterov=True, lr=6e-4, adam_lr=6e-4, betas=(0.9, 0.95), eps=1e-8,
                     weight_decay=0.1):
    """The hybrid step in one elementwise launch plus the Newton-Schulz
    launches: muon_step over (params, grads, momentum) and the AdamW step over
    the adam_* lists (fp32 moments), as muon_step + muon_adamw_step."""
    P, G, M, S, count = _muon_lane(params, grads, momentum)
    AP, AG, AM, AV, N, acount = _adamw_lane(adam_params, adam_grads, exp_avg, exp_avg_sq)
    lane = _lib.MuonAdamwLane(AP, AG, AM, AV, N, acount, float(adam_lr), float(betas[0]), float(betas[1]),
                              float(eps), float(weight_decay), int(step))
    _bind_stream(params[0].device)
    _check(lib().muon_hybrid_step(P, G, M, float(mu), 1 if nesterov else 0, float(lr), S, count,
                                  ctypes.byref(lane)))


def muon_adamw_step(params, grads, exp_avg, exp_avg_sq, step, lr=6e-4, betas=(0.9, 0.95), eps=1e-8,
                    weight_decay=0.1):
    """AdamW step (the hybrid optimizer's lane for embeddings, head and 1-D
    parameters) over lists of CUDA tensors, updated in place.  Moments are
    fp32; params and grads use the installed config's dtypes."""
    AP, AG, AM, AV, N, count = _adamw_lane(params, grads, exp_avg, exp_avg_sq)
    _bind_stream(params[0].device)
    _check(lib().muon_adamw_step(AP, AG, AM, AV, N, count, float(lr), float(betas[0]), float(betas[1]),
                                 float(eps), float(weight_decay), int(step)))


def muon_default_config():
    cfg = _lib.MuonConfig()
    _check(lib().muon_default_config(ctypes.byref(cfg)))
    return _cfg_to_dict(cfg)


def _cfg_to_dict(cfg):
    return {
        "steps": cfg.steps,
        "coeffs": [tuple(cfg.coeffs[3 * k:3 * k + 3]) for k in range(cfg.steps)],
        "mode": cfg.mode, "restart_mask": cfg.restart_mask, "eps": cfg.eps,
        "momentum_dtype": cfg.momentum_dtype, "param_dtype": cfg.param_dtype,
        "grad_dtype": cfg.grad_dtype, "soft_threshold": cfg.soft_threshold,
    }


def muon_get_config():
    cfg = _lib.MuonConfig()
    _check(lib().muon_get_config(ctypes.byref(cfg)))
    return _cfg_to_dict(cfg)


def muon_set_config(steps=None, coeffs=None, mode=None, restart_mask=None,
                    eps=None, momentum_dtype=None, param_dtype=None, grad_dtype=None,
                    soft_threshold=None):
    """Install a config; unspecified fields keep their current values."""
    cfg = _lib.MuonConfig()
    _check(lib().muon_get_config(ctypes.byref(cfg)))
    if steps is not None:
        cfg.steps = int(steps)
    if coeffs is not None:
        arr = _coeff_array(coeffs, cfg.steps)
        for i in range(3 * cfg.steps):
            cfg.coeffs[i] = arr[i]
    if mode is not None:
        cfg.mode = _form_bits(mode)
    if restart_mask is not None:
        cfg.restart_mask = int(restart_mask)
    if eps is not None:
        cfg.eps = float(eps)
    if momentum_dtype is not None:
        cfg.momentum_dtype = momentum_dtype
    if param_dtype is not None:
        cfg.param_dtype = param_dtype
    if grad_dtype is not None:
        cfg.grad_dtype = grad_dtype
    if soft_threshold is not None:
        cfg.soft_threshold = float(soft_threshold)
    _check(lib().muon_set_config(ctypes.byref(cfg)))


def muon_reset_config():
    """Install the default config and remove every per-shape schedule."""
    cfg = _lib.MuonConfig()
    _check(lib().muon_default_config(ctypes.byref(cfg)))
    _check(lib().muon_set_config(ctypes.byref(cfg)))
    _check(lib().muon_clear_shape_coeffs())


def muon_set_shape_coeffs(rows, cols, coeffs):
    """Register the Newton-Schulz schedule of muon_step for rows x cols
    matrices (and their transposes): a list of (a, b, c) triples, one per
    step (an empty list: normalisation only)."""
    triples = [tuple(float(x) for x in t) for t in coeffs]
    if any(len(t) != 3 for t in triples):
        raise ValueError("coeffs must be (a, b, c) triples")
    flat = [x for t in triples for x in t]
    arr = (ctypes.c_float * max(len(flat), 1))(*flat)
    _check(lib().muon_set_shape_coeffs(int(rows), int(cols), arr, len(triples)))


def muon_get_shape_coeffs(rows, cols):
    """The registered schedule of rows x cols matrices, or None."""
    arr = (ctypes.c_float * (3 * MUON_MAX_STEPS))()
    steps = ctypes.c_int(-1)
    _check(lib().muon_get_shape_coeffs(int(rows), int(cols), arr, ctypes.byref(steps)))
    if steps.value < 0:
        return None
    return [tuple(arr[3 * k:3 * k + 3]) for k in range(steps.value)]


def muon_clear_shape_coeffs():
    _check(lib().muon_clear_shape_coeffs())


def muon_device_status(device=None):
    """(status, first bad matrix index or -1); synchronises the bound stream."""
    import torch
    _bind_stream(device if device is not None else torch.cuda.current_device())
    bad = ctypes.c_int(-1)
    rc = lib().muon_device_status(ctypes.byref(bad))
    return rc, bad.value


def muon_debug_corrupt_guard(index, device=None):
    """Debug canary mode (MUON_DEBUG_CANARY=1): overwrite one byte of a
    workspace guard of the current plan, for tests of the guard check."""
    import torch
    _bind_stream(device if device is not None else torch.cuda.current_device())
    _check(lib().muon_debug_corrupt_guard(int(index)))


def muon_release_workspace():
    _check(lib().muon_release_workspace())


def muon_profile_enable(on=True):
    _check(lib().muon_profile_enable(1 if on else 0))


def muon_profile_reset():
    _check(lib().muon_profile_reset())


def muon_profile_read():
    """Per kernel kind: launches, total_ms, flops, bytes (CUDA-event timed)."""
    arr = (_lib.MuonKernelStats * 8)()
    n = ctypes.c_int(0)
    _check(lib().muon_profile_read(arr, 8, ctypes.byref(n)))
    out = {}
    for i in range(n.value):
        s = arr[i]
        out[s.name.decode()] = {"launches": s.launches, "total_ms": s.total_ms,
                                "flops": s.flops, "bytes": s.bytes}
    return out


def muon_launch_count():
    return int(lib().muon_launch_count())


def muon_version():
    return int(lib().muon_version())
