"""Host-side tests of the C ABI (no GPU): the library loads, exports every
symbol include/muon.h declares, and validates arguments before touching a
device."""
import ctypes
import os
import re

import pytest

import matrix_orthogonalizing_optimizer_step_b200 as mo
from matrix_orthogonalizing_optimizer_step_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "muon.h")


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(_lib.LIB_PATH):
        from matrix_orthogonalizing_optimizer_step_b200 import build
        build.build()
    return mo.lib()


def header_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"MUON_API\s+[\w\s\*]+?\b(muon_\w+)\s*\(", text)))


def test_every_header_symbol_is_exported(lib):
    names = header_functions()
    assert len(names) >= 10
    assert sorted(_lib.EXPORTS) == names
    for n in names:
        assert hasattr(lib, n), n


def test_version_and_defaults(lib):
    assert lib.muon_version() == 10000
    cfg = mo.muon_default_config()
    assert cfg["steps"] == 5
    for t in cfg["coeffs"]:
        assert t == pytest.approx((3.4445, -4.7750, 2.0315), rel=1e-6)
    assert cfg["mode"] == mo.MUON_NS_AUTO
    assert cfg["restart_mask"] == 1 << 2
    assert cfg["eps"] == pytest.approx(1e-7)
    assert cfg["momentum_dtype"] == mo.MUON_DTYPE_BF16
    assert cfg["param_dtype"] == mo.MUON_DTYPE_F32
    assert cfg["grad_dtype"] == mo.MUON_DTYPE_BF16
    assert cfg["soft_threshold"] == 0.0


def test_config_roundtrip_and_validation(lib):
    mo.muon_reset_config()
    mo.muon_set_config(steps=3, coeffs=[(2, -1.5, 0.5), (3, -4, 2), (1, 0, 0)], mode="gram",
                       restart_mask=0b10, eps=1e-6)
    c = mo.muon_get_config()
    assert c["steps"] == 3 and c["mode"] == mo.MUON_NS_GRAM and c["restart_mask"] == 2
    assert c["coeffs"][1] == pytest.approx((3, -4, 2))
    for bad in [dict(steps=17), dict(steps=-1), dict(mode=7), dict(eps=float("nan")),
                dict(momentum_dtype=5), dict(param_dtype=9), dict(grad_dtype=3),
                dict(soft_threshold=-1.0), dict(soft_threshold=float("inf"))]:
        with pytest.raises(mo.MuonError) as e:
            mo.muon_set_config(**bad)
        assert e.value.code in (mo.MUON_ERR_INVALID_ARG, mo.MUON_ERR_UNSUPPORTED)
    # a rejected config leaves the installed one untouched
    assert mo.muon_get_config()["steps"] == 3
    mo.muon_reset_config()
    assert lib.muon_set_config(None) == mo.MUON_ERR_INVALID_ARG
    assert lib.muon_get_config(None) == mo.MUON_ERR_INVALID_ARG


def test_orthogonalize_argument_errors(lib):
    co = (ctypes.c_float * 15)(*([3.4445, -4.775, 2.0315] * 5))
    dummy = ctypes.c_void_p(0x1000)
    f = lib.muon_orthogonalize
    assert f(0, 4, 4, dummy, co, 5, 0) == mo.MUON_ERR_INVALID_ARG
    assert f(1, 0, 4, dummy, co, 5, 0) == mo.MUON_ERR_INVALID_ARG
    assert f(1, 4, -3, dummy, co, 5, 0) == mo.MUON_ERR_INVALID_ARG
    assert f(1, 4, 4, None, co, 5, 0) == mo.MUON_ERR_INVALID_ARG
    assert f(1, 4, 4, dummy, None, 5, 0) == mo.MUON_ERR_INVALID_ARG
    assert f(1, 4, 4, dummy, co, 17, 0) == mo.MUON_ERR_INVALID_ARG
    assert f(1, 4, 4, dummy, co, -1, 0) == mo.MUON_ERR_INVALID_ARG
    assert f(1, 4, 4, dummy, co, 5, 0x4000) == mo.MUON_ERR_INVALID_ARG
    assert f(1, 4, 4, dummy, co, 5, 9) == mo.MUON_ERR_INVALID_ARG
    nan = (ctypes.c_float * 3)(float("nan"), 1, 1)
    assert f(1, 4, 4, dummy, nan, 1, 0) == mo.MUON_ERR_INVALID_ARG
    assert b"" != lib.muon_last_error()


def test_step_argument_errors(lib):
    vp = ctypes.c_void_p
    P = (vp * 2)(0x1000, 0x2000)
    Z = (vp * 2)(0x1000, None)
    S = (ctypes.c_int * 4)(4, 4, 8, 8)
    Sbad = (ctypes.c_int * 4)(4, 0, 8, 8)
    f = lib.muon_step
    assert f(P, P, P, 0.95, 1, 1e-3, S, 0) == mo.MUON_ERR_INVALID_ARG
    assert f(None, P, P, 0.95, 1, 1e-3, S, 2) == mo.MUON_ERR_INVALID_ARG
    assert f(P, P, P, 0.95, 1, 1e-3, None, 2) == mo.MUON_ERR_INVALID_ARG
    assert f(P, Z, P, 0.95, 1, 1e-3, S, 2) == mo.MUON_ERR_INVALID_ARG
    assert f(P, P, P, 0.95, 1, 1e-3, Sbad, 2) == mo.MUON_ERR_INVALID_ARG
    assert f(P, P, P, float("inf"), 1, 1e-3, S, 2) == mo.MUON_ERR_INVALID_ARG
    assert f(P, P, P, 0.95, 1, float("nan"), S, 2) == mo.MUON_ERR_INVALID_ARG


def test_no_device_reports_cuda_error(lib):
    """Valid arguments on a host without a usable GPU fail with MUON_ERR_CUDA
    (never a silent CPU fallback)."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    co = (ctypes.c_float * 15)(*([3.4445, -4.775, 2.0315] * 5))
    rc = lib.muon_orthogonalize(1, 8, 8, ctypes.c_void_p(0x1000), co, 5, 0)
    assert rc == mo.MUON_ERR_CUDA
    assert b"CUDA" in lib.muon_last_error() or b"device" in lib.muon_last_error()


def test_profile_api_without_device(lib):
    mo.muon_profile_reset()
    stats = mo.muon_profile_read()
    assert set(stats) == {"momentum_norm", "gemm_tc", "gemm_f32", "scale_apply", "adamw"}
    assert all(v["launches"] == 0 for v in stats.values())
    assert mo.muon_launch_count() >= 0


def test_binding_validates_before_calling_the_library():
    """The Python binding rejects malformed arguments itself (no device is
    touched): list lengths, dimensions, shapes, contiguity, device, dtype."""
    import torch
    a = torch.zeros(4, 8, dtype=torch.bfloat16)
    b = torch.zeros(4, 8, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        mo.muon_step([a], [b, b], [a])                       # list lengths differ
    with pytest.raises(ValueError):
        mo.muon_step([], [], [])                              # empty
    with pytest.raises(ValueError):
        mo.muon_step([torch.zeros(32)], [torch.zeros(32)], [torch.zeros(32)])  # not 2D
    with pytest.raises(ValueError):
        mo.muon_step([a], [torch.zeros(8, 4, dtype=torch.bfloat16)], [a])      # shape mismatch
    with pytest.raises(ValueError):
        mo.muon_step([a], [torch.zeros(8, 4, dtype=torch.bfloat16).t()], [a])  # not contiguous
    with pytest.raises(ValueError):
        mo.muon_orthogonalize(a)                              # not a CUDA tensor
    with pytest.raises(ValueError):
        mo.muon_adamw_step([torch.zeros(8)], [torch.zeros(9)], [torch.zeros(8)], [torch.zeros(8)], 1)
    with pytest.raises(ValueError):
        mo.muon_adamw_step([torch.zeros(8)], [], [torch.zeros(8)], [torch.zeros(8)], 1)


def test_shape_schedule_table(lib):
    """Per-shape schedules (host-only calls): registration keyed by the short
    and long side, replacement, lookup, validation and clearing."""
    mo.muon_reset_config()
    assert mo.muon_get_shape_coeffs(384, 1536) is None
    mo.muon_set_shape_coeffs(384, 1536, [(3.0, -4.0, 2.0), (2.0, -1.5, 0.5)])
    assert mo.muon_get_shape_coeffs(1536, 384) == [(3.0, -4.0, 2.0), (2.0, -1.5, 0.5)]  # transpose shares it
    mo.muon_set_shape_coeffs(1536, 384, [(1.5, -0.5, 0.0)])                              # replaces it
    assert mo.muon_get_shape_coeffs(384, 1536) == [(1.5, -0.5, 0.0)]
    mo.muon_set_shape_coeffs(64, 64, [])                                                 # normalise only
    assert mo.muon_get_shape_coeffs(64, 64) == []
    for bad in [(0, 5, [(1, 0, 0)]), (5, -1, [(1, 0, 0)]), (8, 8, [(float("inf"), 0, 0)]),
                (8, 8, [(1, 0, 0)] * 17)]:
        with pytest.raises(mo.MuonError) as e:
            mo.muon_set_shape_coeffs(*bad)
        assert e.value.code == mo.MUON_ERR_INVALID_ARG
    mo.muon_clear_shape_coeffs()
    for k in range(mo.MUON_MAX_SHAPE_SCHEDULES):
        mo.muon_set_shape_coeffs(8, 8 + k, [(1, 0, 0)])
    with pytest.raises(mo.MuonError):
        mo.muon_set_shape_coeffs(8, 1000, [(1, 0, 0)])
    mo.muon_set_shape_coeffs(8, 8, [(2, 0, 0)])  # replacing an entry is still allowed when full
    mo.muon_reset_config()  # also clears the table
    assert mo.muon_get_shape_coeffs(8, 8) is None


def test_offload_argument_errors(lib):
    """muon_step_offload checks every argument before touching a device;
    valid arguments on a host without a GPU give MUON_ERR_CUDA."""
    vp = ctypes.c_void_p
    P = (vp * 2)(0x1000, 0x2000)
    Z = (vp * 2)(0x1000, None)
    S = (ctypes.c_int * 4)(4, 4, 8, 8)
    f = lib.muon_step_offload
    assert f(P, P, P, P, P, 0.95, 1, 1e-3, S, 2, 0) == mo.MUON_ERR_INVALID_ARG     # chunks < 1
    assert f(P, P, P, P, P, 0.95, 1, 1e-3, S, 0, 2) == mo.MUON_ERR_INVALID_ARG     # count < 1
    assert f(P, Z, P, P, P, 0.95, 1, 1e-3, S, 2, 2) == mo.MUON_ERR_INVALID_ARG     # null host grad
    assert f(P, P, P, P, Z, 0.95, 1, 1e-3, S, 2, 2) == mo.MUON_ERR_INVALID_ARG     # null host param
    assert f(P, P, Z, P, P, 0.95, 1, 1e-3, S, 2, 2) == mo.MUON_ERR_INVALID_ARG     # null device grad
    assert f(P, P, P, P, P, float("nan"), 1, 1e-3, S, 2, 2) == mo.MUON_ERR_INVALID_ARG
    import torch
    if not torch.cuda.is_available():
        assert f(P, P, P, P, P, 0.95, 1, 1e-3, S, 2, 2) == mo.MUON_ERR_CUDA
        assert f(P, None, P, P, None, 0.95, 1, 1e-3, S, 2, 1) == mo.MUON_ERR_CUDA


def _groups_by_definition(w, chunks):
    """The grouping rule stated in include/muon.h, applied by search: each
    bound is the first index after the previous one at which the running
    total reaches k/g of the whole (while a matrix remains for every later
    group), or at which only one matrix remains per later group."""
    n, g = len(w), min(chunks, len(w))
    if sum(w) == 0:
        w = [1] * n
    total = sum(w)
    bounds = [0]
    for k in range(1, g):
        cands = [j for j in range(bounds[-1] + 1, n + 1)
                 if n - j >= g - k and (sum(w[:j]) * g >= total * k or n - j == g - k)]
        bounds.append(cands[0])
    return bounds + [n]


def test_offload_grouping(lib):
    import random
    rng = random.Random(7)
    assert mo.muon_offload_chunks([10] * 8, 4) == [0, 2, 4, 6, 8]
    assert mo.muon_offload_chunks([1, 1, 1, 100], 4) == [0, 1, 2, 3, 4]   # a heavy tail still splits
    assert mo.muon_offload_chunks([5], 8) == [0, 1]
    assert mo.muon_offload_chunks([0, 0, 0], 2) == [0, 2, 3]             # all-zero weights count matrices
    for _ in range(300):
        n = rng.randint(1, 40)
        w = [rng.choice([0, 1, 7, 1000, rng.randint(0, 10 ** 9)]) for _ in range(n)]
        c = rng.randint(1, 12)
        b = mo.muon_offload_chunks(w, c)
        assert len(b) == min(c, n) + 1 and b[0] == 0 and b[-1] == n
        assert all(x < y for x, y in zip(b, b[1:]))
        assert b == _groups_by_definition(w, c), (w, c)
    # equal weights split evenly; a real layer set splits at layer bounds
    layer = [4096 * 4096, 1024 * 4096, 1024 * 4096, 4096 * 4096, 14336 * 4096, 14336 * 4096, 4096 * 14336]
    assert mo.muon_offload_chunks(layer * 32, 8) == list(range(0, 225, 28))
    for bad in [([1], 0), ([], 2), ([-1, 2], 2)]:
        with pytest.raises(mo.MuonError):
            mo.muon_offload_chunks(*bad)


def test_offload_binding_validates_host_tensors():
    import torch
    a = torch.zeros(4, 8, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        mo.muon_step_offload([a], [a], [a], grads_host=[a, a])   # one host tensor per parameter
    with pytest.raises(ValueError):
        mo.muon_step_offload([a], [a], [a], params_host=[a])     # not pinned
