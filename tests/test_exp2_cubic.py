"""The FMA-pipe 2^x of the bf16 prefill kernel (device_common.cuh, exp2_poly_pair).

The kernel computes one exponent pair in sixteen as 2^n * p(x - n), n = round(x),
with a cubic p fitted by relative-error least squares on 64 Chebyshev nodes of
[-1/2, 1/2] (csrc/exp2_cubic_fit.py).  CPU: the fit reproduces the constants in
the kernel source, and a float32 emulation of the kernel's steps stays within
the stated relative bound against fp64 2^x.  GPU: the device function itself
(through segpaged_eval_exp2_fma) meets the same bound.
"""
from __future__ import annotations

import importlib.util
import re
from pathlib import Path

import numpy as np
import pytest

ROOT = Path(__file__).resolve().parent.parent
CSRC = ROOT / "head_aware_paged_build_b200" / "csrc"
BOUND = 7.8e-5  # the cubic's 7.74e-5 plus the fp32 evaluation


def _fit_module():
    spec = importlib.util.spec_from_file_location("exp2_cubic_fit", CSRC / "exp2_cubic_fit.py")
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def kernel_coefficients() -> np.ndarray:
    """c0..c3 as written in exp2_poly_pair (Horner order in the source: c3, c2, c1, c0)."""
    src = (CSRC / "device_common.cuh").read_text()
    body = src[src.index("void exp2_poly_pair"):]
    body = body[:body.index("\n}\n")]
    vals = [float(x) for x in re.findall(r"f2_pack\(([0-9.]+)f, \1f\)", body)]
    vals = [v for v in vals if v not in (12582912.0,)]
    assert len(vals) == 4, vals
    return np.array(vals[::-1], dtype=np.float32)


def emulate(x: np.ndarray, c: np.ndarray) -> np.ndarray:
    """The kernel's steps in float32 (an FMA is emulated as an fp64 product-sum rounded once to fp32)."""
    f32 = np.float32
    x = np.maximum(x.astype(f32), f32(-126.0))
    r = f32(12582912.0)
    t = (x + r).astype(f32)
    j = (t - r).astype(f32)
    f = (x.astype(np.float64) - j.astype(np.float64)).astype(f32)
    fma = lambda a, b, cc: (np.asarray(a, np.float64) * np.asarray(b, np.float64) + np.float64(cc)).astype(f32)
    p = fma(np.full_like(f, c[3]), f, c[2])
    p = fma(p, f, c[1])
    p = fma(p, f, c[0])
    bits = (p.view(np.uint32).astype(np.uint64) + (t.view(np.uint32).astype(np.uint64) << np.uint64(23)))
    return (bits & np.uint64(0xFFFFFFFF)).astype(np.uint32).view(np.float32)


def test_fit_reproduces_the_kernel_constants():
    mod = _fit_module()
    c = mod.fit().astype(np.float32)
    assert np.array_equal(c, kernel_coefficients())
    assert mod.max_rel_error(c.astype(np.float64)) < 7.75e-5


def grid() -> np.ndarray:
    rng = np.random.default_rng(7)
    dense = np.linspace(-125.0, 8.0, 2_000_001, dtype=np.float64)
    near_half = np.concatenate([np.arange(-125, 8) + 0.5 + d for d in (-1e-6, 0.0, 1e-6)])
    rand = rng.uniform(-125.0, 8.0, 1_000_000)
    return np.concatenate([dense, near_half, rand]).astype(np.float32)


def test_emulated_kernel_meets_the_relative_bound():
    x = grid()
    y = emulate(x, kernel_coefficients()).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    assert float(np.max(np.abs(y / ref - 1.0))) <= BOUND
    # below the clamp (masked scores, -inf) the value is negligible and never negative
    low = emulate(np.array([-126.0, -130.0, -1e30, -np.inf], np.float32), kernel_coefficients())
    assert np.all(low >= 0) and np.all(low <= 2.0 ** -125)


@pytest.mark.gpu
def test_device_exp2_meets_the_relative_bound():
    import torch

    from head_aware_paged_build_b200 import segpaged as S

    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    x = torch.from_numpy(grid()).cuda()
    y = torch.empty_like(x)
    S.segpaged_eval_exp2_fma(x.data_ptr(), y.data_ptr(), x.numel(), torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    yd = y.cpu().double().numpy()
    ref = np.exp2(x.cpu().double().numpy())
    assert float(np.max(np.abs(yd / ref - 1.0))) <= BOUND
    # the device agrees with the float32 emulation of its steps to within one unit in the last place
    em = emulate(x.cpu().numpy(), kernel_coefficients())
    assert int(np.max(np.abs(y.cpu().numpy().view(np.int32).astype(np.int64) - em.view(np.int32)))) <= 1
    lo = torch.tensor([-126.0, -130.0, -1e30, float("-inf")], device="cuda")
    ylo = torch.empty_like(lo)
    S.segpaged_eval_exp2_fma(lo.data_ptr(), ylo.data_ptr(), 4, torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    assert bool((ylo >= 0).all()) and bool((ylo <= 2.0 ** -125).all())
