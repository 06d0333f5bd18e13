"""Accuracy of the two exponentials the tensor-core importance kernel mixes,
through the fc_selftest_exp2 C-ABI entry: the special-function unit
(ex2.approx) and the FMA-pipe range reduction + degree-3 polynomial, against
numpy's float64 exp2 (relative error bounds: 7.6e-5 for the polynomial, the
maximum of its float32 evaluation over [-1/2, 1/2] that the fitting script
prints; 2^-21 for the special-function unit) and against each other."""

import ctypes

import numpy as np
import pytest
import torch

import cache_gating_kv_b200 as fc

pytestmark = pytest.mark.gpu


def _run(x):
    lib = fc.library()
    lib.fc_selftest_exp2.restype = ctypes.c_int
    lib.fc_selftest_exp2.argtypes = [ctypes.c_void_p] * 3 + [ctypes.c_int, ctypes.c_void_p]
    xd = torch.from_numpy(x.astype(np.float32)).cuda()
    ym = torch.empty_like(xd)
    yp = torch.empty_like(xd)
    st = lib.fc_selftest_exp2(xd.data_ptr(), ym.data_ptr(), yp.data_ptr(), xd.numel(),
                              torch.cuda.current_stream().cuda_stream)
    assert st == 0, lib.fc_last_error()
    torch.cuda.synchronize()
    return ym.cpu().numpy(), yp.cpu().numpy()


def test_polynomial_exp2_relative_error():
    rng = np.random.default_rng(0)
    x = np.concatenate([np.linspace(-125, 126, 400002), rng.uniform(-30, 1, 200000),
                        np.arange(-125, 127).astype(np.float64) + 0.5, [0.0, -0.0, 1e-7]])
    x = x[: x.size // 2 * 2].astype(np.float32)
    ym, yp = _run(x)
    ref = np.exp2(x.astype(np.float64))
    rel_p = np.abs(yp - ref) / ref
    assert rel_p.max() < 7.6e-5, rel_p.max()
    normal = x >= -126
    rel_m = np.abs(ym[normal] - ref[normal]) / ref[normal]
    assert rel_m.max() < 2.0 ** -21
    assert np.all(yp > 0)


def test_polynomial_exp2_clamps_below():
    x = np.array([-np.inf, -1e30, -200.0, -125.0], np.float32)
    ym, yp = _run(x)
    assert np.all(ym[:3] == 0)
    np.testing.assert_allclose(yp, 2.0 ** -125, rtol=7.6e-5)


def test_bounded_wait_gives_up_and_context_stays_usable():
    """A wait on an mbarrier nothing arrives on returns after its limit and
    records an error word; the context keeps working afterwards."""
    lib = fc.library()
    lib.fc_selftest_wait_timeout.restype = ctypes.c_int
    lib.fc_selftest_wait_timeout.argtypes = [ctypes.c_longlong, ctypes.c_void_p, ctypes.c_void_p]
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    st = lib.fc_selftest_wait_timeout(2_000_000, err.data_ptr(),
                                      torch.cuda.current_stream().cuda_stream)
    assert st == 0, lib.fc_last_error()
    torch.cuda.synchronize()
    assert int(err.item()) == 1
    # the device is still usable: a regular library call succeeds
    ym, yp = _run(np.array([0.0, 1.0], np.float32))
    assert ym[1] == 2.0 and abs(yp[1] - 2.0) < 2 * 7.6e-5
