"""The FMA-pipe exponential of the multi-query kernel's softmax (exp2_poly):
its range reduction and polynomial checked on the CPU in fp32 arithmetic
against numpy's exp2 (relative error < 1e-5 over the whole range the softmax
uses, exact 0 below -126), and the device function against exp2 in fp64."""
import os

import numpy as np
import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(os.path.dirname(HERE), "paged_kv_cache_437_b200", "csrc", "mq_attention.cuh")


def _coefficients():
    # the constants as they stand in the kernel source
    import re

    text = open(SRC).read()
    body = text[text.index("float exp2_poly(float x)"):]
    body = body[:body.index("return x < -126.f")]
    nums = [float(v) for v in re.findall(r"(-?\d+\.\d+)f", body)]
    # the Horner chain's constants, highest degree first: c4, c3, c2, c1, c0
    assert len(nums) == 5
    return nums


def _emulate(x):
    x = np.asarray(x, dtype=np.float32)
    c = _coefficients()
    c4, c3, c2, c1, c0 = (np.float32(v) for v in c)
    xc = np.maximum(x, np.float32(-126.0))
    magic = np.float32(12582912.0)
    t = (xc + magic).astype(np.float32)
    f = (xc - (t - magic)).astype(np.float32)
    p = (f * c4 + c3).astype(np.float32)
    p = (p * f + c2).astype(np.float32)
    p = (p * f + c1).astype(np.float32)
    p = (p * f + c0).astype(np.float32)
    n = t.view(np.int32) - np.int32(0x4B400000)
    r = (p.view(np.int32) + (n << 23)).view(np.float32)
    return np.where(x < -126.0, np.float32(0.0), r)


def test_source_constants_are_the_fit():
    import importlib.util

    spec = importlib.util.spec_from_file_location(
        "gen", os.path.join(os.path.dirname(SRC), "gen_exp2_poly.py"))
    gen = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(gen)
    c, err = gen.fit()
    assert err < 1e-5
    got = _coefficients()
    assert np.allclose(got, c[::-1], rtol=0, atol=5e-9)


def test_cpu_emulation_error_bound():
    x = np.concatenate([np.linspace(-126.0, 8.0, 2_000_001, dtype=np.float32),
                        np.float32([-0.5, 0.5, 0.0, -1.0, 1.0, 7.99, -125.5])])
    got = _emulate(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    assert np.max(np.abs(got / ref - 1.0)) < 1e-5
    assert np.all(_emulate(np.float32([-126.5, -200.0, -np.inf])) == 0.0)


@pytest.mark.gpu
def test_device_exp2_poly():
    import torch

    import paged_kv_cache_437_b200 as pkv

    x = torch.cat([torch.linspace(-126.0, 8.0, 1 << 21), torch.tensor([-126.5, -300.0, float("-inf"), 0.0])]).cuda()
    y = torch.empty_like(x)
    assert pkv.lib.pkv_test_exp2_poly(x.data_ptr(), y.data_ptr(), x.numel(), pkv._stream_ptr(None)) == pkv.PKV_OK
    torch.cuda.synchronize()
    xs, ys = x.cpu().double().numpy(), y.cpu().double().numpy()
    ok = xs >= -126.0
    assert np.max(np.abs(ys[ok] / np.exp2(xs[ok]) - 1.0)) < 1e-5
    assert np.all(ys[~ok] == 0.0)
    # the CPU emulation of the same steps agrees to the last bit (same fp32
    # operations; the device may fuse differently only where it uses fmaf)
    emu = _emulate(x.cpu().numpy()).astype(np.float64)
    assert np.max(np.abs(ys[ok] / emu[ok] - 1.0)) < 2e-7
