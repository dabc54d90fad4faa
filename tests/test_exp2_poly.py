"""The softmax kernels' FMA-pipe exponential (veda_ptx.cuh, exp2_fma_x2), pinned on the CPU
against the exact 2^x: its constants are read from the kernel source and its steps are
emulated in fp32 (each fused multiply-add rounded once, from the exact fp64 product)."""
import math
import pathlib
import re

import numpy as np

SRC = pathlib.Path(__file__).resolve().parents[1] / "block_sparse_attention_max_b200" / "csrc"


def _constants():
    text = (SRC / "veda_ptx.cuh").read_text()
    c = [float(re.search(rf"kExp2C{k} = ([0-9.e-]+)f", text).group(1)) for k in range(5)]
    shift = re.search(r"kExp2Shift = ([0-9.]+)f \+ ([0-9.]+)f", text)
    return np.array(c, dtype=np.float32), np.float32(float(shift.group(1)) + float(shift.group(2)))


def _f32(x):
    return np.float32(x)


def _fma(a, b, c):
    return _f32(np.float64(a) * np.float64(b) + np.float64(c))


def _exp2_kernel(x, c, shift):
    x = _f32(max(_f32(x), _f32(-127.0)))
    t = _f32(x + shift)
    j = _f32(t + (-shift))
    f = _fma(j, _f32(-1.0), x)
    p = _fma(c[4], f, c[3])
    for k in (2, 1, 0):
        p = _fma(p, f, c[k])
    bits = (int(np.array([t], dtype=np.float32).view(np.uint32)[0]) << 23) & 0xFFFFFFFF
    scale = np.array([bits], dtype=np.uint32).view(np.float32)[0]
    return _f32(p * scale)


def test_constants_match_the_fit_script():
    import importlib.util
    spec = importlib.util.spec_from_file_location("fit_exp2_poly", SRC / "fit_exp2_poly.py")
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    coeffs, err = mod.fit()
    c, shift = _constants()
    assert np.array_equal(coeffs, c)
    assert err < 3e-6
    assert shift == np.float32(1.5 * 2 ** 23 + 127)


def test_relative_error_on_the_whole_range_and_exact_zeros():
    c, shift = _constants()
    rng = np.random.default_rng(7)
    xs = np.concatenate([np.linspace(-126.0, 0.0, 60001), -30.0 * rng.random(20000), -rng.random(5000),
                         np.arange(-126, 1, dtype=np.float64), np.arange(-126, 0) + 0.5])
    worst = max(abs(float(_exp2_kernel(x, c, shift)) - 2.0 ** float(np.float32(x))) / 2.0 ** float(np.float32(x))
                for x in xs)
    assert worst < 1e-5, worst
    for x in (-127.0, -127.5, -200.0, -math.inf):
        assert _exp2_kernel(x, c, shift) == 0.0
    assert _exp2_kernel(0.0, c, shift) == np.float32(c[0])     # 2^0 = C0 (1 - 7e-7)
    assert _exp2_kernel(-1.0, c, shift) == np.float32(c[0] * 0.5)
