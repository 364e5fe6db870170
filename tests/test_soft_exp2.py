"""The attention kernel's software exp2 (Cody-Waite reduction + fitted cubic),
replayed in float32 on the host: relative error, the exponent-field add and
the clamps that keep very negative inputs (masked scores) tiny and very large
ones (a score far above the running max) finite and huge."""
import numpy as np


def soft_exp2_f32(x):
    f32 = np.float32
    x = np.minimum(np.maximum(x.astype(f32), f32(-126.0)), f32(127.0))
    t = (x + f32(12582912.0)).astype(f32)
    f = (x - (t - f32(12582912.0))).astype(f32)
    p = (f32(0.05521968) * f + f32(0.24260941)).astype(f32)
    p = (p * f + f32(0.69325167)).astype(f32)
    p = (p * f + f32(0.99992800)).astype(f32)
    bits = (p.view(np.uint32).astype(np.uint64) + (t.view(np.uint32).astype(np.uint64) << 23)) & 0xFFFFFFFF
    return bits.astype(np.uint32).view(np.float32)


def test_relative_error_and_range():
    x = np.linspace(-120.0, 8.0, 400001).astype(np.float32)
    y = soft_exp2_f32(x).astype(np.float64)
    rel = np.abs(y - np.exp2(x.astype(np.float64))) / np.exp2(x.astype(np.float64))
    assert rel.max() < 1e-4            # far below bf16's half ulp (2^-9)


def test_masked_and_tiny_inputs_stay_finite_and_tiny():
    x = np.array([-np.inf, -1e30, -300.0, -127.5, -126.0], dtype=np.float32)
    y = soft_exp2_f32(x)
    assert np.all(np.isfinite(y)) and np.all(y >= 0) and np.all(y < 1e-37)


def test_large_inputs_stay_finite_and_huge():
    """An argument far above the running max must not wrap the exponent field:
    the result stays finite and above the softmax's partial-sum limit (1024),
    so the half is redone against a raised running max."""
    x = np.array([10.5, 127.0, 128.0, 200.0, 369.0, 1e30, np.inf], dtype=np.float32)
    y = soft_exp2_f32(x)
    assert np.all(np.isfinite(y)) and np.all(y > 1024.0)
    assert np.all(y[1:] >= np.float32(2.0 ** 126))
