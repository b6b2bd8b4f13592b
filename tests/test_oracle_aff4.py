"""Pins of the aff4 codec oracle (oracle/aff4.py): the nibble order against a
hand table, the affine form on all 16 codes, the page's q4_0 identity
(scale = d, bias = -8 d gives (q - 8) d exactly), and a pure-Python brute
force of the routed forward through aff4 experts."""
import math

import numpy as np

import moe_inputs as gen
from oracle import aff4 as A
from oracle import formats as F
from oracle import moe as M


def f16(v):
    return np.array(v, np.float16).view(np.uint16)


def test_unpack_hand_table():
    # byte 0x3A: element 0 = 0xA (low nibble), element 1 = 0x3
    q = np.array([[0x3A, 0xF0, 0x01]], np.uint8)
    assert A.unpack_u4(q).tolist() == [[10, 3, 0, 15, 1, 0]]


def test_affine_form_on_all_codes():
    codes = np.arange(16, dtype=np.uint8)
    q = (codes[0::2] | (codes[1::2] << 4)).astype(np.uint8)[None, :]         # 16 codes, one row
    q = np.concatenate([q, q], axis=1)                                      # K = 32: one block
    s, b = 0.0625, -0.4375                                                  # exact in fp16
    w = A.dequantize(q, f16([[s]]), f16([[b]]))
    assert w.shape == (1, 32)
    assert np.array_equal(w[0, :16], np.arange(16) * s + b)


def test_q4_0_grid_is_represented_exactly():
    """The page: a q4_0 grid w = (q - 8) d is an aff4 block with scale = d,
    bias = -8 d."""
    rng = np.random.default_rng(0)
    codes = rng.integers(0, 16, size=(4, 64)).astype(np.uint8)
    q = (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)
    d = np.array([[2.0 ** -9 * 1.25, 2.0 ** -7], [3.0 * 2 ** -12, 2.0 ** -10], [1.0, 0.5], [2 ** -14, 2 ** -6]])
    w = A.dequantize(q, f16(d), f16(-8 * d))
    want = (codes.astype(np.float64) - 8) * np.repeat(d, 32, axis=1)
    assert np.array_equal(w, want)


def _aff4_tiny(seed, e=4, h=64, i=32):
    gq, gs, gb, dq, ds, db = gen.make_aff4_experts(seed, e=e, h=h, i=i)
    return A.Aff4Experts(gq, gs, gb, dq, ds, db)


def test_forward_through_aff4_vs_pure_python():
    ex = _aff4_tiny(3)
    rt = gen.make_router(4, e=4, h=64, top_k=2)
    x = gen.make_x(5, 3, 64)
    got = M.forward(x, ex, rt)
    f = lambda b: float(np.asarray(b, np.uint16).view(np.float16))  # noqa: E731

    def w(q, s, b, n, k):
        byte = int(q[n, k // 2])
        c = byte & 0xF if k % 2 == 0 else byte >> 4
        return c * f(s[n, k // 32]) + f(b[n, k // 32])

    gelu = lambda g: 0.5 * g * (1 + math.tanh(math.sqrt(2 / math.pi) * (g + 0.044715 * g ** 3)))  # noqa: E731
    ids, wts, _ = M.route(x, rt)
    want = np.zeros((3, 64))
    for t in range(3):
        xt = [F.bf16_to_f64(x[t, k]).item() for k in range(64)]
        for j, e in enumerate(ids[t]):
            gu = [sum(w(ex.gate_up_q[e], ex.gate_up_s[e], ex.gate_up_b[e], n, k) * xt[k] for k in range(64))
                  for n in range(64)]
            hh = [gelu(gu[n]) * gu[32 + n] for n in range(32)]
            for n in range(64):
                want[t, n] += wts[t, j] * sum(w(ex.down_q[e], ex.down_s[e], ex.down_b[e], n, k) * hh[k]
                                              for k in range(32))
    assert np.allclose(got, want, rtol=1e-11, atol=1e-13 * np.abs(want).max())
