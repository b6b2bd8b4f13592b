"""Pins of the W4A4 oracle (oracle/w4a4.py): a pure-Python brute force on
tiny shapes whose quantiser searches the E4M3 and E2M1 grids directly (no
call into the oracle's encoders), the lossless case where x is already on the
NVFP4 grid (the hidden then equals the W4A16 oracle's, itself pinned by brute
force), and the size of the activation-quantisation error against W4A16."""
import math

import numpy as np
import pytest

import moe_inputs as gen
from oracle import formats as F
from oracle import moe as M
from oracle import w4a4 as W

E_T, K_T, H_T, I_T = 4, 2, 64, 32
GX, GH = np.float32(2.0 ** -7), np.float32(2.0 ** -9)


def tiny(seed=0, T=3):
    ex = gen.make_experts(seed, e=E_T, h=H_T, i=I_T)
    rt = gen.make_router(seed + 1, e=E_T, h=H_T, top_k=K_T)
    x = gen.make_x(seed + 2, T, H_T)
    return x, ex, rt


E2M1 = [F.e2m1_decode(c).item() for c in range(16)]
E4M3 = [(F.e4m3_decode(c).item(), c) for c in range(0x7F)]   # finite, non-negative


def _nearest(cands, v):
    """Nearest candidate value to v (exact real distance), ties to the even
    code; cands = [(value, code)]."""
    best = None
    for val, code in cands:
        key = (abs(val - v), code & 1)
        if best is None or key < best[0]:
            best = (key, val, code)
    return best[1], best[2]


def _bf_quantize_block(vals, G):
    """One block of 16 float32 values -> (scale code, 16 codes), by search."""
    f32 = np.float32
    amax = max(abs(float(v)) for v in vals)
    if G > 0:
        t = float(f32(f32(f32(amax) / f32(6.0)) / f32(G)))
        s_val, s_code = (448.0, 0x7E) if t >= 448.0 else _nearest(E4M3, t)
    else:
        s_val, s_code = 0.0, 0
    d = float(f32(f32(s_val) * f32(G)))
    codes = []
    for v in vals:
        sign = 8 if math.copysign(1.0, float(v)) < 0 else 0
        if d == 0:
            codes.append(sign)
            continue
        x = abs(float(f32(f32(v) / f32(d))))
        mag = 7 if x > 6.0 else _nearest([(E2M1[c], c) for c in range(8)], x)[1]
        codes.append(sign | mag)
    return s_code, codes


def _bf_quantize_rows(rows, G):
    """rows: list of lists of float32 -> list of (list of dequantised values)."""
    out = []
    for r in rows:
        deq = []
        for b in range(0, len(r), 16):
            s_code, codes = _bf_quantize_block(r[b:b + 16], G)
            sv = F.e4m3_decode(s_code).item()
            deq += [E2M1[c] * sv * float(G) for c in codes]
        out.append(deq)
    return out


def _brute_force_w4a4(x_bits, ex, rt, gx, gh):
    T, H = x_bits.shape
    I, k = ex.I, rt.top_k
    ids, w, _ = M.route(x_bits, rt)

    def weight(q, s, g, n, kk):
        byte = int(q[n, kk // 2])
        code = byte & 0xF if kk % 2 == 0 else byte >> 4
        return E2M1[code] * F.e4m3_decode(int(s[n, kk // 16])).item() * float(g)

    x32 = F.bf16_to_f32(x_bits)
    xq = _bf_quantize_rows([[x32[t, kk] for kk in range(H)] for t in range(T)], gx)
    y = [[0.0] * H for _ in range(T)]
    for t in range(T):
        for j in range(k):
            e = int(ids[t, j])
            gu = [sum(weight(ex.gate_up_q[e], ex.gate_up_s[e], ex.gate_up_g[e], n, kk) * xq[t][kk]
                      for kk in range(H)) for n in range(2 * I)]
            h = [0.5 * gu[n] * (1 + math.tanh(math.sqrt(2 / math.pi) * (gu[n] + 0.044715 * gu[n] ** 3)))
                 * gu[I + n] for n in range(I)]
            hq = _bf_quantize_rows([[np.float32(v) for v in h]], gh)[0]
            for n in range(H):
                o = sum(weight(ex.down_q[e], ex.down_s[e], ex.down_g[e], n, kk) * hq[kk] for kk in range(I))
                y[t][n] += float(w[t, j]) * o
    return np.array(y)


@pytest.mark.parametrize("seed", [3, 4])
def test_forward_vs_pure_python_brute_force(seed):
    x, ex, rt = tiny(seed)
    got = W.forward(x, ex, rt, GX, GH)
    want = _brute_force_w4a4(x, ex, rt, GX, GH)
    assert np.allclose(got, want, rtol=1e-11, atol=1e-13 * np.abs(want).max())


def test_quantize_act_vs_grid_search():
    rng = np.random.default_rng(5)
    v = (rng.standard_normal((6, 64)) * np.exp(rng.uniform(-3, 3, (6, 1)))).astype(np.float32)
    v[0, :16] = 0.0
    v[1, 16:32] = -0.0
    v[2, 5] = 1e4                       # block scale saturates at 448
    q, s = W.quantize_act(v, GX)
    codes = F.unpack_nibbles(q)
    for r in range(v.shape[0]):
        for b in range(4):
            s_code, cs = _bf_quantize_block(list(v[r, 16 * b:16 * b + 16]), GX)
            assert s[r, b] == s_code
            assert codes[r, 16 * b:16 * b + 16].tolist() == cs


def _on_grid_x(rng, T, H, gx):
    """bf16 activations that NVFP4 with global gx reproduces exactly: every
    block holds a +-6 code and a scale below 448."""
    codes = rng.integers(0, 16, size=(T, H), dtype=np.uint8)
    for t in range(T):
        for b in range(H // 16):
            codes[t, 16 * b + rng.integers(0, 16)] = rng.choice([0x7, 0xF])
    sc = rng.integers(0x20, 0x60, size=(T, H // 16), dtype=np.uint8)
    v = np.repeat(F.e4m3_decode(sc), 16, axis=1) * F.e2m1_decode(codes) * float(gx)
    bits = gen.bf16_bits(v.astype(np.float32))
    assert np.array_equal(F.bf16_to_f64(bits), v)
    return bits, codes, sc


def test_on_grid_activations_are_lossless_and_give_the_w4a16_hidden():
    x, ex, rt = tiny(7, T=4)
    bits, codes, sc = _on_grid_x(np.random.default_rng(8), 4, H_T, GX)
    parts = W.forward(bits, ex, rt, GX, GH, return_parts=True)
    assert np.array_equal(F.unpack_nibbles(parts["xq"]), codes)
    assert np.array_equal(parts["xs"], sc)
    xf = F.bf16_to_f64(bits)
    for t in range(4):
        for j in range(K_T):
            wgu, _ = M.expert_dense(ex, int(parts["ids"][t, j]))
            want = M.expert_hidden(xf[t:t + 1], wgu)[0].astype(np.float32)
            assert np.array_equal(parts["h32"][t * K_T + j], want)


def test_down_from_codes_matches_forward():
    x, ex, rt = tiny(9, T=4)
    parts = W.forward(x, ex, rt, GX, GH, return_parts=True)
    y = W.down_from_codes(parts["hq"], parts["hs"], GH, parts["ids"], parts["w"], ex, 4)
    assert np.allclose(y, parts["y64"], rtol=1e-12, atol=1e-15)


def test_activation_quantisation_error_is_that_of_fp4():
    """Against W4A16 on the full-size layer: each NVFP4 rounding of an
    activation row costs about 10% relative rms error per element (E2M1 has
    one mantissa bit; a block's largest element sets its scale), and with
    weights uncorrelated with the errors y inherits about that much per
    rounding, two roundings in all: well below 30%, and far from the factor
    a wrong global or a dropped scale would give."""
    ex = gen.make_experts(0, e=8)
    rt = gen.make_router(0, e=8)
    x = gen.make_x(1, 2)
    y4 = W.forward(x, ex, rt, gen.W4A4_GX, gen.W4A4_GH)
    y16 = M.forward(x, ex, rt)
    rel = np.linalg.norm(y4 - y16) / np.linalg.norm(y16)
    assert 0.02 < rel < 0.3, rel
