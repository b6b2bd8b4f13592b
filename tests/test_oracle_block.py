"""Pins of the full-block oracle (oracle/block.py): torch's rms_norm, linear
and gelu for its pieces, a pure-Python brute force of the whole layer
dataflow listing on tiny shapes, and properties a misplaced norm, a wrong
router input or a missing residual would break."""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as TF

import moe_inputs as gen
from oracle import block as B
from oracle import formats as F
from oracle import moe as M

H_T, DI_T, E_T, I_T, K_T = 64, 24, 4, 32, 2


def tiny_block(seed=0, eps=1e-6):
    ex = gen.make_experts(seed, e=E_T, h=H_T, i=I_T)
    rt = gen.make_router(seed + 1, e=E_T, h=H_T, top_k=K_T)
    b = gen.make_block(seed + 2, h=H_T, di=DI_T)
    return B.BlockParams(ex, rt, b.dense_gate, b.dense_up, b.dense_down, b.pre_ff_norm, b.post_ff_norm_1,
                         b.pre_ff_norm_2, b.post_ff_norm_2, b.post_ff_norm, b.layer_scalar, eps)


def t64(bits):
    return torch.from_numpy(F.bf16_to_f64(bits))


def test_rmsnorm_and_dense_mlp_vs_torch():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((5, H_T)) * 3
    p = tiny_block()
    want = TF.rms_norm(torch.from_numpy(x), (H_T,), weight=t64(p.pre_ff_norm), eps=1e-6).numpy()
    assert np.allclose(B.rmsnorm(x, p.pre_ff_norm, 1e-6), want, rtol=1e-14, atol=0)
    xt = torch.from_numpy(x)
    h = TF.linear(TF.gelu(TF.linear(xt, t64(p.dense_gate)), approximate="tanh") * TF.linear(xt, t64(p.dense_up)),
                  t64(p.dense_down))
    assert np.allclose(B.dense_mlp(x, p.dense_gate, p.dense_up, p.dense_down), h.numpy(), rtol=1e-12, atol=1e-15)


def _brute_force_block(x_bits, p):
    """The layer dataflow listing element by element in pure Python (the
    experts' weights decoded from their E2M1 / E4M3 / FP32 storage)."""
    T, H = x_bits.shape
    ex, rt = p.experts, p.router
    e2m1 = [F.e2m1_decode(c).item() for c in range(16)]
    e4m3 = [F.e4m3_decode(c).item() for c in range(256)]
    bf = lambda a: [float(v) for v in F.bf16_to_f64(np.asarray(a)).ravel()]  # noqa: E731
    gelu = lambda g: 0.5 * g * (1 + math.tanh(math.sqrt(2 / math.pi) * (g + 0.044715 * g ** 3)))  # noqa: E731

    def norm(v, w):
        inv = 1.0 / math.sqrt(sum(a * a for a in v) / len(v) + p.eps)
        return [a * inv * b for a, b in zip(v, bf(w))]

    def to_bf16(v):
        return bf(F.f64_to_bf16_rne(np.array(v)))

    def wq(q, s, g, n, k):
        byte = int(q[n, k // 2])
        return e2m1[byte & 0xF if k % 2 == 0 else byte >> 4] * e4m3[int(s[n, k // 16])] * float(g)

    Wg, Wu = np.array(bf(p.dense_gate)).reshape(DI_T, H), np.array(bf(p.dense_up)).reshape(DI_T, H)
    Wd = np.array(bf(p.dense_down)).reshape(H, DI_T)
    out = []
    for t in range(T):
        res = bf(x_bits[t])
        x1 = to_bf16(norm(res, p.pre_ff_norm))
        gd = [sum(Wg[n, k] * x1[k] for k in range(H)) for n in range(DI_T)]
        ud = [sum(Wu[n, k] * x1[k] for k in range(H)) for n in range(DI_T)]
        hd = [gelu(a) * b for a, b in zip(gd, ud)]
        h = [sum(Wd[n, k] * hd[k] for k in range(DI_T)) for n in range(H)]
        h1 = norm(h, p.post_ff_norm_1)
        # router on the raw residual
        inv = 1.0 / math.sqrt(sum(a * a for a in res) / H + rt.eps)
        r = [res[k] * inv * bf(rt.scale)[k] * H ** -0.5 for k in range(H)]
        proj = np.array(bf(rt.proj)).reshape(E_T, H)
        logits = [sum(r[k] * proj[e, k] for k in range(H)) for e in range(E_T)]
        m = max(logits)
        pr = [math.exp(l - m) for l in logits]
        pr = [v / sum(pr) for v in pr]
        sel = sorted(range(E_T), key=lambda e: (-pr[e], e))[:K_T]
        ps = sum(pr[e] for e in sel)
        x2 = to_bf16(norm(res, p.pre_ff_norm_2))
        y = [0.0] * H
        for e in sel:
            we = pr[e] / ps * bf(rt.per_expert_scale)[e]
            gu = [sum(wq(ex.gate_up_q[e], ex.gate_up_s[e], ex.gate_up_g[e], n, k) * x2[k] for k in range(H))
                  for n in range(2 * I_T)]
            he = [gelu(gu[n]) * gu[I_T + n] for n in range(I_T)]
            for n in range(H):
                y[n] += we * sum(wq(ex.down_q[e], ex.down_s[e], ex.down_g[e], n, k) * he[k] for k in range(I_T))
        h2 = norm(y, p.post_ff_norm_2)
        s = norm([a + b for a, b in zip(h1, h2)], p.post_ff_norm)
        out.append([(a + b) * bf(p.layer_scalar)[0] for a, b in zip(res, s)])
    return np.array(out)


@pytest.mark.parametrize("seed", [0, 5])
def test_block_vs_pure_python_brute_force(seed):
    p = tiny_block(seed)
    x = gen.make_x(seed + 10, 2, H_T)
    got = B.forward(x, p)
    want = _brute_force_block(x, p)
    assert np.allclose(got, want, rtol=1e-10, atol=1e-12 * np.abs(want).max())


def test_router_reads_the_raw_residual():
    """With a non-uniform pre_feedforward_layernorm_2 weight the normed and
    the raw residual route differently; the block routes on the raw one."""
    p = tiny_block(3)
    p.router = gen.make_router(4, e=128, h=H_T)
    p.experts = gen.make_experts(3, e=128, h=H_T, i=I_T)
    p.pre_ff_norm_2 = gen.bf16_bits(np.random.default_rng(9).uniform(0.1, 3.0, H_T).astype(np.float32))
    x = gen.make_x(11, 16, H_T)
    parts = B.forward(x, p, return_parts=True)
    assert np.array_equal(parts["ids"], M.route(x, p.router)[0])
    assert not np.array_equal(parts["ids"], M.route(parts["x2"], p.router)[0])


def test_zero_post_norm_leaves_the_scaled_residual():
    p = tiny_block(6)
    p.post_ff_norm = np.zeros(H_T, np.uint16)
    x = gen.make_x(12, 3, H_T)
    assert np.array_equal(B.forward(x, p), F.bf16_to_f64(x) * F.bf16_to_f64(p.layer_scalar)[0])


def test_feedforward_part_is_invariant_to_the_residual_scale():
    """With eps = 0 every norm, and so the whole feed-forward part, ignores a
    power-of-two scale of x, while the residual scales with it:
    out(c x) - c x s = out(x) - x s."""
    p = tiny_block(7, eps=0.0)
    p.router.eps = 0.0
    x = gen.make_x(13, 4, H_T)
    s = F.bf16_to_f64(p.layer_scalar)[0]
    X = F.bf16_to_f64(x)
    f1 = B.forward(x, p) - X * s
    for c in (4.0, 2.0 ** -6):
        xc = gen.bf16_bits((X * c).astype(np.float32))
        fc = B.forward(xc, p) - X * c * s
        assert np.allclose(fc, f1, rtol=1e-9, atol=1e-9 * np.abs(f1).max())
