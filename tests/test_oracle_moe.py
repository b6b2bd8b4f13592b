"""Pins of the oracle's router, permutation and expert maths: library routines
(torch rms_norm / softmax / gelu / topk), invariants (renormalised weights sum
to one, softmax-then-renormalise = softmax over the selected logits,
equivariance under expert and token permutations), a pure-Python dense
brute force over all experts on tiny shapes, and the identical-experts case
that reduces to a plain matmul chain."""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as TF

import moe_inputs as gen
from oracle import formats as F
from oracle import moe as M
from oracle import quantize as Q

E_T, K_T, H_T, I_T = 4, 2, 64, 32   # tiny shapes


def tiny(seed=0, T=5, bias=False):
    ex = gen.make_experts(seed, e=E_T, h=H_T, i=I_T)
    b = np.random.default_rng(seed).normal(0, 0.01, E_T).astype(np.float32) if bias else None
    rt = gen.make_router(seed + 1, e=E_T, h=H_T, bias=b, top_k=K_T)
    x = gen.make_x(seed + 2, T, H_T)
    return x, ex, rt


# ------------------------------------------------------------------- library
def test_rmsnorm_softmax_gelu_vs_torch():
    rng = np.random.default_rng(0)
    x = rng.standard_normal((7, 96))
    ref = TF.rms_norm(torch.from_numpy(x), (96,), eps=1e-6).numpy()
    assert np.allclose(M.rmsnorm_scale_free(x, 1e-6), ref, rtol=1e-14, atol=0)
    lg = rng.standard_normal((7, 128)) * 5
    assert np.allclose(M.softmax(lg), torch.softmax(torch.from_numpy(lg), -1).numpy(), rtol=1e-13, atol=1e-300)
    g = np.linspace(-8, 8, 1001)
    ref = TF.gelu(torch.from_numpy(g), approximate="tanh").numpy()
    assert np.allclose(M.gelu_tanh(g), ref, rtol=1e-13, atol=1e-15)
    # GELU-tanh, not SiLU and not the erf form
    assert abs(M.gelu_tanh(np.array([1.0]))[0] - 0.8411919906082768) < 1e-15


def test_router_vs_torch_ops():
    x, _, _ = tiny()
    rt = gen.make_router(3, e=128, h=H_T)
    ids, w, logits = M.route(x, rt)
    xt = torch.from_numpy(F.bf16_to_f64(x))
    r = TF.rms_norm(xt, (H_T,), eps=rt.eps) * torch.from_numpy(F.bf16_to_f64(rt.scale)) * H_T ** -0.5
    lg = TF.linear(r, torch.from_numpy(F.bf16_to_f64(rt.proj)))
    assert np.allclose(logits, lg.numpy(), rtol=1e-12, atol=1e-15)
    p = torch.softmax(lg, -1)
    top = torch.topk(p, 8, dim=-1)
    assert np.array_equal(ids, top.indices.numpy())
    wref = top.values / top.values.sum(-1, keepdim=True) * torch.from_numpy(F.bf16_to_f64(rt.per_expert_scale))[top.indices]
    assert np.allclose(w, wref.numpy(), rtol=1e-12)


def test_top_k_ties_lower_id_first():
    p = np.array([[0.1, 0.3, 0.3, 0.2, 0.3, 0.05]])
    assert M.top_k(p, 4).tolist() == [[1, 2, 4, 3]]


# ---------------------------------------------------------------- invariants
def test_weights_sum_to_one_before_per_expert_scale():
    x, _, rt = tiny(T=9)
    rt = gen.make_router(5, e=128, h=H_T)
    rt.per_expert_scale = gen.bf16_bits(np.ones(128, np.float32))
    _, w, _ = M.route(x, rt)
    assert np.allclose(w.sum(-1), 1.0, rtol=0, atol=1e-14)


def test_softmax_then_renormalise_equals_softmax_over_selected_logits():
    x = gen.make_x(7, 16, H_T)
    rt = gen.make_router(8, e=128, h=H_T)
    ids, w, logits = M.route(x, rt)
    sel = np.take_along_axis(logits, ids.astype(np.int64), -1)
    alt = M.softmax(sel) * F.bf16_to_f64(rt.per_expert_scale)[ids]
    assert np.allclose(w, alt, rtol=1e-13)


def test_expert_permutation_equivariance():
    x = gen.make_x(9, 12, H_T)
    rt = gen.make_router(10, e=128, h=H_T, bias=np.random.default_rng(1).normal(0, .01, 128).astype(np.float32))
    perm = np.random.default_rng(2).permutation(128)
    rt2 = gen.Router(rt.proj[perm], rt.scale, rt.per_expert_scale[perm], rt.logit_bias[perm], rt.eps, rt.top_k)
    ids, w, _ = M.route(x, rt)
    ids2, w2, _ = M.route(x, rt2)
    assert np.array_equal(perm[ids2], ids)
    assert np.allclose(w2, w, rtol=1e-13)


def test_token_permutation_invariance_of_forward():
    x, ex, rt = tiny(T=6, bias=True)
    perm = np.random.default_rng(3).permutation(6)
    y = M.forward(x, ex, rt)
    y2 = M.forward(x[perm], ex, rt)
    assert np.allclose(y2, y[perm], rtol=1e-13, atol=1e-18)


def test_permute_is_stable_and_consistent():
    rng = np.random.default_rng(4)
    ids = np.stack([rng.choice(16, 4, replace=False) for _ in range(50)]).astype(np.int32)
    counts, offsets, ss, pos = M.permute(ids, 16)
    flat = ids.ravel()
    assert counts.sum() == flat.size and offsets[-1] == flat.size
    for e in range(16):
        seg = ss[offsets[e]:offsets[e + 1]]
        assert np.all(flat[seg] == e) and np.all(np.diff(seg) > 0)
    assert np.array_equal(ss[pos], np.arange(flat.size))


# ---------------------------------------------------------------- brute force
def _brute_force_forward(x_bits, ex, rt):
    """Pure-Python dense evaluation: every expert on every token, each output
    weighted by the token's routing weight for that expert (0 if unselected).
    Element values come from the E2M1 / E4M3 / bf16 decoders (pinned above)."""
    T, H = x_bits.shape
    E, I, k = ex.E, ex.I, rt.top_k
    e2m1 = [F.e2m1_decode(c).item() for c in range(16)]
    e4m3 = [F.e4m3_decode(c).item() for c in range(256)]

    def weight(q, s, g, n, kk):
        byte = int(q[n, kk // 2])
        code = byte & 0xF if kk % 2 == 0 else byte >> 4
        return e2m1[code] * e4m3[int(s[n, kk // 16])] * float(g)

    def bf(b):
        return F.bf16_to_f64(b).item()

    y = [[0.0] * H for _ in range(T)]
    for t in range(T):
        xt = [bf(x_bits[t, kk]) for kk in range(H)]
        inv = 1.0 / math.sqrt(sum(v * v for v in xt) / H + rt.eps)
        r = [xt[kk] * inv * bf(rt.scale[kk]) * H ** -0.5 for kk in range(H)]
        logits = [sum(r[kk] * bf(rt.proj[e, kk]) for kk in range(H)) for e in range(E)]
        if rt.logit_bias is not None:
            logits = [l + float(b) for l, b in zip(logits, rt.logit_bias)]
        m = max(logits)
        ex_ = [math.exp(l - m) for l in logits]
        p = [v / sum(ex_) for v in ex_]
        sel = sorted(range(E), key=lambda e: (-p[e], e))[:k]
        psum = sum(p[e] for e in sel)
        mask = [p[e] / psum * bf(rt.per_expert_scale[e]) if e in sel else 0.0 for e in range(E)]
        for e in range(E):
            gu = [sum(weight(ex.gate_up_q[e], ex.gate_up_s[e], ex.gate_up_g[e], n, kk) * xt[kk]
                      for kk in range(H)) for n in range(2 * I)]
            h = [0.5 * gu[n] * (1 + math.tanh(math.sqrt(2 / math.pi) * (gu[n] + 0.044715 * gu[n] ** 3)))
                 * gu[I + n] for n in range(I)]
            for n in range(H):
                o = sum(weight(ex.down_q[e], ex.down_s[e], ex.down_g[e], n, kk) * h[kk] for kk in range(I))
                y[t][n] += mask[e] * o
    return np.array(y)


@pytest.mark.parametrize("bias", [False, True])
def test_forward_vs_pure_python_dense_brute_force(bias):
    x, ex, rt = tiny(seed=11, T=3, bias=bias)
    got = M.forward(x, ex, rt)
    want = _brute_force_forward(x, ex, rt)
    assert np.allclose(got, want, rtol=1e-11, atol=1e-13 * np.abs(want).max())


def test_identical_experts_reduce_to_matmul_chain():
    x, ex, rt = tiny(seed=12, T=8)
    for a in (ex.gate_up_q, ex.gate_up_s, ex.down_q, ex.down_s):
        a[:] = a[0]
    ex.gate_up_g[:] = ex.gate_up_g[0]
    ex.down_g[:] = ex.down_g[0]
    rt.per_expert_scale = gen.bf16_bits(np.ones(E_T, np.float32))
    y = M.forward(x, ex, rt)
    X = F.bf16_to_f64(x)
    Wg = Q.dequantize(ex.gate_up_q[0][:I_T], ex.gate_up_s[0][:I_T], ex.gate_up_g[0])
    Wu = Q.dequantize(ex.gate_up_q[0][I_T:], ex.gate_up_s[0][I_T:], ex.gate_up_g[0])
    Wd = Q.dequantize(ex.down_q[0], ex.down_s[0], ex.down_g[0])
    g = np.matmul(X, Wg.T)
    u = np.matmul(X, Wu.T)
    hh = TF.gelu(torch.from_numpy(g), approximate="tanh").numpy() * u
    assert np.allclose(y, np.matmul(hh, Wd.T), rtol=1e-12, atol=1e-16)


def test_forward_output_bf16_rounding():
    x, ex, rt = tiny(seed=13, T=4)
    parts = M.forward(x, ex, rt, return_parts=True)
    ref = torch.from_numpy(parts["y64"]).float().to(torch.bfloat16)  # fp64->fp32->bf16 (double rounding)
    diff = parts["y_bf16"].astype(np.int32) - ref.view(torch.int16).numpy().view(np.uint16).astype(np.int32)
    assert np.all(np.abs(diff) <= 1)   # equal except on rare double-rounding cases


def test_ids_override_uses_given_ids():
    x, ex, rt = tiny(seed=14, T=4)
    ids, w, _ = M.route(x, rt)
    swapped = ids[:, ::-1].copy()
    ids2, w2, _ = M.route(x, rt, ids_override=swapped)
    assert np.array_equal(ids2, swapped)
    assert np.allclose(w2, w[:, ::-1], rtol=1e-14)
    y1 = M.forward(x, ex, rt)
    y2 = M.forward(x, ex, rt, ids_override=swapped)
    assert np.allclose(y1, y2, rtol=1e-12, atol=1e-18)


# ------------------------------------------------------------- chain link pin
def _nearest_bf16(v: np.ndarray) -> np.ndarray:
    """The bf16 value nearest to each fp64 value (ties to the even mantissa),
    found among torch's bf16 neighbours: torch rounds through fp32, so its
    result may be one ulp off, and the nearest of it and its two neighbours is
    the correctly rounded value."""
    b = torch.from_numpy(v).float().to(torch.bfloat16)
    cands = torch.stack([torch.nextafter(b, torch.full_like(b, -np.inf)), b,
                         torch.nextafter(b, torch.full_like(b, np.inf))]).double().numpy()
    bits = torch.stack([torch.nextafter(b, torch.full_like(b, -np.inf)), b,
                        torch.nextafter(b, torch.full_like(b, np.inf))]).view(torch.int16).numpy()
    d = np.abs(cands - v[None])
    best = d.min(0)
    tie_ok = (d == best[None]) & ((bits & 1) == 0)
    pick = np.where(tie_ok.any(0), np.argmax(tie_ok, 0), np.argmin(d, 0))
    return np.take_along_axis(cands, pick[None], 0)[0]


def test_residual_rmsnorm_vs_torch_rms_norm():
    rng = np.random.default_rng(21)
    H = 96
    res = rng.standard_normal((6, H)) * np.array([1e-3, 1.0, 1e3, 5.0, 1e-6, 1e5])[:, None]
    y = gen.bf16_bits(rng.standard_normal((6, H)).astype(np.float32) * 0.01)
    res2, xb = M.residual_rmsnorm(res, y, eps=1e-6)
    y_t = torch.from_numpy(y.view(np.int16)).view(torch.bfloat16).double()
    want_res = torch.from_numpy(res) + y_t               # the residual takes y first
    assert np.array_equal(res2, want_res.numpy())
    want_x = TF.rms_norm(want_res, (H,), eps=1e-6).numpy()   # eps inside the square root
    assert np.array_equal(F.bf16_to_f64(xb), _nearest_bf16(want_x))


def test_residual_rmsnorm_constant_row_closed_form():
    c = 0.75
    res = np.full((1, 64), c)
    y = np.zeros((1, 64), np.uint16)                     # +0.0 in bf16
    res2, xb = M.residual_rmsnorm(res, y, eps=0.25)
    assert np.all(res2 == c)
    # x = c / sqrt(c^2 + eps) = 0.75 / sqrt(0.8125) = 0.83205..., nearest bf16 0.83203125
    assert np.all(F.bf16_to_f64(xb) == 0.83203125)


# ---------------------------------------------------------- gated hidden pin
def _brute_force_hidden(x_bits, ex, e):
    """Pure-Python h = gelu_tanh(gate) * up of expert e for each row of x, with
    the weights decoded element by element (E2M1 x E4M3 x global)."""
    T, H = x_bits.shape
    I = ex.I
    e2m1 = [F.e2m1_decode(c).item() for c in range(16)]
    e4m3 = [F.e4m3_decode(c).item() for c in range(256)]

    def wgu(n, kk):
        byte = int(ex.gate_up_q[e][n, kk // 2])
        code = byte & 0xF if kk % 2 == 0 else byte >> 4
        return e2m1[code] * e4m3[int(ex.gate_up_s[e][n, kk // 16])] * float(ex.gate_up_g[e])

    out = []
    for t in range(T):
        xt = [F.bf16_to_f64(x_bits[t, kk]).item() for kk in range(H)]
        gate = [sum(wgu(n, kk) * xt[kk] for kk in range(H)) for n in range(I)]
        up = [sum(wgu(I + n, kk) * xt[kk] for kk in range(H)) for n in range(I)]
        out.append([0.5 * g * (1 + math.tanh(math.sqrt(2 / math.pi) * (g + 0.044715 * g ** 3))) * u
                    for g, u in zip(gate, up)])
    return np.array(out)


@pytest.mark.parametrize("e", [0, 3])
def test_expert_hidden_vs_pure_python(e):
    x, ex, _ = tiny(seed=15, T=3)
    wgu, _ = M.expert_dense(ex, e)
    got = M.expert_hidden(F.bf16_to_f64(x), wgu)
    want = _brute_force_hidden(x, ex, e)
    assert got.shape == (3, I_T)
    assert np.allclose(got, want, rtol=1e-12, atol=1e-14 * np.abs(want).max())
