"""moe_nvfp4_forward on the GPU against the fp64 oracle: the routing
intermediates (ids, weights, permutation) and the gated hidden h per step,
and the output y, on the layer shapes of the decode and prefill workloads,
activations across the bf16 range, and the chained layer stack."""
import numpy as np
import pytest
import torch

import moe_inputs as gen
import nvfp4_weight_only_router_b200 as lib
from oracle import formats as F
from oracle import moe as M
from tests.gpu_common import (bf16_from_dev, bf16_to_dev, check_forward, check_ids,
                              check_weights)

pytestmark = pytest.mark.gpu


def _oracle_y(x, ex, rt, ids_gpu, differ):
    """Oracle output; tokens whose ids legitimately differ use the GPU's ids."""
    override = None
    if differ.any():
        ids0, _, _ = M.route(x, rt)
        override = np.where(differ[:, None], ids_gpu, ids0)
    return M.forward(x, ex, rt, ids_override=override)


def _run(layer, x, dev):
    y = layer(bf16_to_dev(x, dev))
    torch.cuda.synchronize()
    assert lib.device_status() == 0
    return y


def _check_permutation(v, ids):
    """The forward's permutation, bit-exact against the oracle's stable
    grouping of the GPU ids."""
    counts, offsets, sorted_slot, slot_pos = M.permute(ids, 128)
    assert np.array_equal(v["counts"].cpu().numpy(), counts)
    assert np.array_equal(v["offsets"].cpu().numpy(), offsets)
    assert np.array_equal(v["sorted_slot"].cpu().numpy(), sorted_slot)
    assert np.array_equal(v["slot_pos"].cpu().numpy(), slot_pos)
    return counts, offsets, sorted_slot


def _check_hidden(v, x, ex, experts, counts, offsets, sorted_slot, max_rows=None):
    """The gated hidden h of the given experts (rows in sorted order, at their
    true scale) against the oracle's fp64 h: relative L2 < 1e-3 per expert
    (the f16 rounding of h costs ~2^-11 / sqrt(3))."""
    h = lib.unscaled_hidden(v).cpu().numpy()
    X = F.bf16_to_f64(x)
    for e in experts:
        lo, hi = offsets[e], offsets[e + 1]
        if max_rows is not None:
            hi = min(hi, lo + max_rows)
        assert hi > lo, e
        wgu, _ = M.expert_dense(ex, e)
        h_ref = M.expert_hidden(X[sorted_slot[lo:hi] // 8], wgu)
        rel = np.linalg.norm(h[lo:hi] - h_ref) / np.linalg.norm(h_ref)
        assert rel < 1e-3, (e, rel)


@pytest.mark.parametrize("T", [1, 3, 8, 17, 64])
def test_forward_decode_shapes(layer0, dev, T):
    ex, rt = layer0["ex"], layer0["rt"]
    layer = lib.MoeLayer(layer0["dex"], layer0["drt"], max_tokens=T)
    x = gen.make_x(1000 + T, T)
    y = _run(layer, x, dev)
    v = layer.views(T)
    ids, w = v["ids"].cpu().numpy(), v["weights"].cpu().numpy()
    ids0, w0, logits = M.route(x, rt)
    differ = check_ids(ids, ids0, logits)
    check_weights(w, w0, differ)
    counts, offsets, sorted_slot = _check_permutation(v, ids)
    _check_hidden(v, x, ex, np.flatnonzero(counts), counts, offsets, sorted_slot)
    # output
    y64 = _oracle_y(x, ex, rt, ids, differ)
    check_forward(bf16_from_dev(y), y64)


@pytest.fixture(scope="module")
def packed_experts(layer0):
    return layer0["dex"].packed()


@pytest.mark.parametrize("T", [1, 8, 64, 256, 300])
def test_forward_packed_codes(layer0, packed_experts, dev, T):
    """With the packed code tiles the decode GEMVs (T <= 256) stream whole
    16 KB blocks; the arithmetic is unchanged, so y is bit-identical to the
    forward on the plain codes (T = 300 takes the tensor-core GEMMs, which read
    the plain codes either way); on few tokens also against the oracle."""
    ex, rt = layer0["ex"], layer0["rt"]
    plain = lib.MoeLayer(layer0["dex"], layer0["drt"], max_tokens=T)
    packed = lib.MoeLayer(packed_experts, layer0["drt"], max_tokens=T)
    x = gen.make_x(1100 + T, T)
    y1 = _run(plain, x, dev)
    y2 = _run(packed, x, dev)
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))
    if T <= 8:
        ids = packed.views(T)["ids"].cpu().numpy()
        ids0, _, logits = M.route(x, rt)
        differ = check_ids(ids, ids0, logits)
        check_forward(bf16_from_dev(y2), _oracle_y(x, ex, rt, ids, differ))


def test_forward_repeat_is_deterministic(layer0, dev):
    layer = lib.MoeLayer(layer0["dex"], layer0["drt"], max_tokens=64)
    xd = bf16_to_dev(gen.make_x(77, 64), dev)
    y1 = layer(xd).clone()
    y2 = layer(xd)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)


@pytest.mark.parametrize("T", [257, 300])
def test_forward_tensor_core_path(layer0, dev, T):
    """Above 256 tokens the expert GEMMs run on tcgen05 (64-token tiles) and
    the permutation takes the multi-chunk kernels."""
    ex, rt = layer0["ex"], layer0["rt"]
    layer = lib.MoeLayer(layer0["dex"], layer0["drt"], max_tokens=T)
    x = gen.make_x(2000 + T, T)
    y = _run(layer, x, dev)
    v = layer.views(T)
    ids = v["ids"].cpu().numpy()
    ids0, _, logits = M.route(x, rt)
    differ = check_ids(ids, ids0, logits)
    counts, offsets, sorted_slot = _check_permutation(v, ids)
    order = np.argsort(counts)
    hot, cold = order[-2:], [e for e in order if counts[e] > 0][:2]
    _check_hidden(v, x, ex, list(hot) + list(cold), counts, offsets, sorted_slot)
    sample = np.unique(np.r_[0, T - 1, np.random.default_rng(T).choice(T, 24, replace=False)])
    y64 = _oracle_y(x[sample], ex, rt, ids[sample], differ[sample])
    check_forward(bf16_from_dev(y)[sample], y64)


def test_forward_prefill_zipf_sampled(layer0, dev):
    """The prefill workload: T=4096 with the Zipf-skewed router bias; all
    tokens' ids checked, the output on a sample of 40 tokens."""
    ex = layer0["ex"]
    rt = gen.make_router(1, bias=gen.zipf_bias(7))
    layer = lib.MoeLayer(layer0["dex"], lib.Router.from_host(rt, dev), max_tokens=4096)
    x = gen.make_x(2, 4096)
    y = _run(layer, x, dev)
    v = layer.views(4096)
    ids = v["ids"].cpu().numpy()
    ids0, w0, logits = M.route(x, rt)
    differ = check_ids(ids, ids0, logits)
    counts, offsets, sorted_slot = _check_permutation(v, ids)
    assert counts.max() > 1000 and (counts < 20).sum() > 5   # the skew the workload asks for
    # h of the two hottest experts (first 256 rows: several 192-token tiles)
    # and of two cold ones (a single ragged tile)
    order = np.argsort(counts)
    cold = [e for e in order if counts[e] > 0][:2]
    _check_hidden(v, x, ex, list(order[-2:]) + cold, counts, offsets, sorted_slot, max_rows=256)
    sample = np.unique(np.r_[0, 4095, np.random.default_rng(3).choice(4096, 38, replace=False)])
    y64 = _oracle_y(x[sample], ex, rt, ids[sample], differ[sample])
    check_forward(bf16_from_dev(y)[sample], y64)


def test_residual_rmsnorm_chain_step(dev):
    rng = np.random.default_rng(5)
    res = rng.standard_normal((8, 2816)).astype(np.float32)
    y = gen.bf16_bits(rng.standard_normal((8, 2816)).astype(np.float32) * 0.01)
    rd = torch.from_numpy(res).to(dev)
    xo = torch.empty((8, 2816), dtype=torch.bfloat16, device=dev)
    lib.residual_rmsnorm(rd, bf16_to_dev(y, dev), xo)
    torch.cuda.synchronize()
    res2, x_ref = M.residual_rmsnorm(res.astype(np.float64), y)
    assert np.allclose(rd.cpu().numpy(), res2, rtol=0, atol=1e-6)
    got = F.bf16_to_f64(bf16_from_dev(xo))
    # fp32 vs fp64 normalisation may flip a bf16 rounding: at most one ulp
    assert np.all(np.abs(got - F.bf16_to_f64(x_ref)) <= np.abs(F.bf16_to_f64(x_ref)) * 2 ** -7 + 1e-30)


# ------------------------------------------------------ activation range
def _check_rows(y_bits, y64):
    """The forward bar applied to every token row on its own (rows of very
    different magnitude must each meet it)."""
    for t in range(y64.shape[0]):
        check_forward(y_bits[t:t + 1], y64[t:t + 1])


def _range_x(T, seed):
    """Rows of N(0,1) activations scaled by 10^k for k from -6 to 6, plus rows
    that mix magnitudes (one element 10^6 among ordinary ones; one element
    10^-6 among ordinary ones)."""
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((T, 2816)).astype(np.float64)
    for t in range(T):
        x[t] *= 10.0 ** ((t % 13) - 6)
    x[1, 7] = 1e6
    x[2, 100:] = 1e-6 * np.sign(x[2, 100:])
    return gen.bf16_bits(x.astype(np.float32))


@pytest.mark.parametrize("T", [13, 300])
def test_forward_activation_range(layer0, dev, T):
    """bf16 activations from 1e-6 to 1e6 go through the f16 operands of both
    expert paths (streaming GEMV at T=13, tensor cores at T=300) under the
    exact per-token power-of-two prescale: every row meets the forward bar,
    and no range error is recorded."""
    ex, rt = layer0["ex"], layer0["rt"]
    layer = lib.MoeLayer(layer0["dex"], layer0["drt"], max_tokens=T)
    x = _range_x(T, 31 + T)
    y = _run(layer, x, dev)
    v = layer.views(T)
    ids = v["ids"].cpu().numpy()
    ids0, _, logits = M.route(x, rt)
    differ = check_ids(ids, ids0, logits)
    rows = np.arange(T) if T <= 16 else np.r_[0:16, T - 3:T]
    y64 = _oracle_y(x[rows], ex, rt, ids[rows], differ[rows])
    _check_rows(bf16_from_dev(y)[rows], y64)


def _scaled_gate_up(layer0, dev, factor):
    ex = layer0["ex"]
    ex2 = gen.Experts(ex.gate_up_q, ex.gate_up_s, (ex.gate_up_g * np.float32(factor)).astype(np.float32),
                      ex.down_q, ex.down_s, ex.down_g)
    dex = layer0["dex"]
    dex2 = lib.Experts(dex.gate_up_q, dex.gate_up_s, torch.from_numpy(ex2.gate_up_g).to(dev),
                       dex.down_q, dex.down_s, dex.down_g)
    return ex2, dex2


@pytest.mark.parametrize("T", [8, 300])
def test_forward_large_hidden_in_range(layer0, dev, T):
    """Experts whose gate_up gain is 300x the generated one (|h| up to ~6e3
    for activations of unit maximum, far beyond the raw f16 range for
    activations of size 10^3): still within the prescaled f16 range, so every
    row meets the forward bar."""
    ex2, dex2 = _scaled_gate_up(layer0, dev, 300.0)
    rt = layer0["rt"]
    layer = lib.MoeLayer(dex2, layer0["drt"], max_tokens=T)
    x = gen.bf16_bits(F.bf16_to_f64(gen.make_x(41 + T, T)) * 1000.0)
    y = _run(layer, x, dev)
    ids = layer.views(T)["ids"].cpu().numpy()
    ids0, _, logits = M.route(x, rt)
    differ = check_ids(ids, ids0, logits)
    rows = np.arange(min(T, 12))
    y64 = _oracle_y(x[rows], ex2, rt, ids[rows], differ[rows])
    _check_rows(bf16_from_dev(y)[rows], y64)


@pytest.mark.parametrize("T", [8, 300])
def test_forward_hidden_overflow_is_reported(layer0, dev, T):
    """Gate_up gains of 3000x push the prescaled h past the f16 range: the
    call saturates and records NVFP4_ERR_RANGE (no silent result)."""
    _, dex2 = _scaled_gate_up(layer0, dev, 3000.0)
    layer = lib.MoeLayer(dex2, layer0["drt"], max_tokens=T)
    layer(bf16_to_dev(gen.make_x(51 + T, T), dev))
    torch.cuda.synchronize()
    assert lib.device_status() == lib.capi.NVFP4_ERR_RANGE
    assert lib.device_status() == 0   # read and cleared


# ------------------------------------------------------ chained layer stack
def test_stack_chained_layers(dev):
    """The stack workload's chain x_{l+1} = x_l + moe_l(rmsnorm(x_l)) (fp32
    residual, bf16 layer inputs) over three independently seeded layers at
    T = 8: each layer's y against the oracle on that layer's input, each link
    against the oracle link, and the chain end to end against an oracle chain
    run from the same tokens (residual increments within the forward bar)."""
    T, L = 8, 3
    seeds = gen.layer_seed_plan(L)
    x0 = gen.make_x(61, T)
    res = torch.from_numpy(F.bf16_to_f64(x0).astype(np.float32)).to(dev)
    xn = torch.empty((T, 2816), dtype=torch.bfloat16, device=dev)
    lib.residual_rmsnorm(res, None, xn)
    res_o = F.bf16_to_f64(x0)
    _, x_o = M.residual_rmsnorm(res_o, np.zeros_like(x0))
    for sd in seeds:
        ex, rt = gen.make_experts(sd), gen.make_router(1000 + sd)
        layer = lib.MoeLayer(lib.Experts.from_host(ex, dev), lib.Router.from_host(rt, dev), max_tokens=T)
        x_l = bf16_from_dev(xn)
        res_l = res.double().cpu().numpy()
        y = layer(xn)
        torch.cuda.synchronize()
        assert lib.device_status() == 0
        ids = layer.views(T)["ids"].cpu().numpy()
        ids0, _, logits = M.route(x_l, rt)
        differ = check_ids(ids, ids0, logits)
        y_bits = bf16_from_dev(y)
        check_forward(y_bits, _oracle_y(x_l, ex, rt, ids, differ))
        lib.residual_rmsnorm(res, y, xn)
        torch.cuda.synchronize()
        res_ref, x_ref = M.residual_rmsnorm(res_l, y_bits)
        assert np.allclose(res.double().cpu().numpy(), res_ref, rtol=2 ** -23, atol=0)
        got = F.bf16_to_f64(bf16_from_dev(xn))
        assert np.all(np.abs(got - F.bf16_to_f64(x_ref)) <= np.abs(F.bf16_to_f64(x_ref)) * 2 ** -7)
        # the oracle's own chain; its inputs differ from the GPU chain's by bf16
        # rounding flips, so where the selections differ at a near-tie of the
        # oracle chain's logits (< 1e-4) it takes the GPU's ids
        ids_o, _, logits_o = M.route(x_o, rt)
        take = np.zeros(T, bool)
        for t in np.flatnonzero(np.any(ids != ids_o, axis=1)):
            j = ids[t] != ids_o[t]
            take[t] = np.all(np.abs(logits_o[t, ids[t][j]] - logits_o[t, ids_o[t][j]]) < 1e-4)
        y_o = M.forward(x_o, ex, rt, ids_override=np.where(take[:, None], ids, ids_o))
        res_o, x_o = M.residual_rmsnorm(res_o, F.f64_to_bf16_rne(y_o))
        del layer
    d_gpu = res.double().cpu().numpy() - F.bf16_to_f64(x0)
    d_o = res_o - F.bf16_to_f64(x0)
    assert np.linalg.norm(d_gpu - d_o) / np.linalg.norm(d_o) <= 2e-3


# ------------------------------------------------------ dense over-read
@pytest.mark.parametrize("T", [1, 8, 33])
def test_forward_dense_over_read(layer0, dev, T):
    """The dense over-read (every token through all 128 experts, weighted by
    its routing weights, 0 for unselected experts) computes the same branch:
    its y meets the forward bar against the oracle, like the routed forward's."""
    ex, rt = layer0["ex"], layer0["rt"]
    layer = lib.MoeLayer(layer0["dex"], layer0["drt"], max_tokens=T)
    x = gen.make_x(71 + T, T)
    xd = bf16_to_dev(x, dev)
    y_sparse = layer(xd)
    ids = layer.views(T)["ids"].cpu().numpy()
    y_dense = layer.forward_dense_into(xd, torch.empty_like(xd))
    torch.cuda.synchronize()
    assert lib.device_status() == 0
    ids0, _, logits = M.route(x, rt)
    differ = check_ids(ids, ids0, logits)
    y64 = _oracle_y(x, ex, rt, ids, differ)
    check_forward(bf16_from_dev(y_dense), y64)
    check_forward(bf16_from_dev(y_sparse), y64)
