"""moe_nvfp4_forward on the GPU against the fp64 oracle: the routing
intermediates (ids, weights, permutation) and the gated hidden h per step,
and the output y, on the layer shapes of the decode and prefill workloads."""
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
    # permutation: exact against the oracle's stable grouping of the GPU ids
    counts, offsets, sorted_slot, slot_pos = M.permute(ids, 128)
    assert np.array_equal(v["counts"].cpu().numpy(), counts)
    assert np.array_equal(v["offsets"].cpu().numpy(), offsets)
    assert np.array_equal(v["sorted_slot"].cpu().numpy(), sorted_slot)
    assert np.array_equal(v["slot_pos"].cpu().numpy(), slot_pos)
    # gated hidden h (f16, sorted rows) against the oracle's fp64 h
    h = v["h"].float().cpu().numpy().astype(np.float64)
    X = F.bf16_to_f64(x)
    h_ref = np.empty_like(h)
    for e in np.flatnonzero(counts):
        rows = sorted_slot[offsets[e]:offsets[e + 1]]
        wgu, _ = M.expert_dense(ex, e)
        h_ref[offsets[e]:offsets[e + 1]] = M.expert_hidden(X[rows // 8], wgu)
    rel_h = np.linalg.norm(h - h_ref) / np.linalg.norm(h_ref)
    assert rel_h < 1e-3, rel_h
    # output
    y64 = _oracle_y(x, ex, rt, ids, differ)
    check_forward(bf16_from_dev(y), y64)


def test_forward_repeat_is_deterministic(layer0, dev):
    layer = lib.MoeLayer(layer0["dex"], layer0["drt"], max_tokens=64)
    xd = bf16_to_dev(gen.make_x(77, 64), dev)
    y1 = layer(xd).clone()
    y2 = layer(xd)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)


@pytest.mark.parametrize("T", [257, 300])
def test_forward_atomic_combine_path(layer0, dev, T):
    ex, rt = layer0["ex"], layer0["rt"]
    layer = lib.MoeLayer(layer0["dex"], layer0["drt"], max_tokens=T)
    x = gen.make_x(2000 + T, T)
    y = _run(layer, x, dev)
    v = layer.views(T)
    ids = v["ids"].cpu().numpy()
    ids0, _, logits = M.route(x, rt)
    differ = check_ids(ids, ids0, logits)
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
    counts = v["counts"].cpu().numpy()
    assert counts.max() > 1000 and (counts < 20).sum() > 5   # the skew the workload asks for
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
