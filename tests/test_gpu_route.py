"""moe_route on the GPU against the oracle router (fp64)."""
import numpy as np
import pytest
import torch

import moe_inputs as gen
import nvfp4_weight_only_router_b200 as lib
from oracle import moe as M
from tests.gpu_common import bf16_to_dev, check_ids, check_weights

pytestmark = pytest.mark.gpu


def _check(x, rt, drt, dev):
    ids, w = lib.route(bf16_to_dev(x, dev), drt)
    torch.cuda.synchronize()
    ids, w = ids.cpu().numpy(), w.cpu().numpy()
    ids0, w0, logits = M.route(x, rt)
    differ = check_ids(ids, ids0, logits)
    check_weights(w, w0, differ)
    return differ


@pytest.mark.parametrize("T", [1, 5, 16, 17, 64, 257, 300])
def test_route_layer_router(layer0, dev, T):
    x = gen.make_x(100 + T, T)
    _check(x, layer0["rt"], layer0["drt"], dev)


def test_route_prefill_zipf_bias(dev):
    rt = gen.make_router(1, bias=gen.zipf_bias(7))
    drt = lib.Router.from_host(rt, dev)
    x = gen.make_x(2, 4096)
    differ = _check(x, rt, drt, dev)
    assert differ.mean() < 1e-3


def test_route_unsupported_hidden_size(dev):
    # hidden sizes that are not 8 to 16 slices of 256 are refused up front
    rt = gen.make_router(5, h=640)
    drt = lib.Router.from_host(rt, dev)
    with pytest.raises(lib.NVFP4Error) as e:
        lib.route(bf16_to_dev(gen.make_x(6, 3, 640), dev), drt)
    assert e.value.status == lib.capi.NVFP4_ERR_UNSUPPORTED


@pytest.mark.parametrize("T", [1, 5, 64, 256])
def test_route_cluster_with_logit_bias(dev, T):
    """A logit bias through the few-token cluster kernel: a random bias (the
    Zipf bias of the prefill workload is checked at T = 4096 and at T = 64)."""
    bias = np.random.default_rng(T).normal(0, 0.05, 128).astype(np.float32) if T != 64 else gen.zipf_bias(7)
    rt = gen.make_router(1, bias=bias)
    drt = lib.Router.from_host(rt, dev)
    _check(gen.make_x(300 + T, T), rt, drt, dev)


def test_route_ties_pick_lower_id(dev):
    # identical router rows -> identical logits; top-8 must be the lowest ids
    rt = gen.make_router(8)
    rt.proj[:] = rt.proj[0]
    drt = lib.Router.from_host(rt, dev)
    x = gen.make_x(9, 4)
    ids, _ = lib.route(bf16_to_dev(x, dev), drt)
    assert (ids.cpu().numpy() == np.arange(8)[None, :]).all()


@pytest.mark.parametrize("h,T", [(2048, 3), (2048, 40), (4096, 17), (2048, 300), (4096, 600), (3072, 257)])
def test_route_hidden_sizes_all_paths(dev, h, T):
    # clusters of 8, 12 and 16 CTAs (h = 2048, 3072, 4096; T <= 256) and the
    # wide kernel (T > 256) at other hidden sizes than the layer's
    rt = gen.make_router(20 + h, h=h)
    drt = lib.Router.from_host(rt, dev)
    x = gen.make_x(21 + T, T, h)
    _check(x, rt, drt, dev)
