"""moe_aff4_forward (the routed branch with experts in the aff4 codec: u4
codes, fp16 scale and bias per (row, K-block of 32)) on the GPU against the
fp64 oracle, on both expert paths."""
import numpy as np
import pytest
import torch

import moe_inputs as gen
import nvfp4_weight_only_router_b200 as lib
from oracle import aff4 as A
from oracle import moe as M
from tests.gpu_common import bf16_from_dev, bf16_to_dev, check_forward, check_ids

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def aff4_layer(layer0, dev):
    arrays = gen.make_aff4_experts(9)
    return {"ex": A.Aff4Experts(*arrays), "dex": lib.Aff4Experts.from_host(arrays, dev)}


@pytest.mark.parametrize("T", [1, 8, 64, 300])
def test_aff4_forward(layer0, aff4_layer, dev, T):
    """T <= 256: the streaming GEMV with the aff4 dequantisation in registers;
    T = 300: the tensor-core GEMMs with it in the dequant warps (24 sampled
    tokens)."""
    rt = layer0["rt"]
    layer = lib.Aff4Layer(aff4_layer["dex"], layer0["drt"], max_tokens=T)
    x = gen.make_x(800 + T, T)
    y = layer(bf16_to_dev(x, dev))
    torch.cuda.synchronize()
    assert lib.device_status() == 0
    ids = layer.ids(T).cpu().numpy()
    rows = np.arange(T) if T <= 64 else np.unique(np.r_[0, T - 1, np.random.default_rng(T).choice(T, 22, replace=False)])
    ids0, _, logits = M.route(x[rows], rt)
    differ = check_ids(ids[rows], ids0, logits)
    override = np.where(differ[:, None], ids[rows], ids0) if differ.any() else None
    y64 = M.forward(x[rows], aff4_layer["ex"], rt, ids_override=override)
    check_forward(bf16_from_dev(y)[rows], y64)
