"""moe_block_forward (the full feed-forward block: dense MLP in parallel with
the NVFP4 sparse branch, five norms, the router on the raw residual,
layer_scalar) on the GPU against the fp64 block oracle."""
import numpy as np
import pytest
import torch

import moe_inputs as gen
import nvfp4_weight_only_router_b200 as lib
from oracle import block as B
from oracle import moe as M
from tests.gpu_common import bf16_from_dev, bf16_to_dev, check_forward, check_ids

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def block0(layer0, dev):
    b = gen.make_block(200)
    return {"b": b, "db": lib.DenseParts.from_host(b, dev)}


def _params(layer0, b):
    return B.BlockParams(layer0["ex"], layer0["rt"], b.dense_gate, b.dense_up, b.dense_down, b.pre_ff_norm,
                         b.post_ff_norm_1, b.pre_ff_norm_2, b.post_ff_norm_2, b.post_ff_norm, b.layer_scalar)


def _run_and_check(layer0, block0, dev, T, rows=None, b=None, db=None):
    b = b if b is not None else block0["b"]
    db = db if db is not None else block0["db"]
    blk = lib.MoeBlock(layer0["dex"], layer0["drt"], db, max_tokens=T)
    x = gen.make_x(500 + T, T)
    y = blk(bf16_to_dev(x, dev))
    torch.cuda.synchronize()
    assert lib.device_status() == 0
    ids = blk.ids(T).cpu().numpy()
    rows = np.arange(T) if rows is None else rows
    # the router reads the raw residual
    ids0, _, logits = M.route(x[rows], layer0["rt"])
    differ = check_ids(ids[rows], ids0, logits)
    override = np.where(differ[:, None], ids[rows], ids0) if differ.any() else None
    out64 = B.forward(x[rows], _params(layer0, b), ids_override=override)
    return check_forward(bf16_from_dev(y)[rows], out64)


@pytest.mark.parametrize("T", [1, 8, 64])
def test_block_decode(layer0, block0, dev, T):
    _run_and_check(layer0, block0, dev, T)


@pytest.mark.parametrize("T", [300, 1024])
def test_block_tensor_core_paths(layer0, block0, dev, T):
    """Above 256 tokens the experts take the tensor-core GEMMs and the dense
    MLP the 256-/128-token tiles without K splits; 24 sampled tokens."""
    rows = np.unique(np.r_[0, T - 1, np.random.default_rng(T).choice(T, 22, replace=False)])
    _run_and_check(layer0, block0, dev, T, rows)


@pytest.mark.parametrize("which", ["dense_only", "sparse_only"])
def test_block_each_branch_alone(layer0, block0, dev, which):
    """One branch silenced through its post-norm weight (post_ff_norm_2 = 0
    leaves the dense branch; post_ff_norm_1 = 0 the sparse one), so an error in
    either branch cannot hide behind the other."""
    b = gen.make_block(200)
    if which == "dense_only":
        b.post_ff_norm_2 = np.zeros_like(b.post_ff_norm_2)
    else:
        b.post_ff_norm_1 = np.zeros_like(b.post_ff_norm_1)
    _run_and_check(layer0, block0, dev, 64, b=b, db=lib.DenseParts.from_host(b, dev))
