"""moe_permute on the GPU against the oracle's stable grouping by expert,
bit-exact, from a single slot to the largest token count (many 1024-slot
chunks, experts spanning chunks), and the out-of-range id check."""
import numpy as np
import pytest
import torch

import nvfp4_weight_only_router_b200 as lib
from oracle import moe as M

pytestmark = pytest.mark.gpu


def _ids(T, seed, zipf=False):
    """8 distinct experts per token: uniformly, or with Zipf-skewed expert
    popularity (hot experts get thousands of slots)."""
    rng = np.random.default_rng(seed)
    key = rng.random((T, 128))
    if zipf:
        key = key ** (1.0 / (np.arange(1, 129) ** -1.1 * 50.0))
    return np.argsort(-key, axis=1)[:, :8].astype(np.int32)


def _permute(ids, dev):
    out = lib.permute(torch.from_numpy(ids).to(dev))
    torch.cuda.synchronize()
    return [o.cpu().numpy() for o in out]


@pytest.mark.parametrize("T,zipf", [(1, False), (5, False), (128, False), (129, True), (257, False),
                                    (4096, True), (9000, False), (65536, True)])
def test_permute_exact(dev, T, zipf):
    ids = _ids(T, T, zipf)
    got = _permute(ids, dev)
    assert lib.device_status() == 0
    want = M.permute(ids, 128)
    for g, w, name in zip(got, want, ("counts", "offsets", "sorted_slot", "slot_pos")):
        assert np.array_equal(g, w), name
    if zipf and T >= 4096:
        assert want[0].max() > 1024   # an expert whose slots span several chunks


def test_permute_out_of_range_id_is_reported(dev):
    """Ids outside [0, 128) record NVFP4_ERR_DEVICE; those slots are left out
    (slot_pos -1, not counted) and the valid slots are grouped exactly as the
    oracle groups the valid slots alone."""
    T = 3000
    ids = _ids(T, 7)
    ids[5, 2] = 200
    ids[2999, 7] = -1
    ids[1500, 0] = 128
    counts, offsets, sorted_slot, slot_pos = _permute(ids, dev)
    assert lib.device_status() == lib.capi.NVFP4_ERR_DEVICE
    flat = ids.ravel()
    valid = (flat >= 0) & (flat < 128)
    c0, o0, s0, _ = M.permute(flat[valid].reshape(-1, 1), 128)
    idx = np.flatnonzero(valid)
    assert np.array_equal(counts, c0) and np.array_equal(offsets, o0)
    assert np.array_equal(sorted_slot[:o0[-1]], idx[s0])
    assert np.all(slot_pos[~valid] == -1)
    assert np.array_equal(sorted_slot[slot_pos[valid]], idx)
