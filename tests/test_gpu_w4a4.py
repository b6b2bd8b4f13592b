"""moe_w4a4_forward (NVFP4 activations on the block-scaled FP4 tensor cores)
on the GPU against the W4A4 oracle.

What is unique is compared exactly; where a floating-point sum decides an
integer the comparison allows what that sum may legitimately decide:
  * packed weight codes and scales: bit-exact against the documented layouts;
  * x codes and scales: bit-exact (both sides quantise the same bf16 values
    with the same fp32 steps);
  * hidden codes and scales: the GPU forms h from fp32 tensor-core sums, the
    oracle from fp64 ones, so a block may round differently where h / d lies
    at a rounding threshold to within the sums' difference; such blocks must
    be rare and still a valid rounding of the oracle's h;
  * y against the oracle's down GEMM and combine on the GPU's own hidden
    codes: the forward bar (bf16 output, fp32 against fp64 sums);
  * y end to end against the oracle: the forward bar widened by the few
    hidden blocks that may round the other way.
"""
import numpy as np
import pytest
import torch

import moe_inputs as gen
import nvfp4_weight_only_router_b200 as lib
from oracle import formats as F
from oracle import moe as M
from oracle import w4a4 as W
from tests.gpu_common import bf16_from_dev, bf16_to_dev, check_forward, check_ids, forward_errors

pytestmark = pytest.mark.gpu

H, I, E, K8 = 2816, 704, 128, 8
GX, GH = gen.W4A4_GX, gen.W4A4_GH


@pytest.fixture(scope="module")
def layer(layer0, dev):
    return lib.W4A4Layer(layer0["dex"], layer0["drt"], GX, GH, max_tokens=4096)


def _padded_rows(counts, offsets, nt):
    """Padded row of every sorted position (the documented layout)."""
    tiles = (counts + nt - 1) // nt
    start = np.concatenate([[0], np.cumsum(tiles)[:-1]]) * nt
    rows = np.empty(int(offsets[-1]), np.int64)
    for e in range(E):
        rows[offsets[e]:offsets[e + 1]] = start[e] + np.arange(counts[e])
    return rows


def _swizzled_rows(buf, rows, nt, nchunk, nbytes):
    """Rows [len(rows), nbytes] of codes stored tile-major in 128-byte swizzled
    blocks (tile p, chunk c: nt rows of 128 bytes; byte k of row r at
    128 r + 16 ((k / 16) ^ (r % 8)) + k % 16)."""
    k = np.arange(nchunk * 128)
    c, kk = k // 128, k % 128
    tile, r = rows // nt, rows % nt
    idx = ((tile[:, None] * nchunk + c[None, :]) * nt + r[:, None]) * 128 \
        + 16 * ((kk[None, :] // 16) ^ (r[:, None] % 8)) + kk[None, :] % 16
    return buf[idx][:, :nbytes]


def _chunk_scales(chunks, rows, nt, K):
    """Scales [len(rows), K/16] of the given padded rows from the 512-byte chunks."""
    g = K // 64
    tile, r = rows // nt, rows % nt
    b = np.arange(K // 16)
    idx = (tile[:, None] * g + b[None, :] // 4) * 512 + 16 * (r[:, None] % 32) + 4 * (r[:, None] // 32) + b[None, :] % 4
    return chunks[idx]


def test_pack_layout(layer, layer0):
    """Codes: block (e, j, c) holds tile rows L of K bytes 128 c.. in the
    128-byte swizzle; scales: chunk (e, j, q) byte 16 r0 + 4 r1 + i = scale of
    tile row r0 + 32 r1, block 4 q + i; gate_up tile rows interleave the gate
    and up rows of 16 hidden units per lane quarter."""
    ex = layer0["ex"]
    Lq = np.arange(128)
    qd, w = Lq >> 5, Lq & 31
    gu_pk = layer.experts.gate_up_pk.cpu().numpy().reshape(E, 11, 11 * 128 * 128)
    dn_pk = layer.experts.down_pk.cpu().numpy().reshape(E, 22, 3 * 128 * 128)
    gu = layer.gate_up_sf.cpu().numpy().reshape(E, 11, 44, 32, 4, 4)   # e, j, q, r0, r1, i
    dn = layer.down_sf.cpu().numpy().reshape(E, 22, 11, 32, 4, 4)
    L = np.arange(128).reshape(4, 32).T           # [r0, r1] -> tile row
    for e in (0, 77, 127):
        for j in (0, 5, 10):
            grow = np.where(w < 16, 0, I) + j * 64 + qd * 16 + (w & 15)
            assert np.array_equal(_swizzled_rows(gu_pk[e, j], Lq, 128, 11, H // 2), ex.gate_up_q[e][grow])
            grow2 = grow[L]
            want = ex.gate_up_s[e][grow2].reshape(32, 4, 44, 4).transpose(2, 0, 1, 3)
            assert np.array_equal(gu[e, j], want)
        for j in (0, 13, 21):
            got = _swizzled_rows(dn_pk[e, j], Lq, 128, 3, 384)
            assert np.array_equal(got[:, :I // 2], ex.down_q[e][j * 128 + Lq])
            assert not got[:, I // 2:].any()
            want = ex.down_s[e][j * 128 + L].reshape(32, 4, 11, 4).transpose(2, 0, 1, 3)
            assert np.array_equal(dn[e, j], want)


def _run(layer, dev, x):
    T = x.shape[0]
    y = layer(bf16_to_dev(x, dev))
    torch.cuda.synchronize()
    assert lib.device_status() == 0
    v = {k: (t.cpu().numpy() if isinstance(t, torch.Tensor) else t) for k, t in layer.views(T).items()}
    return bf16_from_dev(y), v


def _check_valid_rounding(codes, scales, h):
    """Blocks [n, 16] whose codes and scale the GPU chose differently from the
    oracle: each must be the method's rounding of some h' within the fp32
    sums' error of the oracle's h (relative 1e-5 of the element plus 1e-6 of
    the block maximum).  Both roundings are monotone, so the GPU's scale must
    lie between those of the block maxima at the ends of that range, and each
    code, under the GPU's scale, between the codes of the element's ends."""
    tol = 1e-5 * np.abs(h) + 1e-6 * np.abs(h).max(axis=1, keepdims=True)
    amax = np.abs(h).max(axis=1)
    tmax = tol.max(axis=1)
    f32 = np.float32
    s_lo = F.e4m3_encode_satfinite(((f32(np.maximum(amax - tmax, 0)) / f32(6)) / GH).astype(np.float64))
    s_hi = F.e4m3_encode_satfinite(((f32(amax + tmax) / f32(6)) / GH).astype(np.float64))
    assert np.all((s_lo <= scales) & (scales <= s_hi)), "hidden block scale outside its rounding range"
    d = (F.e4m3_decode(scales).astype(f32) * GH).astype(f32)[:, None]
    v_lo = F.e2m1_decode(F.e2m1_encode((h - tol).astype(f32) / d))
    v_hi = F.e2m1_decode(F.e2m1_encode((h + tol).astype(f32) / d))
    v = F.e2m1_decode(codes)
    assert np.all((v_lo <= v) & (v <= v_hi)), "hidden code outside its rounding range"


def _check_heavy_tailed(y_bits, y64, rel_bar, abs_bar):
    yg = F.bf16_to_f64(y_bits)
    assert np.all(np.isfinite(yg))
    rel = np.linalg.norm(yg - y64) / np.linalg.norm(y64)
    assert rel <= rel_bar, rel
    rms = np.sqrt(np.mean(y64 ** 2))
    excess = np.abs(yg - y64) - (abs_bar * rms + 2.0 ** -8 * np.abs(y64))
    assert excess.max() <= 0, excess.max()


def _saturating_x(T, seed):
    """x with some 16-element blocks scaled by 40 (|x| up to ~200): their block
    scale saturates at 448 under Gx (whose range is 8) and their largest codes
    at 6, the method's satfinite behaviour."""
    x = F.bf16_to_f32(gen.make_x(seed, T)).copy()
    rng = np.random.default_rng(seed)
    for t in range(T):
        for b in rng.choice(H // 16, 6, replace=False):
            x[t, 16 * b:16 * b + 16] *= 40.0
    return gen.bf16_bits(x)


@pytest.mark.parametrize("T,kind", [(1, "n"), (8, "n"), (64, "n"), (256, "n"), (257, "n"), (300, "n"), (1025, "n"),
                                    (2048, "n"), (16, "sat")])
def test_w4a4_forward(layer, layer0, dev, T, kind):
    """T <= 256: 16-token tiles; 257..1024: 64; above: 128 (the oracle on 12
    sampled tokens above 64); "sat": blocks whose scale saturates."""
    ex, rt = layer0["ex"], layer0["rt"]
    x = gen.make_x(900 + T, T) if kind == "n" else _saturating_x(T, 990)
    y, v = _run(layer, dev, x)
    nt = v["tile_tokens"]
    rows_of_pos = _padded_rows(v["counts"].astype(np.int64), v["offsets"].astype(np.int64), nt)
    toks = np.arange(T) if T <= 64 else np.unique(np.r_[0, T - 1, np.random.default_rng(T).choice(T, 10, replace=False)])
    ids0, _, logits = M.route(x[toks], rt)
    differ = check_ids(v["ids"][toks], ids0, logits)
    override = np.where(differ[:, None], v["ids"][toks], ids0) if differ.any() else None
    ref = W.forward(x[toks], ex, rt, GX, GH, ids_override=override, return_parts=True)

    # x codes and scales: every slot of a sampled token holds its token's quantised row
    slots = (toks[:, None] * K8 + np.arange(K8)[None, :]).ravel()
    prow = rows_of_pos[v["slot_pos"][slots]]
    xq = np.repeat(ref["xq"], K8, axis=0)
    xs = np.repeat(ref["xs"], K8, axis=0)
    assert np.array_equal(_swizzled_rows(v["x_codes"], prow, nt, 11, H // 2), xq)
    assert np.array_equal(_chunk_scales(v["x_scales"], prow, nt, H), xs)

    # hidden codes: rare, valid threshold decisions only
    hq_gpu = _swizzled_rows(v["h_codes"], prow, nt, 3, I // 2)
    hs_gpu = _chunk_scales(v["h_scales"], prow, nt, I)
    local = (np.arange(len(toks))[:, None] * K8 + np.arange(K8)[None, :]).ravel()
    hq_ref, hs_ref, h32 = ref["hq"][local], ref["hs"][local], ref["h32"][local]
    codes_gpu, codes_ref = F.unpack_nibbles(hq_gpu), F.unpack_nibbles(hq_ref)
    bad = (codes_gpu != codes_ref).reshape(len(local), I // 16, 16).any(-1) | (hs_gpu != hs_ref)
    assert bad.mean() < 2e-3, f"{bad.mean():.2e} of hidden blocks differ"
    if bad.any():
        _check_valid_rounding(codes_gpu.reshape(len(local), I // 16, 16)[bad], hs_gpu[bad],
                              h32.astype(np.float64).reshape(len(local), I // 16, 16)[bad])

    # y from the GPU's own hidden codes: the forward bar; with saturating inputs
    # y has outliers whose bf16 rounding alone (half an ulp, up to 2^-8 |y|)
    # exceeds 2e-2 rms(y), so there the max-abs bar is taken per element with
    # that rounding added
    y_own = W.down_from_codes(hq_gpu, hs_gpu, GH, ref["ids"], ref["w"], ex, len(toks))
    if kind == "sat":
        _check_heavy_tailed(y[toks], y_own, 2e-3, 2e-2)
        _check_heavy_tailed(y[toks], ref["y64"], 4e-3, 4e-2)
        return
    check_forward(y[toks], y_own)
    # end to end
    rel, mx = forward_errors(y[toks], ref["y64"])
    assert rel <= 4e-3 and mx <= 4e-2, (rel, mx)


def test_w4a4_hidden_padding_rows_are_zero(layer, dev):
    T = 24
    x = gen.make_x(950, T)
    _, v = _run(layer, dev, x)
    nt = v["tile_tokens"]
    counts = v["counts"].astype(np.int64)
    rows = _padded_rows(counts, v["offsets"].astype(np.int64), nt)
    total = int(((counts + nt - 1) // nt).sum()) * nt
    pad = np.setdiff1d(np.arange(total), rows)
    assert pad.size > 0
    assert not _swizzled_rows(v["h_codes"], pad, nt, 3, I // 2).any()
    assert not _chunk_scales(v["h_scales"], pad, nt, I).any()


def test_w4a4_repeat_is_deterministic(layer, dev):
    x = bf16_to_dev(gen.make_x(960, 512), dev)
    y1 = layer(x)
    y2 = layer(x)
    torch.cuda.synchronize()
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))
