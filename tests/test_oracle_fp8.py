"""Pins for the oracle's fp8 (e4m3) payload (CPU only).

The e4m3 codec is checked against torch's float8_e4m3fn (a library routine)
on every code and on in-range values, and against the OCP E4M3 definition for
what torch does differently (saturation to +-448 instead of NaN).  Row
quantization is pinned by its closed forms (the largest magnitude maps to
448, a zero row has scale 1, the round trip is within e4m3's half-ulp), fp8
dispatch by the row-copy property, and fp8 combine by the rounding bound of
an fp64 sum of the dequantized terms and by the pages' tolerance for an fp8
combine (rtol 0.02 / atol 0.15, TensorRT-LLM PR #13888, ConfigurableMoE
commit).
"""
import numpy as np
import pytest
import torch

from combine_moe_layout_06_b200 import inputs


def _bits_to_f64(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def test_e4m3_decode_every_code(oracle_mod):
    codes = np.arange(256, dtype=np.uint8)
    mine = oracle_mod.e4m3_to_f32(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).float().numpy()
    finite = ~np.isnan(ref)
    assert np.array_equal(mine[finite], ref[finite])
    assert np.all(np.isnan(mine[~finite])) and (~finite).sum() == 2
    assert np.nanmax(mine) == 448.0 and np.nanmin(mine) == -448.0


def test_e4m3_encode_matches_torch_in_range(oracle_mod):
    rng = np.random.default_rng(5)
    vals = np.concatenate([
        rng.standard_normal(20000).astype(np.float32) * 50,
        rng.standard_normal(5000).astype(np.float32) * 1e-2,   # subnormal range
        oracle_mod.e4m3_to_f32(np.arange(0, 127, dtype=np.uint8)),  # every finite value
    ])
    vals = vals[np.abs(vals) <= 448]
    # midpoints between neighbouring codes: ties go to the even code
    pos = oracle_mod.e4m3_to_f32(np.arange(0, 127, dtype=np.uint8)).astype(np.float64)
    mids = ((pos[:-1] + pos[1:]) / 2).astype(np.float32)
    vals = np.concatenate([vals, mids, -mids])
    got = oracle_mod.f32_to_e4m3(vals)
    ref = torch.from_numpy(vals).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(got, ref)


def test_e4m3_saturates(oracle_mod):
    got = oracle_mod.f32_to_e4m3(np.array([449.0, 1e6, -500.0, np.inf, -np.inf], np.float32))
    assert got.tolist() == [0x7E, 0x7E, 0xFE, 0x7E, 0xFE]
    assert oracle_mod.f32_to_e4m3(np.array([np.nan], np.float32)).tolist() == [0x7F]


def test_quantize_rows_closed_forms(oracle_mod):
    x = inputs.random_bf16((50, 96), seed=3, scale=3.0)
    x[7] = 0                                                   # a zero row
    q, scale = oracle_mod.quantize_rows_fp8(x)
    xf = _bits_to_f64(x)
    amax = np.abs(xf).max(axis=1)
    nz = amax > 0
    assert np.all(scale[~nz] == 1.0) and np.all(q[~nz] == 0)
    assert np.allclose(scale[nz], (amax[nz] / 448.0).astype(np.float32), rtol=0, atol=0)
    deq = oracle_mod.e4m3_to_f32(q).reshape(q.shape).astype(np.float64) * scale[:, None]
    # the largest magnitude of every row decodes to +-448
    assert np.all(np.abs(oracle_mod.e4m3_to_f32(q).reshape(q.shape)).max(axis=1)[nz] == 448.0)
    # normals: relative error <= 2^-4 (3 mantissa bits, half-ulp); tiny values: absolute
    err = np.abs(deq - xf)
    assert np.all(err <= 2.0 ** -4 * np.abs(xf) + scale[:, None] * 2.0 ** -10 + 1e-30)


def test_quantize_rows_nan_has_no_magnitude(oracle_mod):
    x = inputs.random_bf16((3, 40), seed=8, scale=2.0)
    x[0, 3] = 0x7FC0                      # quiet NaN
    x[0, 9] = 0xFFC0                      # negative quiet NaN
    clean = x.copy()
    clean[0, [3, 9]] = 0                  # the same row with zeros where the NaNs are
    q, s = oracle_mod.quantize_rows_fp8(x)
    qc, sc = oracle_mod.quantize_rows_fp8(clean)
    assert s[0] == sc[0], "the scale comes from the finite values"
    assert q[0, 3] == 0x7F and q[0, 9] == 0x7F
    keep = np.ones(40, bool)
    keep[[3, 9]] = False
    assert np.array_equal(q[0, keep], qc[0, keep])


def test_dispatch_fp8_rows_are_copies(oracle_mod):
    d = inputs.make_random(60, 32, 12, 4, seed=9)
    lay = oracle_mod.layout(d["topk_idx"], 12, 3)
    q, s = oracle_mod.dispatch_fp8(d["x"], lay["slot"])
    qx, sx = oracle_mod.quantize_rows_fp8(d["x"])
    for t in range(60):
        for j in range(4):
            row = lay["slot"][t, j]
            assert np.array_equal(q[row], qx[t]) and s[row] == sx[t]


@pytest.mark.parametrize("T,H,E,k,R", [(40, 64, 8, 2, 2), (33, 136, 13, 4, 5), (100, 16, 32, 8, 8)])
def test_combine_fp8_bounds(oracle_mod, T, H, E, k, R):
    d = inputs.make_random(T, H, E, k, seed=T + H)
    lay = oracle_mod.layout(d["topk_idx"], E, R)
    eo = inputs.random_bf16((T * k, H), seed=2 * T + H)
    q, s = oracle_mod.quantize_rows_fp8(eo)
    w = d["topk_w"]
    y = _bits_to_f64(oracle_mod.combine_fp8(q, s, w, lay["slot"]))
    qf = oracle_mod.e4m3_to_f32(q).reshape(q.shape).astype(np.float64)
    # coefficient w*scale rounds once in fp32, then k FMAs, then bf16
    coef = (w[:, :, None] * s[lay["slot"]][:, :, None]).astype(np.float32).astype(np.float64)
    terms = np.stack([coef[:, j] * qf[lay["slot"][:, j]] for j in range(k)], axis=-1)
    exact = terms.sum(-1)
    bound = 2.0 ** -8 * np.abs(exact) + (1 + 2.0 ** -8) * k * 2.0 ** -24 * np.abs(terms).sum(-1) + 1e-45
    assert np.all(np.abs(y - exact) <= bound)
    # against the bf16 combine of the unquantized rows: the pages' fp8 tolerance
    ref = _bits_to_f64(oracle_mod.combine(eo, w, lay["slot"]))
    assert np.all(np.abs(y - ref) <= 0.15 + 0.02 * np.abs(ref))
