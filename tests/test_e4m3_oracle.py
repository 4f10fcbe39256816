"""Pins for the e4m3 codec and the per-tile quantiser of the oracle."""

import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import (E4M3_MAX, attention_ref, dequantize_e4m3_tiles, e4m3_decode,
                    e4m3_encode_rne_satfinite, quantize_e4m3_tiles)


def test_format_constants():
    vals = e4m3_decode(np.arange(256, dtype=np.uint8))
    assert np.nanmax(vals) == 448.0 == E4M3_MAX
    assert np.isnan(vals[0x7F]) and np.isnan(vals[0xFF])
    assert np.sum(np.isnan(vals)) == 2            # no infinities, two NaNs
    assert vals[0x01] == 2.0 ** -9                  # smallest subnormal
    assert vals[0x08] == 2.0 ** -6                  # smallest normal
    assert vals[0x38] == 1.0


def test_all_codes_round_trip():
    codes = np.arange(256, dtype=np.uint8)
    finite = ~np.isnan(e4m3_decode(codes))
    back = e4m3_encode_rne_satfinite(e4m3_decode(codes[finite]))
    assert np.array_equal(back, codes[finite])


def test_matches_torch_cast_inside_range():
    """torch.float8_e4m3fn conversion (a library routine used as a black box)
    rounds to nearest even but does not saturate, so compare where |x| <= 464."""
    rng = np.random.default_rng(1)
    x = np.concatenate([
        rng.standard_normal(200000).astype(np.float32) * 50,
        rng.standard_normal(50000).astype(np.float32) * 1e-2,
        rng.uniform(-464, 464, 50000).astype(np.float32),
    ])
    pos = e4m3_decode(np.arange(0x7F, dtype=np.uint8))
    mids = ((pos[1:] + pos[:-1]) / 2).astype(np.float32)      # exact ties
    x = np.concatenate([x, mids, -mids]).astype(np.float32)
    ours = e4m3_encode_rne_satfinite(x)
    theirs = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ours, theirs)


def test_ties_go_to_even_and_saturation():
    assert e4m3_encode_rne_satfinite(np.array([464.0]))[0] == 0x7E   # tie 448|480 -> 448 (even)
    assert e4m3_encode_rne_satfinite(np.array([1.0625]))[0] == 0x38  # tie 1|1.125 -> 1.0
    assert e4m3_encode_rne_satfinite(np.array([1.1875]))[0] == 0x3A  # tie 1.125|1.25 -> 1.25
    big = e4m3_encode_rne_satfinite(np.array([449.0, 1e6, -1e30, np.float32(3e38)]))
    assert list(big) == [0x7E, 0x7E, 0xFE, 0x7E]
    assert e4m3_encode_rne_satfinite(np.array([np.nan]))[0] == 0x7F
    assert e4m3_encode_rne_satfinite(np.array([-0.0]))[0] == 0x80


def _bf16(shape, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(shape, generator=g) * scale).to(torch.bfloat16)


def test_quantiser_scale_and_codes():
    x = _bf16((2, 3, 300, 32), 2)          # 3 tiles per head, ragged last tile
    x[1, 2, 128:256] = 0                   # an all-zero tile
    codes, scales = quantize_e4m3_tiles(x)
    assert codes.shape == (2, 3, 300, 32) and scales.shape == (2, 3, 3)
    assert scales[1, 2, 1] == 1.0 and not codes[1, 2, 128:256].any()
    xf = x.float().numpy()
    for b in range(2):
        for h in range(3):
            for t in range(3):
                blk = xf[b, h, t * 128:(t + 1) * 128]
                amax = np.float32(np.abs(blk).max())
                if amax == 0:
                    continue
                assert scales[b, h, t] == np.float32(448.0) / amax
                # the absolute maximum lands on the largest code
                assert (codes[b, h, t * 128:(t + 1) * 128] & 0x7F).max() == 0x7E


def test_quantiser_error_envelope():
    """|x - dequant(x)| <= 2^-4 |x| in the normal range, <= 2^-10 / scale below it."""
    x = _bf16((1, 2, 256, 64), 3)
    codes, scales = quantize_e4m3_tiles(x)
    deq = dequantize_e4m3_tiles(codes, scales)
    xf = x.double().numpy()
    sc = np.repeat(scales.astype(np.float64), 128, axis=2)[..., None]
    bound = np.maximum(np.abs(xf) * 2.0 ** -4, 2.0 ** -10 / sc) * (1 + 1e-6)
    assert np.all(np.abs(deq - xf) <= bound)


def test_fp8_scale_folding_identity():
    """The page's FP8 identity: S on the quantised operands times
    1/(q_scale*k_scale) equals S on the dequantised operands."""
    q, k = _bf16((1, 1, 256, 128), 4), _bf16((1, 1, 256, 128), 5)
    cq, sq = quantize_e4m3_tiles(q)
    ck, sk = quantize_e4m3_tiles(k)
    raw = e4m3_decode(cq[0, 0]) @ e4m3_decode(ck[0, 0]).T          # on the codes' values
    tile = np.arange(256) // 128
    folded = raw * (1.0 / (sq[0, 0][tile][:, None].astype(np.float64) *
                           sk[0, 0][tile][None, :].astype(np.float64)))
    deq = dequantize_e4m3_tiles(cq, sq)[0, 0] @ dequantize_e4m3_tiles(ck, sk)[0, 0].T
    assert np.max(np.abs(folded - deq)) <= 1e-12 * np.max(np.abs(deq))


def test_fp8_attention_envelope():
    """Attention on dequantised Q/K stays near attention on the source values
    for N(0,1) inputs (quantisation moves each score by a few 1e-2)."""
    q, k, v = _bf16((1, 2, 256, 128), 4), _bf16((1, 2, 256, 128), 5), _bf16((1, 2, 256, 128), 6)
    cq, sq = quantize_e4m3_tiles(q)
    ck, sk = quantize_e4m3_tiles(k)
    o_src, l_src = attention_ref(q, k, v, 1 / math.sqrt(128), True)
    o_deq, l_deq = attention_ref(dequantize_e4m3_tiles(cq, sq), dequantize_e4m3_tiles(ck, sk), v,
                                 1 / math.sqrt(128), True)
    err = np.abs(o_src - o_deq)
    assert 0 < err.max() < 0.15 and err.mean() < 1e-2
    assert np.max(np.abs(l_src - l_deq)) < 0.15


def test_page_accounting_golden():
    """FLOP and byte accounting pinned to the figures the pages print."""
    from oracle import attention_flops
    from tiled_attention_12_b200.synth import Case

    path = os.path.join(os.path.dirname(__file__), "golden", "page_accounting.json")
    g = json.load(open(path))
    e = g["gemm_flops_n8192_d128"]
    per_gemm = attention_flops(1, 1, e["n"], e["d"], False) / 2
    assert abs(per_gemm / 2 ** 30 - e["approx_per_gemm_gflop"]) < 0.05 * e["approx_per_gemm_gflop"]
    assert abs(2 * per_gemm / 2 ** 30 - e["approx_total_gflop"]) < 0.05 * e["approx_total_gflop"]
    assert Case("x", 1, 1, e["n"], e["d"], False, 0).flops == attention_flops(1, 1, e["n"], e["d"], False)
    assert Case("x", 2, 3, 100, 64, True, 0).flops == attention_flops(2, 3, 100, 64, True)
    s = g["score_matrix_bytes_n8192_fp32"]
    assert s["n"] ** 2 * 4 == s["mib"] * 2 ** 20
    big = g["score_matrix_bytes_n131072"]
    assert big["n"] ** 2 * 4 == big["gib"] * 2 ** 30
