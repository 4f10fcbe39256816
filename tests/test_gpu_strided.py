"""GPU checks of the strided forward (fa_fwd_strided through fa_fwd on
non-contiguous views): the (batch, seq, heads, dim) layout, q/k/v sliced out
of one packed projection, and an output written into a padded buffer.

The kernel's arithmetic does not depend on where a row lives, so a strided
call must return exactly the bytes of the contiguous call on the same values;
one case per layout is also gated against the fp64 oracle."""

from __future__ import annotations

import pytest
import torch

import tiled_attention_12_b200 as fa
from oracle import attention_ref, dequantize_e4m3_tiles, quantize_e4m3_tiles
from parity_util import TOL_16, gate
from tiled_attention_12_b200.synth import Case, make_qkv

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _bnhd(x):
    """The same values stored (batch, seq, heads, dim), seen as [B, H, N, d]."""
    return x.transpose(1, 2).contiguous().transpose(1, 2)


def _run(q, k, v, causal, code=None, o=None):
    o, lse = fa.fa_fwd(q, k, v, o=o, causal=causal, dtype=code)
    torch.cuda.synchronize()
    assert fa.fa_last_device_status() == 0
    return o, lse


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [200, 1000, 2048])
@pytest.mark.parametrize("d", [32, 64, 128])
def test_bnhd_layout_is_bit_identical(d, N, causal, dtype):
    case = Case("bnhd", 2, 3, N, d, causal, seed=N + d)
    q, k, v = (t.to(DEV) for t in make_qkv(case, dtype=dtype))
    oc, lc = _run(q, k, v, causal)
    qs, ks, vs = _bnhd(q), _bnhd(k), _bnhd(v)
    assert not qs.is_contiguous() and qs.stride() == (N * 3 * d, d, 3 * d, 1)
    os_, ls = _run(qs, ks, vs, causal)
    assert os_.stride() == vs.stride()          # output in the same layout as v
    assert torch.equal(os_, oc) and torch.equal(ls, lc)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("d", [64, 128])
def test_packed_qkv_slices(d, causal):
    """q, k, v as slices of one [B, N, 3, H, d] projection output."""
    B, H, N = 2, 4, 777
    case = Case("packed", B, H, N, d, causal, seed=d)
    q, k, v = (t.to(DEV) for t in make_qkv(case))
    qkv = torch.empty((B, N, 3, H, d), device=DEV, dtype=torch.bfloat16)
    for i, t in enumerate((q, k, v)):
        qkv[:, :, i] = t.transpose(1, 2)
    qs, ks, vs = (qkv[:, :, i].transpose(1, 2) for i in range(3))
    assert qs.stride() == (N * 3 * H * d, d, 3 * H * d, 1)
    oc, lc = _run(q, k, v, causal)
    os_, ls = _run(qs, ks, vs, causal, o=torch.empty_like(q))
    assert torch.equal(os_, oc) and torch.equal(ls, lc)


def test_output_into_padded_buffer_leaves_padding():
    """O written into the first d columns of rows 64 elements wider."""
    B, H, N, d = 1, 2, 300, 64
    case = Case("pad", B, H, N, d, True, seed=5)
    q, k, v = (t.to(DEV) for t in make_qkv(case))
    buf = torch.full((B, H, N, d + 64), 7.0, device=DEV, dtype=torch.bfloat16)
    o = buf[..., :d]
    assert o.stride() == (H * N * (d + 64), N * (d + 64), d + 64, 1)
    _run(q, k, v, True, o=o)
    oc, _ = _run(q, k, v, True)
    assert torch.equal(o, oc)
    assert bool((buf[..., d:] == 7.0).all())


@pytest.mark.parametrize("causal", [False, True])
def test_bnhd_against_oracle(causal):
    case = Case("bnhd_ref", 1, 2, 777, 64, causal, seed=9)
    q, k, v = make_qkv(case)
    o, lse = _run(_bnhd(q.to(DEV)), _bnhd(k.to(DEV)), _bnhd(v.to(DEV)), causal)
    ro, rl = attention_ref(q, k, v, case.softmax_scale, causal)
    gate(o, ro, lse, rl, tol=TOL_16, what="bnhd")


@pytest.mark.parametrize("causal", [False, True])
def test_e4m3_strided_matches_contiguous(causal):
    """FA_E4M3 with strided q, k: the quantiser reads the views and writes
    contiguous codes, so the result equals the contiguous call's; also gated
    against the oracle on the dequantised codes."""
    case = Case("bnhd_fp8", 2, 2, 640, 128, causal, seed=13)
    q, k, v = make_qkv(case)
    qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
    oc, lc = _run(qd, kd, vd, causal, code=fa.FA_E4M3)
    os_, ls = _run(_bnhd(qd), _bnhd(kd), _bnhd(vd), causal, code=fa.FA_E4M3)
    assert torch.equal(os_, oc) and torch.equal(ls, lc)
    cq, sq = quantize_e4m3_tiles(q)
    ck, sk = quantize_e4m3_tiles(k)
    ro, rl = attention_ref(dequantize_e4m3_tiles(cq, sq), dequantize_e4m3_tiles(ck, sk), v,
                           case.softmax_scale, causal)
    gate(os_, ro, ls, rl, tol=TOL_16, what="e4m3 bnhd")


def test_many_work_tiles_bnhd():
    """B2 H8 N8192 d128: more work tiles than SMs, (batch, seq, heads, dim)."""
    case = Case("bnhd_big", 2, 8, 8192, 128, True, seed=17, value_scale=0.5)
    q, k, v = (t.to(DEV) for t in make_qkv(case))
    oc, lc = _run(q, k, v, True)
    os_, ls = _run(_bnhd(q), _bnhd(k), _bnhd(v), True)
    assert torch.equal(os_, oc) and torch.equal(ls, lc)


def test_bad_strides_raise():
    q = torch.zeros((1, 2, 256, 64), device=DEV, dtype=torch.bfloat16)
    wide = torch.zeros((1, 2, 256, 68), device=DEV, dtype=torch.bfloat16)[..., :64]   # row stride 68
    with pytest.raises(fa.FaError):
        fa.fa_fwd(wide, q, q)
