"""fa_fwd_e4m3_noalloc: the e4m3 forward for callers that cannot allocate.

Callers inside allocator or memory-pool callbacks, on devices whose memory is
already handed out to a pool they do not own, or under a no-allocation-after-
start-up policy cannot let the library cudaMalloc its quantisation scratch.
This entry point uses a static device array instead.  The test checks,
through the C ABI, that two calls in a row match the regular FA_E4M3 path of
fa_fwd within the FP8 tolerance of the other tests, and that the second call
leaves the device's free memory unchanged.  Collected last on purpose.
"""

from __future__ import annotations

import numpy as np
import pytest
import torch

from tiled_attention_12_b200 import binding as B
from tiled_attention_12_b200.synth import Case, make_qkv

from parity_util import TOL_FP8, gate

pytestmark = pytest.mark.gpu


def _inputs(seed, N, causal):
    c = Case("na", 1, 3, N, 128, causal, seed=seed, outlier_frac=0.01)
    return c, [t.cuda() for t in make_qkv(c)]


def _call(L, q, k, v, o, lse, c):
    return L.fa_fwd_e4m3_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                                 c.B, c.H, c.N, c.d, c.softmax_scale, int(c.causal),
                                 torch.cuda.current_stream().cuda_stream)


def test_noalloc_matches_regular_e4m3_path_twice():
    L = B.load()
    runs = [(_inputs(7, 1000, True)), (_inputs(8, 777, False))]
    for i, (c, (q, k, v)) in enumerate(runs):
        o_ref, lse_ref = B.fa_fwd(q, k, v, causal=c.causal, dtype=B.FA_E4M3)
        o = torch.empty_like(v)
        lse = torch.empty((c.B, c.H, c.N), device="cuda", dtype=torch.float32)
        torch.cuda.synchronize()
        free_before = torch.cuda.mem_get_info()[0]
        assert _call(L, q, k, v, o, lse, c) == B.FA_OK
        torch.cuda.synchronize()
        if i == 1:   # set-up happened in the first call; later calls allocate nothing
            assert torch.cuda.mem_get_info()[0] == free_before
        gate(o, o_ref.float().cpu().double().numpy(), lse, lse_ref.cpu().double().numpy(), tol=TOL_FP8,
             what=f"no-alloc call {i}")


def test_noalloc_rejects_sizes_beyond_its_scratch():
    L = B.load()
    P = 1 << 20   # never dereferenced: the size check comes first
    s = torch.cuda.current_stream().cuda_stream
    too_many = B.load().fa_fwd_e4m3_noalloc(P, P, P, P * 2, None, 1, 16, 8192, 128, 0.1, 1, s)
    assert too_many == B.FA_ERR_TOO_LARGE
    assert L.fa_status_string(B.FA_ERR_TOO_LARGE).startswith(b"problem exceeds")
