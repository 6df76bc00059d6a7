"""The allocation-free decode entry point (spa_sparse_attn_decode_noalloc).

It serves callers that cannot allocate device memory for the call (a plugin
interface that passes only input and output buffers, a hot loop that must not call
cudaMalloc). These tests call it through the C-ABI and check that, on two calls in
a row, it returns bit for bit what the workspace-taking spa_sparse_attn_decode
returns (the same kernels on the same inputs, only the partials live elsewhere),
that both agree with the CPU oracle within the bf16 tolerance of the other parity
tests, and that sizes needing more scratch than the built-in 8 MiB are refused.
This file is collected last, so a run that stops at its first failure has run
everything else.
"""
import ctypes

import numpy as np
import pytest
import torch

import block_sparse_long_stats_b200 as spa
import oracle
from workloads import PARITY_WORKLOADS, generate

pytestmark = pytest.mark.gpu

TOL = 2e-2   # bf16 output tolerance used by the other parity tests
P, I, F = ctypes.c_void_p, ctypes.c_int, ctypes.c_float


def _noalloc():
    f = spa.lib().spa_sparse_attn_decode_noalloc
    f.argtypes = [P, P, P, I, I, I, I, I, I, I, P, I, P, F, P, P]
    f.restype = I
    return f


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda().view(torch.bfloat16)


@pytest.mark.parametrize("key", ["d_bf16_blk16", "d_bf16_blk64"])
def test_noalloc_decode_matches_workspace_decode_on_two_calls(key):
    w = PARITY_WORKLOADS[key]
    x = generate(w)
    q, k, v = _dev(x["q"]), _dev(x["k"]), _dev(x["v"])
    mean, var = spa.spa_block_stats(k, w.block)
    idx, cnt = spa.spa_select(q, mean, var, w.T, w.block, w.scale, w.top_p)
    ref = spa.spa_sparse_attn_decode(q, k, v, w.block, idx, cnt, w.scale)
    torch.cuda.synchronize()
    o_ref, _ = oracle.attention(x["q"], x["k"], x["v"], w.dtype, w.block, idx.cpu().numpy(),
                                cnt.cpu().numpy(), w.scale)
    f = _noalloc()
    stream = P(torch.cuda.current_stream().cuda_stream)
    for call in range(2):
        out = torch.full_like(q, float("nan"))
        st = f(P(q.data_ptr()), P(k.data_ptr()), P(v.data_ptr()), 1, w.B, w.Hq, w.Hkv, w.T, w.d,
               w.block, P(idx.data_ptr()), idx.shape[-1], P(cnt.data_ptr()), w.scale,
               P(out.data_ptr()), stream)
        assert st == 0, spa.spa_last_error()
        torch.cuda.synchronize()
        assert torch.equal(out.view(torch.int16), ref.view(torch.int16)), call
        err = float(np.abs(out.float().cpu().numpy().reshape(o_ref.shape) - o_ref).max())
        assert err <= TOL, (call, err)
    assert spa.spa_get_device_error() == 0


def test_noalloc_decode_refuses_sizes_beyond_its_scratch():
    f = _noalloc()
    q = torch.zeros((1, 1, 1, 128), dtype=torch.bfloat16, device="cuda")
    idx = torch.zeros((1,), dtype=torch.int32, device="cuda")
    # B=64, Hq=64, T=2^20: the split-KV partials need far more than 8 MiB; the call
    # is refused on the host before anything is launched or read.
    B, Hq, Hkv, T, blk = 64, 64, 8, 1 << 20, 16
    need = spa.spa_decode_workspace_bytes(B, Hq, Hkv, T, 128, blk)
    assert need > 8 << 20
    p = P(q.data_ptr())
    st = f(p, p, p, 1, B, Hq, Hkv, T, 128, blk, P(idx.data_ptr()), T // blk, P(idx.data_ptr()),
           0.088, p, P(torch.cuda.current_stream().cuda_stream))
    assert st == 2                                   # SPA_ERR_UNSUPPORTED
    assert "maximum" in spa.spa_last_error()
