"""The prefill path from host buffers (spa_prefill_host): the chunked, three-stream
pipeline runs the same kernels on each (b, kv-head) chunk, so its output must equal
the device-resident path's bit for bit, for every chunking (one pair per chunk, several
pairs, a ragged last chunk, fewer chunks than slots), for pinned and pageable host
memory, on a side stream; and it must match the oracle where the lists agree."""
import numpy as np
import pytest
import torch

import oracle
import block_sparse_long_stats_b200 as spa
from tests._parity import to_host
from workloads import PARITY_WORKLOADS, generate

pytestmark = pytest.mark.gpu

TOL = {"bf16": 2e-2, "f32": 1e-4}


def host_tensors(x, dtype, pin):
    def conv(a):
        if dtype == "bf16":
            t = torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)
        else:
            t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
        return t.pin_memory() if pin else t.clone()
    return conv(x["q"]), conv(x["k"]), conv(x["v"])


def run_both(w, pin=True, stream=None):
    x = generate(w)
    qh, kh, vh = host_tensors(x, w.dtype, pin)
    out = spa.spa_prefill_host(qh, kh, vh, w.block, w.top_p, w.scale, w.n_sink, w.n_local,
                               w.k_min, stream=stream)
    (stream or torch.cuda.current_stream()).synchronize()
    r = spa.prefill(qh.cuda(), kh.cuda(), vh.cuda(), w.block, w.top_p, w.scale, w.n_sink,
                    w.n_local, w.k_min)
    torch.cuda.synchronize()
    return x, out, r


@pytest.mark.parametrize("key", ["p_bf16_blk128", "p_bf16_blk64", "p_f32_d64", "p_f32_d128"])
def test_host_pipeline_equals_device_path(key):
    w = PARITY_WORKLOADS[key]
    x, out, r = run_both(w)
    assert torch.equal(out.view(torch.int16) if w.dtype == "bf16" else out,
                       r["out"].cpu().view(torch.int16) if w.dtype == "bf16" else r["out"].cpu())
    assert spa.spa_get_device_error() == 0


@pytest.mark.parametrize("B,Hq,Hkv,T", [(5, 4, 2, 700), (1, 2, 1, 1000), (3, 8, 4, 520),
                                        (9, 4, 1, 300), (1, 8, 1, 700), (2, 8, 2, 520)])
def test_host_pipeline_chunkings(B, Hq, Hkv, T):
    # pairs 10 (chunks of 2), 1 (one chunk, one slot), 12 (chunks of 2), 9 (chunks
    # of 2, the last one pair); 1 and 4 pairs of 8 and 4 heads (one pair per chunk)
    w = PARITY_WORKLOADS["p_bf16_blk64"].with_(B=B, Hq=Hq, Hkv=Hkv, T=T)
    s = torch.cuda.Stream()
    x, out, r = run_both(w, pin=True, stream=s)
    assert torch.equal(out.view(torch.int16), r["out"].cpu().view(torch.int16))


def test_host_pipeline_pageable_memory():
    w = PARITY_WORKLOADS["p_bf16_blk128"]
    x, out, r = run_both(w, pin=False)
    assert torch.equal(out.view(torch.int16), r["out"].cpu().view(torch.int16))


def test_host_pipeline_matches_oracle():
    w = PARITY_WORKLOADS["p_bf16_blk128"]
    x, out, r = run_both(w)
    sel = oracle.select(x["q"], x["k"], w.dtype, w.block, w.scale, w.top_p, w.n_sink, w.n_local,
                        w.k_min)
    o_out, _ = oracle.attention(x["q"], x["k"], x["v"], w.dtype, w.block, sel["idx"],
                                sel["count"], w.scale)
    g_idx, g_cnt = r["idx"].cpu().numpy(), r["count"].cpu().numpy()
    got = to_host(out)
    checked = 0
    for b in range(w.B):
        for h in range(w.Hq):
            for i in range(w.nq):
                c = g_cnt[b, h, i]
                if c == sel["count"][b, h, i] and np.array_equal(g_idx[b, h, i, :c],
                                                                  sel["idx"][b, h, i, :c]):
                    rows = slice(i * w.block, min(w.T, (i + 1) * w.block))
                    assert np.abs(got[b, h, rows] - o_out[b, h, rows]).max() <= TOL[w.dtype]
                    checked += 1
    assert checked >= 0.9 * w.B * w.Hq * w.nq
