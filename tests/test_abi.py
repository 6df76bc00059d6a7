"""The C-ABI library loads and exports every call include/spa.h declares, and the
host-side checks reject bad arguments before any launch. CPU only: nothing here
reaches a kernel or needs a device."""
import ctypes
import os
import re
import subprocess

import pytest

from block_sparse_long_stats_b200 import build as spa_build

HEADER = os.path.join(os.path.dirname(os.path.dirname(__file__)), "include", "spa.h")


@pytest.fixture(scope="module")
def lib():
    path = spa_build.build()
    return ctypes.CDLL(path)


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(spa_[a-z_]+)\s*\(", src)))


def test_header_declares_the_pipeline_calls():
    names = declared_functions()
    for n in ("spa_block_stats", "spa_select", "spa_sparse_attn_prefill",
              "spa_sparse_attn_decode", "spa_decode_workspace_bytes", "spa_get_device_error"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    for n in declared_functions():
        assert hasattr(lib, n), f"{n} declared in spa.h but not exported"


def test_only_the_abi_is_exported():
    out = subprocess.run(["nm", "-D", "--defined-only", spa_build.LIB], capture_output=True,
                         text=True, check=True).stdout
    exported = {l.split()[-1] for l in out.splitlines() if " T " in l}
    ours = {s for s in exported if s.startswith("spa_")}
    assert ours == set(declared_functions())


def test_status_strings(lib):
    lib.spa_status_string.restype = ctypes.c_char_p
    assert lib.spa_status_string(0) == b"ok"
    assert lib.spa_status_string(1) == b"invalid argument"
    assert lib.spa_status_string(2) == b"unsupported shape or dtype"


P = ctypes.c_void_p
FAKE = P(0x10000)   # aligned, never dereferenced: every call below fails a host check first


def _last(lib):
    lib.spa_last_error.restype = ctypes.c_char_p
    return lib.spa_last_error().decode()


def test_selftest_wait_limit_host_checks(lib):
    f = lib.spa_selftest_wait_timeout
    f.argtypes = [ctypes.c_int, P]
    assert f(0, None) == 1
    assert f(-5, None) == 1
    assert f(1000001, None) == 1
    assert "limit_us" in _last(lib)


def test_block_stats_host_checks(lib):
    f = lib.spa_block_stats
    f.argtypes = [P] + [ctypes.c_int] * 8 + [P, P, P]
    assert f(None, 1, 1, 1, 64, 128, 64, 0, 1, FAKE, FAKE, None) == 1
    assert f(FAKE, 1, 0, 1, 64, 128, 64, 0, 1, FAKE, FAKE, None) == 1
    assert f(FAKE, 1, 1, 1, 64, 128, 64, 0, 2, FAKE, FAKE, None) == 1      # range beyond nb
    assert "range" in _last(lib)
    assert f(FAKE, 1, 1, 1, 64, 96, 64, 0, 1, FAKE, FAKE, None) == 2       # d = 96
    assert f(FAKE, 1, 1, 1, 64, 128, 48, 0, 1, FAKE, FAKE, None) == 2      # block 48
    assert f(P(0x10008), 1, 1, 1, 64, 128, 64, 0, 1, FAKE, FAKE, None) == 1  # misaligned


def test_select_host_checks(lib):
    f = lib.spa_select
    I, F = ctypes.c_int, ctypes.c_float
    f.argtypes = [P, I, P, P, I, I, I, I, I, I, I, F, F, I, I, I, P, I, P, P]
    ok = dict(B=1, Hq=4, Hkv=2, Lq=256, T=256, d=128, block=64, scale=0.1, top_p=0.9, n_sink=1,
              n_local=1, k_min=0, cap=4)

    def call(**kw):
        a = dict(ok, **kw)
        return f(FAKE, 1, FAKE, FAKE, a["B"], a["Hq"], a["Hkv"], a["Lq"], a["T"], a["d"],
                 a["block"], a["scale"], a["top_p"], a["n_sink"], a["n_local"], a["k_min"], FAKE,
                 a["cap"], FAKE, None)

    assert call(Hq=3) == 1
    assert call(Lq=100) == 1
    assert call(top_p=0.0) == 1
    assert call(scale=-1.0) == 1
    assert call(cap=3) == 1
    assert call(n_sink=-1) == 1
    assert call(d=96) == 2


def test_prefill_and_decode_host_checks(lib):
    I, F = ctypes.c_int, ctypes.c_float
    f = lib.spa_sparse_attn_prefill
    f.argtypes = [P, P, P, I, I, I, I, I, I, I, P, I, P, F, P, P, P]
    assert f(FAKE, FAKE, FAKE, 1, 1, 4, 2, 256, 96, 64, FAKE, 4, FAKE, 0.1, FAKE, None, None) == 2
    assert f(FAKE, FAKE, FAKE, 1, 1, 4, 2, 256, 128, 32, FAKE, 8, FAKE, 0.1, FAKE, None, None) == 2
    assert f(FAKE, FAKE, FAKE, 1, 1, 2, 2, 256, 128, 64, FAKE, 4, FAKE, 0.1, FAKE, None, None) == 2
    assert f(FAKE, FAKE, FAKE, 1, 1, 4, 2, 256, 128, 64, FAKE, 3, FAKE, 0.1, FAKE, None, None) == 1
    assert f(FAKE, FAKE, None, 1, 1, 4, 2, 256, 128, 64, FAKE, 4, FAKE, 0.1, FAKE, None, None) == 1
    g = lib.spa_sparse_attn_decode
    g.argtypes = [P, P, P, I, I, I, I, I, I, I, P, I, P, F, P, P, P]
    assert g(FAKE, FAKE, FAKE, 0, 1, 4, 2, 256, 128, 16, FAKE, 16, FAKE, 0.1, FAKE, FAKE, None) == 2
    assert g(FAKE, FAKE, FAKE, 1, 1, 4, 2, 256, 128, 16, FAKE, 15, FAKE, 0.1, FAKE, FAKE, None) == 1
    assert g(FAKE, FAKE, FAKE, 1, 1, 4, 2, 256, 128, 16, FAKE, 16, FAKE, 0.1, None, FAKE, None) == 1


def test_rla_host_checks(lib):
    I = ctypes.c_int
    f = lib.spa_rla_block_states
    f.argtypes = [P, P, I, I, I, I, I, I, I, I, P, P]
    assert f(FAKE, FAKE, 0, 1, 2, 256, 128, 128, 0, 2, FAKE, None) == 2     # fp32
    assert f(FAKE, FAKE, 1, 1, 2, 256, 64, 128, 0, 2, FAKE, None) == 2      # d = 64
    assert f(FAKE, FAKE, 1, 1, 2, 256, 128, 16, 0, 16, FAKE, None) == 2     # block 16
    assert f(FAKE, FAKE, 1, 1, 2, 256, 128, 128, 0, 3, FAKE, None) == 1     # blk_end > nb
    assert f(FAKE, FAKE, 1, 1, 2, 256, 128, 128, 2, 1, FAKE, None) == 1     # begin > end
    assert f(FAKE, None, 1, 1, 2, 256, 128, 128, 0, 2, FAKE, None) == 1
    g = lib.spa_rla_prefill
    g.argtypes = [P, P, P, P, I, I, I, I, I, I, I, P, I, P, P, P]
    assert g(FAKE, FAKE, FAKE, FAKE, 0, 1, 4, 2, 256, 128, 128, FAKE, 2, FAKE, FAKE, None) == 2
    assert g(FAKE, FAKE, FAKE, FAKE, 1, 1, 4, 2, 256, 128, 32, FAKE, 8, FAKE, FAKE, None) == 2
    assert g(FAKE, FAKE, FAKE, FAKE, 1, 1, 4, 2, 256, 128, 128, FAKE, 1, FAKE, FAKE, None) == 1
    assert g(FAKE, FAKE, FAKE, FAKE, 1, 1, 4, 3, 256, 128, 128, FAKE, 2, FAKE, FAKE, None) == 1
    assert g(FAKE, FAKE, FAKE, None, 1, 1, 4, 2, 256, 128, 128, FAKE, 2, FAKE, FAKE, None) == 1


def test_rla_decode_host_checks(lib):
    I, F = ctypes.c_int, ctypes.c_float
    f = lib.spa_rla_decode_state
    f.argtypes = [P, P, I, I, I, I, I, I, I, P, P]
    assert f(FAKE, FAKE, 0, 1, 2, 256, 128, 0, 256, FAKE, None) == 2       # fp32
    assert f(FAKE, FAKE, 1, 1, 2, 256, 128, 0, 257, FAKE, None) == 1       # beyond T
    assert f(FAKE, FAKE, 1, 1, 2, 256, 128, 9, 8, FAKE, None) == 1         # begin > end
    assert f(FAKE, FAKE, 1, 1, 2, 256, 128, 0, 256, None, None) == 1
    g = lib.spa_sparse_attn_decode_rla
    g.argtypes = [P, P, P, P, I, I, I, I, I, I, I, P, I, P, F, P, P, P, P]
    assert g(FAKE, FAKE, FAKE, FAKE, 1, 1, 4, 2, 256, 128, 128, FAKE, 2, FAKE, 0.1, FAKE, FAKE,
             FAKE, None) == 2                                               # block 128
    assert g(FAKE, FAKE, FAKE, FAKE, 1, 1, 32, 2, 256, 128, 16, FAKE, 16, FAKE, 0.1, FAKE, FAKE,
             FAKE, None) == 2                                               # 16 heads per group
    assert g(FAKE, FAKE, FAKE, FAKE, 1, 1, 4, 2, 256, 128, 16, FAKE, 16, FAKE, 0.1, FAKE, FAKE,
             None, None) == 1                                               # no out_rla
    h = lib.spa_rla_decode_workspace_bytes
    h.restype = ctypes.c_size_t
    h.argtypes = [I] * 6
    d = lib.spa_decode_workspace_bytes
    d.restype = ctypes.c_size_t
    d.argtypes = [I] * 6
    assert h(16, 32, 8, 131072, 128, 16) > d(16, 32, 8, 131072, 128, 16)
    assert h(0, 32, 8, 131072, 128, 16) == 0


def test_quantized_stats_host_checks(lib):
    I, F = ctypes.c_int, ctypes.c_float
    n = lib.spa_quantized_stats_bytes
    n.restype = ctypes.c_size_t
    n.argtypes = [I] * 5
    assert n(16, 8, 131072, 128, 16) == 16 * 8 * 8192 * 136
    assert n(1, 1, 100, 96, 16) == 0                                     # d % 32
    f = lib.spa_quantize_block_stats
    f.argtypes = [P, P, I, I, I, I, I, I, I, P, I, P]
    assert f(FAKE, FAKE, 1, 2, 256, 96, 16, 0, 16, FAKE, 0, None) == 2    # d = 96
    assert f(FAKE, FAKE, 1, 2, 256, 128, 16, 0, 17, FAKE, 1, None) == 1   # beyond nb
    assert f(FAKE, None, 1, 2, 256, 128, 16, 0, 16, FAKE, 0, None) == 1
    assert f(FAKE, FAKE, 1, 2, 256, 128, 16, 0, 16, FAKE, 2, None) == 1   # unknown format
    h = lib.spa_block_stats_quantized
    h.argtypes = [P, I, I, I, I, I, I, I, I, P, P, P, I, P]
    assert h(FAKE, 1, 1, 2, 256, 128, 16, 0, 16, FAKE, FAKE, FAKE, 3, None) == 1   # unknown format
    assert h(FAKE, 1, 1, 2, 256, 96, 16, 0, 16, FAKE, FAKE, FAKE, 1, None) == 2    # d = 96
    g = lib.spa_select_quantized
    g.argtypes = [P, I, P, I, I, I, I, I, I, I, I, F, F, I, I, I, P, I, P, P]
    assert g(FAKE, 1, FAKE, 0, 1, 4, 2, 1, 256, 128, 16, 0.1, 0.9, 1, 1, 0, FAKE, 15, FAKE, None) == 1
    assert g(FAKE, 1, FAKE, 1, 1, 4, 2, 1, 256, 96, 16, 0.1, 0.9, 1, 1, 0, FAKE, 16, FAKE, None) == 2
    assert g(FAKE, 1, None, 0, 1, 4, 2, 1, 256, 128, 16, 0.1, 0.9, 1, 1, 0, FAKE, 16, FAKE, None) == 1
    assert g(FAKE, 1, FAKE, -1, 1, 4, 2, 1, 256, 128, 16, 0.1, 0.9, 1, 1, 0, FAKE, 16, FAKE, None) == 1


def test_early_stop_host_checks(lib):
    I, F = ctypes.c_int, ctypes.c_float
    f = lib.spa_sparse_attn_prefill_early_stop
    f.argtypes = [P, P, P, I, I, I, I, I, I, I, P, I, P, F, I, I, F, P, P, P, P]
    args = lambda dt, d, blk, cap, tau, proc: (FAKE, FAKE, FAKE, dt, 1, 4, 2, 512, d, blk, FAKE, cap,
                                               FAKE, 0.1, 1, 1, tau, FAKE, None, proc, None)
    assert f(*args(1, 128, 64, 8, 0.1, FAKE)) == 2           # block 64
    assert f(*args(0, 128, 128, 4, 0.1, FAKE)) == 2          # fp32
    assert f(*args(1, 128, 128, 3, 0.1, FAKE)) == 1          # cap < nb
    assert f(*args(1, 128, 128, 4, -1.0, FAKE)) == 1         # tau < 0
    assert f(*args(1, 128, 128, 4, 0.1, None)) == 1          # no processed output
    g = lib.spa_select_score_order
    g.argtypes = [P, I, P, P, I, I, I, I, I, I, F, F, I, I, I, P, I, P, P]
    assert g(FAKE, 1, FAKE, FAKE, 1, 4, 2, 512, 96, 128, 0.1, 0.9, 1, 1, 0, FAKE, 4, FAKE, None) == 2
    assert g(FAKE, 1, FAKE, FAKE, 1, 4, 2, 512, 128, 128, 0.1, 0.9, 1, 1, 0, FAKE, 3, FAKE, None) == 1


def test_decode_workspace_size(lib):
    f = lib.spa_decode_workspace_bytes
    f.restype = ctypes.c_size_t
    f.argtypes = [ctypes.c_int] * 6
    n = f(16, 32, 8, 131072, 128, 16)
    assert n > 0 and n % (16 * 32 * 130 * 4) == 0
    assert f(0, 32, 8, 131072, 128, 16) == 0


def test_prefill_host_checks_and_workspace(lib):
    I, F, Z = ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    w = lib.spa_prefill_host_workspace_bytes
    w.restype = Z
    w.argtypes = [I] * 7
    one = w(1, 1, 4, 1, 4096, 128, 128)            # one (b, kv-head) pair: one slot
    assert one > 0 and one % 256 == 0
    # per pair: q + out (4 x 4096 x 128 x 2 each), k, v, mean, var, lists, counts
    G, L, d, nb = 4, 4096, 128, 32
    per_pair = 2 * G * L * d * 2 + 2 * L * d * 2 + 2 * nb * d * 4 + G * nb * nb * 4 + G * nb * 4
    assert per_pair <= one < per_pair + 8 * 256
    assert w(1, 1, 8, 2, 4096, 128, 128) == 2 * one      # two pairs: two chunks, two slots
    assert w(1, 2, 8, 2, 4096, 128, 128) == 3 * one      # four pairs: four chunks, three slots
    assert w(1, 1, 32, 8, 4096, 128, 128) == 3 * one     # eight chunks share three slots
    assert w(1, 8, 32, 8, 4096, 128, 128) >= 3 * 8 * per_pair   # chunks of eight pairs
    assert w(1, 0, 4, 1, 4096, 128, 128) == 0
    assert w(1, 1, 3, 2, 4096, 128, 128) == 0            # Hq not a multiple of Hkv
    f = lib.spa_prefill_host
    f.argtypes = [P, P, P, P, I, I, I, I, I, I, I, F, F, I, I, I, P, Z, P]
    ok = dict(dt=1, B=1, Hq=4, Hkv=1, L=4096, d=128, block=128, top_p=0.9, ws=FAKE, nws=one)

    def call(q=FAKE, **kw):
        a = dict(ok, **kw)
        return f(q, FAKE, FAKE, FAKE, a["dt"], a["B"], a["Hq"], a["Hkv"], a["L"], a["d"],
                 a["block"], 0.1, a["top_p"], 1, 1, 0, a["ws"], a["nws"], None)

    assert call(q=None) == 1
    assert call(Hq=3, Hkv=2) == 1
    assert call(top_p=0.0) == 1
    assert call(d=64) == 2                   # bf16 attention needs d = 128
    assert call(block=32) == 2
    assert call(dt=0, block=16) == 2
    assert call(ws=None) == 1
    assert call(ws=P(0x10010)) == 1          # not 256-byte aligned
    assert call(nws=one - 1) == 1
    assert "workspace" in _last(lib)


def test_binding_fails_loudly_without_cuda_tensors():
    import torch
    import block_sparse_long_stats_b200 as spa
    k = torch.zeros((1, 1, 64, 128), dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        spa.spa_block_stats(k, 64)


def test_decode_workload_fits_the_noalloc_scratch(lib):
    # The allocation-free decode keeps its split-KV partials in a fixed 8 MiB
    # device array; the decode workload (16 sequences, 32/8 heads, 131072 cached
    # tokens, d = 128, block 16) must stay within it whatever the split heuristic.
    f = lib.spa_decode_workspace_bytes
    f.argtypes = [ctypes.c_int] * 6
    f.restype = ctypes.c_size_t
    assert 0 < f(16, 32, 8, 131072, 128, 16) <= 8 << 20
