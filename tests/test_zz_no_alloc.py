"""pa_decode_noalloc: the decode entry point for callers that cannot allocate device memory.

Such callers (an extension inside an engine that owns all device memory, or a
loop that must not call cudaMalloc) get their scratch from a fixed array in
the library.  The test calls the entry point through the C ABI and checks its
output against pa_decode with a caller workspace, on two calls in a row with
different problems, so that whatever the first call left in the shared
scratch cannot leak into the second.  It sits in its own file, collected
last, and depends on nothing the other tests leave behind.
"""

import ctypes

import numpy as np
import pytest

import parity
from parity import DeviceCase, compare, out_f64
from workloads import build_workload, get_config, host_values

pytestmark = pytest.mark.gpu

P = ctypes.c_void_p
STATIC_SCRATCH_BYTES = 32 << 20


def _lib():
    import paged_kv_cache_362_b200 as pa

    lib = pa._lib.LIB
    f = lib.pa_decode_noalloc
    i32 = ctypes.c_int32
    f.argtypes = [P, P, P, P, P, i32, P, i32, i32, i32, i32, i32, i32, ctypes.c_float, i32, i32, ctypes.c_int, P, P]
    f.restype = ctypes.c_int
    return pa, f


def _noalloc(case, partition_size):
    import torch

    pa, f = _lib()
    wl, d = case.wl, case.dev
    c = wl.cfg
    out = torch.full_like(d["q"], float("nan"))
    dt = {"f32": 0, "f16": 1, "bf16": 2}[c.dtype]
    rc = f(P(out.data_ptr()), P(d["q"].data_ptr()), P(d["key_cache"].data_ptr()), P(d["value_cache"].data_ptr()),
           P(case.block_tables.data_ptr()), wl.block_tables.shape[1], P(case.context_lens.data_ptr()), wl.num_seqs,
           c.num_heads, c.num_kv_heads, c.head_dim, 16, wl.num_blocks, c.scale, wl.max_context_len, partition_size,
           dt, P(case.status.data_ptr()), P(torch.cuda.current_stream().cuda_stream))
    assert rc == 0, pa.error_string(rc)
    return out


def _with_workspace(case, partition_size):
    import torch

    pa, _ = _lib()
    wl, d = case.wl, case.dev
    c = wl.cfg
    out = torch.empty_like(d["q"])
    ws = pa.make_workspace(wl.num_seqs, c.num_heads, c.num_kv_heads, c.head_dim, wl.max_context_len, partition_size)
    pa.decode(out, d["q"], d["key_cache"], d["value_cache"], case.block_tables, case.context_lens, c.scale,
              wl.max_context_len, ws, partition_size=partition_size)
    return out


def test_noalloc_matches_workspace_decode_two_calls_in_a_row():
    import torch

    cases = [
        (get_config("qwen_layer", dtype="bf16", num_blocks=900, ctx_kind="fixed",
                    ctx_args=(4000, 17, 1, 2500, 600, 0, 5000)), 256),
        (get_config("qwen_layer", dtype="f16", num_heads=32, num_kv_heads=8, head_dim=64, num_blocks=300,
                    ctx_kind="fixed", ctx_args=(33, 700, 1024, 16, 300)), 0),
    ]
    for k, (cfg, P_) in enumerate(cases):
        wl = build_workload(cfg, seed=40 + k)
        vh = host_values(wl)
        case = DeviceCase(wl, vh)
        got = _noalloc(case, P_)
        ref = _with_workspace(case, P_)
        torch.cuda.synchronize()
        assert int(case.status.item()) == 0
        # same kernels, same inputs: identical bits; and both within tolerance of the oracle
        assert torch.equal(got.view(torch.int16), ref.view(torch.int16)), f"call {k}"
        c = wl.cfg
        oracle = parity.c_oracle.decode(vh["q"], vh["key_cache"], vh["value_cache"], wl.block_tables,
                                        wl.context_lens, c.scale, c.dtype, c.num_kv_heads)
        compare(out_f64(got), oracle, c.dtype, f"noalloc call {k}")


def test_noalloc_fused_merge_two_calls_in_a_row():
    """Two problems of different shape whose long sequences split into 2 to 8 partitions, which the attention
    kernel merges itself through per-(sequence, KV head) counters kept in the shared scratch: one launch per call
    (checked), so the second call only gives the right bits if the first left those counters at zero."""
    import torch

    pa, _ = _lib()
    cases = [
        (get_config("qwen_layer", dtype="f16", num_blocks=700, ctx_kind="fixed",
                    ctx_args=(2048, 700, 1500, 33, 1025, 256, 1800)), 256),
        (get_config("qwen_layer", dtype="bf16", num_heads=16, num_kv_heads=2, num_blocks=600, ctx_kind="fixed",
                    ctx_args=(1900, 512, 1300, 17, 2000)), 256),
    ]
    for k, (cfg, P_) in enumerate(cases):
        wl = build_workload(cfg, seed=60 + k)
        c = wl.cfg
        parts = -(-wl.max_context_len // P_)
        assert 2 <= parts <= 8
        assert pa.decode_launch_count(wl.num_seqs, c.num_heads, c.num_kv_heads, c.head_dim, wl.max_context_len, P_,
                                      c.dtype) == 1
        vh = host_values(wl)
        case = DeviceCase(wl, vh)
        got = _noalloc(case, P_)
        ref = _with_workspace(case, P_)   # a fresh, zeroed workspace
        torch.cuda.synchronize()
        assert int(case.status.item()) == 0
        assert torch.equal(got.view(torch.int16), ref.view(torch.int16)), f"fused call {k}"
        oracle = parity.c_oracle.decode(vh["q"], vh["key_cache"], vh["value_cache"], wl.block_tables,
                                        wl.context_lens, c.scale, c.dtype, c.num_kv_heads)
        compare(out_f64(got), oracle, c.dtype, f"noalloc fused call {k}")


def test_noalloc_rejects_problems_beyond_the_fixed_scratch():
    pa, f = _lib()
    # 1024 sequences x 28 heads x 64 partitions x (128 + 2) floats is far above 32 MiB
    need = pa.decode_workspace_size(1024, 28, 4, 128, 32768, 512)
    assert need > STATIC_SCRATCH_BYTES
    fake = P(0x100000)
    rc = f(fake, fake, fake, fake, fake, 2048, fake, 1024, 28, 4, 128, 16, 40000, 0.088, 32768, 512, 2, None, None)
    assert rc == pa.PA_ERR_UNSUPPORTED
    assert np.isfinite(need)
