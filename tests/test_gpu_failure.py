"""The attention kernel's bounded waits, made to run out on purpose, without a GPU fault.

Every wait inside the decode attention kernel is bounded (2 s by default).  On
expiry the kernel sets PA_ERR_TIMEOUT in the caller's status word, lets the
copies it already issued land, and returns, so the context stays usable.  To
reach that path, the test uses the fault-path hooks of pa_decode_tuned
(include/pa_tuning.h): CTA 0 never publishes its first work item, so the
waits on it can only end through their bound (here 20 ms).  Nothing faults,
traps or spins without a limit.  The test checks that:
  * the call returns (every CTA ended) well within a few wait limits,
  * the status word carries PA_ERR_TIMEOUT,
  * the device still answers,
  * the next call, on a workspace zeroed again, matches the fp64 oracle.
It covers the single-warp shape (fused in-kernel merge) and the two-warp shape
(merge buffers in shared memory, then the reduce kernel).
"""

import time

import numpy as np
import pytest

from oracle import c_oracle
from parity import DeviceCase, compare, out_f64
from workloads import build_workload, get_config, host_values

pytestmark = pytest.mark.gpu

LIMIT_NS = 20_000_000   # 20 ms per wait


def _case(seed):
    cfg = get_config("qwen_layer", dtype="f16", num_blocks=600, ctx_kind="fixed",
                     ctx_args=(1500, 300, 17, 2048, 777, 64, 1200, 905))
    wl = build_workload(cfg, seed=seed)
    vh = host_values(wl)
    return wl, vh, DeviceCase(wl, vh)


def _decode(pa, case, ws, status, tuning, P=256):
    import torch

    wl, d = case.wl, case.dev
    c = wl.cfg
    out = torch.zeros_like(d["q"])
    pa.decode(out, d["q"], d["key_cache"], d["value_cache"], case.block_tables, case.context_lens, c.scale,
              wl.max_context_len, ws, partition_size=P, status=status, tuning=tuning)
    return out


@pytest.mark.parametrize("shape", ["quad", "paired"])
def test_expired_wait_reports_timeout_and_the_device_recovers(shape):
    import torch

    import paged_kv_cache_362_b200 as pa

    wl, vh, case = _case(seed=3)
    c = wl.cfg
    ws = pa.make_workspace(wl.num_seqs, c.num_heads, c.num_kv_heads, c.head_dim, wl.max_context_len, 256)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    ref = c_oracle.decode(vh["q"], vh["key_cache"], vh["value_cache"], wl.block_tables, wl.context_lens, c.scale,
                          c.dtype, c.num_kv_heads)

    # a short limit alone changes nothing: no wait of a healthy call comes near 20 ms
    out = _decode(pa, case, ws, status, pa.tuning(shape=shape, wait_limit_ns=LIMIT_NS))
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    compare(out_f64(out), ref, c.dtype, f"{shape}, short wait limit")

    # CTA 0 never publishes its first item: its waits run out
    torch.cuda.synchronize()
    t0 = time.monotonic()
    _decode(pa, case, ws, status, pa.tuning(shape=shape, wait_limit_ns=LIMIT_NS, stall_first_item=1))
    torch.cuda.synchronize()
    elapsed = time.monotonic() - t0
    st = int(status.item())
    assert st & pa.PA_ERR_TIMEOUT, f"status {st}"
    assert elapsed < 5.0, f"the stalled call took {elapsed:.2f} s"

    # the device still answers
    x = torch.arange(1 << 20, device="cuda", dtype=torch.float32)
    assert float(x.sum().item()) == float(np.arange(1 << 20, dtype=np.float64).sum())

    # after a timeout the workspace is zeroed again; then the call is whole
    ws.zero_()
    status.zero_()
    out = _decode(pa, case, ws, status, None)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    compare(out_f64(out), ref, c.dtype, f"{shape}, after the timeout")


def test_tuning_values_out_of_range_are_rejected():
    import paged_kv_cache_362_b200 as pa

    wl, vh, case = _case(seed=4)
    c = wl.cfg
    ws = pa.make_workspace(wl.num_seqs, c.num_heads, c.num_kv_heads, c.head_dim, wl.max_context_len, 256)
    for bad in (pa.tuning(shape=9), pa.tuning(planner=2), pa.tuning(wait_limit_ns=-1), pa.tuning(stall_first_item=3)):
        with pytest.raises(pa.PagedAttentionError) as e:
            _decode(pa, case, ws, None, bad)
        assert e.value.code == pa.PA_ERR_INVALID_ARG
