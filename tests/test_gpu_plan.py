"""GPU tests of how pa_decode plans its work, against the fp64 oracle.

Two planners exist: each CTA of the attention kernel deriving its own items
(no planning kernel), and a one-CTA planning kernel for problems that do not
fit the first (many sequences, many items per CTA, the fp32 path).  Both must
give the oracle's result.  The merge counters in the workspace must be back at
zero after every call, whatever the problem, so that one workspace serves
problems of any shape.
"""

import os
import subprocess
import sys

import numpy as np
import pytest

from oracle import c_oracle
from parity import DeviceCase, compare, out_f64
from workloads import build_workload, get_config, host_values

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
COUNTER_SLOTS = 16384          # merge counters every workspace reserves at byte 256


def _oracle(wl, vh):
    c = wl.cfg
    return c_oracle.decode(vh["q"], vh["key_cache"], vh["value_cache"], wl.block_tables, wl.context_lens, c.scale,
                           c.dtype, c.num_kv_heads)


def _run(case, ws, P):
    import torch

    import paged_kv_cache_362_b200 as pa

    wl, d = case.wl, case.dev
    c = wl.cfg
    out = torch.full_like(d["q"], float("nan"))
    pa.decode(out, d["q"], d["key_cache"], d["value_cache"], case.block_tables, case.context_lens, c.scale,
              wl.max_context_len, ws, partition_size=P, status=case.status)
    torch.cuda.synchronize()
    assert int(case.status.item()) == 0
    return out


def _problem(B, ctx_lo, ctx_hi, Hq=28, Hkv=4, D=64, dtype="f16", seed=0):
    rng = np.random.default_rng(seed)
    ctx = rng.integers(ctx_lo, ctx_hi + 1, size=B)
    nb = int(sum(-(-int(c) // 16) for c in ctx)) + 8
    cfg = get_config("qwen_layer", dtype=dtype, num_heads=Hq, num_kv_heads=Hkv, head_dim=D, num_blocks=nb,
                     ctx_kind="fixed", ctx_args=tuple(int(c) for c in ctx))
    wl = build_workload(cfg, seed=seed)
    vh = host_values(wl)
    return wl, vh


# (B, ctx range, P, dtype, D, what the sizes exercise)
CASES = [
    (250, 1, 256, 64, "f16", 64, "self-planning, 8 sequence chunks per key search"),
    (200, 1, 4000, 512, "bf16", 128, "self-planning, fused merge of up to 8 partitions"),
    (40, 1, 9000, 128, "bf16", 128, "self-planning, many partitions: reduce kernel"),
    (1000, 1, 256, 64, "f16", 64, "planning kernel: a large batch"),
    (2100, 1, 48, 16, "f16", 64, "planning kernel: more sequences than a CTA can plan in its ring"),
    (4200, 1, 64, 16, "f16", 64, "planning kernel: more (sequence, KV head) pairs than the fixed counters"),
]


@pytest.mark.parametrize("case_args", CASES, ids=[f"B={c[0]} P={c[3]}" for c in CASES])
def test_planners_match_oracle(case_args):
    import torch

    import paged_kv_cache_362_b200 as pa

    B, lo, hi, P, dtype, D, what = case_args
    wl, vh = _problem(B, lo, hi, D=D, dtype=dtype, seed=B)

    c = wl.cfg
    ws = pa.make_workspace(wl.num_seqs, c.num_heads, c.num_kv_heads, D, wl.max_context_len, P)
    case = DeviceCase(wl, vh)
    out = _run(case, ws, P)
    compare(out_f64(out), _oracle(wl, vh), dtype, what)
    ncnt = max(COUNTER_SLOTS, B * c.num_kv_heads)
    cnt = ws[256:256 + 4 * ncnt].view(torch.int32)
    assert int(cnt.abs().sum().item()) == 0, "merge counters not left at zero"


def test_one_workspace_for_problems_of_every_shape():
    """One buffer, sized for the largest problem, serves a series of different problems."""
    import torch

    import paged_kv_cache_362_b200 as pa

    probs = [(_problem(*a[:3], Hq=a[3], Hkv=a[4], D=a[5], dtype=a[6], seed=k), a[7])
             for k, a in enumerate([
                 (64, 100, 3000, 28, 4, 128, "f16", 512),     # fused merges
                 (900, 1, 700, 32, 8, 64, "bf16", 128),       # fused, more counters, other layout
                 (16, 5000, 9000, 28, 4, 128, "f16", 256),    # reduce kernel
                 (64, 100, 3000, 28, 4, 128, "f16", 512),     # first again
             ])]
    need = max(pa.decode_workspace_size(wl.num_seqs, wl.cfg.num_heads, wl.cfg.num_kv_heads, wl.cfg.head_dim,
                                        wl.max_context_len, P) for (wl, _), P in probs)
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    for k, ((wl, vh), P) in enumerate(probs):
        out = _run(DeviceCase(wl, vh), ws, P)
        compare(out_f64(out), _oracle(wl, vh), wl.cfg.dtype, f"problem {k}")
    assert int(ws[256:256 + 4 * COUNTER_SLOTS].view(torch.int32).abs().sum().item()) == 0


def test_launch_counts():
    import paged_kv_cache_362_b200 as pa

    # one partition, tensor cores: the attention kernel alone
    assert pa.decode_launch_count(256, 28, 4, 128, 512, 512, "f16") == 1
    # up to 8 partitions merged inside the attention kernel
    assert pa.decode_launch_count(256, 28, 4, 128, 4096, 512, "f16") == 1
    # 64 partitions: attention + reduce
    assert pa.decode_launch_count(8, 28, 4, 128, 32768, 512, "bf16") == 2
    # fp32 (SIMT path): planning kernel + attention + reduce
    assert pa.decode_launch_count(8, 28, 4, 128, 4096, 512, "f32") == 3
    # too many (sequence, KV head) pairs for the fixed counters: planning kernel too
    assert pa.decode_launch_count(8192, 32, 8, 64, 64, 16, "f16") == 2


@pytest.mark.parametrize("env", [
    {"PA_TEST_DECODE_TUNING": "planner=1"},       # the planning kernel writes the list
    {"PA_TEST_DECODE_TUNING": "order=1"},         # all items by size alone
    {"PA_TEST_DECODE_TUNING": "split=1"},         # partitions of near-equal length
    {"PA_TEST_DECODE_TUNING": "shape=paired"},    # 2 CTAs per SM, two consumer warps, 10-stage ring, reduce kernel
    {"PA_TEST_DECODE_TUNING": "shape=triple"},    # 3 CTAs per SM, 8-stage ring
    {"PA_TEST_DECODE_TUNING": "shape=pair1"},     # 2 CTAs per SM, 13-stage ring
], ids=lambda e: ",".join(f"{v}" for v in e.values()))
def test_scheduling_variants_in_subprocess(env):
    """The same parity cases under the library's scheduling alternatives and kernel shapes (pa_decode_tuned,
    set for the whole child test process), block sizes 8/16/32 with NaN in the unread slots included."""
    cmd = [sys.executable, "-m", "pytest", "-q", "-m", "gpu", "-p", "no:cacheprovider",
           os.path.join(ROOT, "tests", "test_gpu_decode.py"), os.path.join(ROOT, "tests", "test_gpu_plan.py"),
           os.path.join(ROOT, "tests", "test_gpu_block_sizes.py"),
           "-k", "(small_cases_every_element and (28x4 or 16x2)) or full_size_step_every_sequence or bitwise "
                 "or planners_match_oracle or one_workspace or (every_element_nan and (28x4 or 32x2)) "
                 "or long_contexts or bad_block_drops"]
    r = subprocess.run(cmd, cwd=ROOT, env=dict(os.environ, **env), capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-2000:]


# (B, ctx range, P, dtype, D, Hq, Hkv, what the sizes exercise)
PLANNED = [
    (250, 1, 256, 64, "f16", 64, 28, 4, "one partition per sequence"),
    (200, 1, 4000, 512, "bf16", 128, 28, 4, "fused merge of up to 8 partitions"),
    (40, 1, 9000, 128, "bf16", 128, 28, 4, "many partitions: reduce kernel"),
    (1000, 1, 256, 64, "f16", 64, 28, 4, "a large batch"),
    (64, 1, 2000, 0, "bf16", 128, 48, 2, "G = 24: the SIMT kernel"),
]


@pytest.mark.parametrize("planner", ["pa_decode_plan", "pa_decode"])
@pytest.mark.parametrize("case_args", PLANNED, ids=[f"B={c[0]} P={c[3]} G={c[6] // c[7]}" for c in PLANNED])
def test_plan_once_decode_every_layer(case_args, planner):
    """A plan made once, by pa_decode_plan or left by a pa_decode call, then pa_decode_planned over several
    layers' pools: each output equals pa_decode's on that pool bit for bit (the same kernels read the same list)
    and the oracle, and the merge counters end at zero after every call."""
    import torch

    import paged_kv_cache_362_b200 as pa
    from parity import to_host

    B, lo, hi, P, dtype, D, Hq, Hkv, what = case_args
    wl, vh = _problem(B, lo, hi, Hq=Hq, Hkv=Hkv, D=D, dtype=dtype, seed=B + 7)
    c = wl.cfg
    case = DeviceCase(wl, vh)
    d = case.dev
    ws = pa.make_workspace(wl.num_seqs, c.num_heads, c.num_kv_heads, D, wl.max_context_len, P)
    ws_ref = pa.make_workspace(wl.num_seqs, c.num_heads, c.num_kv_heads, D, wl.max_context_len, P)
    # a second layer: the same sequences and tables over other values (exact in the storage type)
    kc2, vc2 = -d["key_cache"], d["value_cache"].flip(-1).contiguous()
    layers = [(d["key_cache"], d["value_cache"]), (kc2, vc2), (d["key_cache"], d["value_cache"])]
    bs = d["key_cache"].shape[2]
    if planner == "pa_decode_plan":
        pa.decode_plan(case.block_tables, case.context_lens, c.num_heads, c.num_kv_heads, D, bs, wl.max_context_len,
                       ws, partition_size=P, status=case.status)
    else:   # a decode of another layer (other values) leaves the plan
        scratch = torch.empty_like(d["q"])
        pa.decode(scratch, d["q"], d["key_cache"].flip(-1).contiguous(), -d["value_cache"], case.block_tables,
                  case.context_lens, c.scale, wl.max_context_len, ws, partition_size=P, status=case.status)
    outs = []
    for k, (kc, vc) in enumerate(layers):
        out = torch.full_like(d["q"], float("nan"))
        pa.decode(out, d["q"], kc, vc, case.block_tables, case.context_lens, c.scale, wl.max_context_len, ws,
                  partition_size=P, status=case.status, planned=True)
        ref = torch.full_like(d["q"], float("nan"))
        pa.decode(ref, d["q"], kc, vc, case.block_tables, case.context_lens, c.scale, wl.max_context_len, ws_ref,
                  partition_size=P, status=case.status)
        torch.cuda.synchronize()
        assert int(case.status.item()) == 0
        assert torch.equal(out.view(torch.int16), ref.view(torch.int16)), f"{what}: layer {k} differs from pa_decode"
        ncnt = max(COUNTER_SLOTS, B * c.num_kv_heads)
        assert int(ws[256:256 + 4 * ncnt].view(torch.int32).abs().sum().item()) == 0, "merge counters not at zero"
        outs.append(out)
    compare(out_f64(outs[0]), _oracle(wl, vh), dtype, what + ", layer 0")
    vh2 = dict(vh, key_cache=to_host(kc2, dtype), value_cache=to_host(vc2, dtype))
    compare(out_f64(outs[1]), _oracle(wl, vh2), dtype, what + ", layer 1")


def test_planned_launch_counts():
    import paged_kv_cache_362_b200 as pa

    # the attention kernel alone, where pa_decode may add a planning kernel
    assert pa.decode_launch_count(256, 28, 4, 128, 4096, 512, "f16", planned=True) == 1
    assert pa.decode_launch_count(8192, 32, 8, 64, 64, 16, "f16", planned=True) == 1
    # attention + reduce
    assert pa.decode_launch_count(8, 28, 4, 128, 32768, 512, "bf16", planned=True) == 2
    # fp32 (SIMT path): attention + reduce, against planning kernel + attention + reduce
    assert pa.decode_launch_count(8, 28, 4, 128, 4096, 512, "f32", planned=True) == 2
