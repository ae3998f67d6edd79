"""GPU parity of paged decode attention against the fp64 oracle.

Small cases compare every output element; full-size workloads compare every
head of a sample of sequences (the longest, the shortest, copy-on-write forks
and seeded picks) in the launch configuration the benchmark times.
"""

import numpy as np
import pytest

import parity
from oracle import c_oracle
from oracle import reference as R
from parity import abs_values, sharp_check, DeviceCase, compare, oracle_step, out_f64
from workloads import build_workload, get_config, host_values

pytestmark = pytest.mark.gpu


def _pa():
    import paged_kv_cache_362_b200 as pa
    return pa


def _decode(case, partition_size=0, out=None, max_ctx=None):
    import torch

    pa = _pa()
    wl, d = case.wl, case.dev
    c = wl.cfg
    max_ctx = wl.max_context_len if max_ctx is None else max_ctx
    ws = pa.make_workspace(wl.num_seqs, c.num_heads, c.num_kv_heads, c.head_dim, max_ctx, partition_size)
    out = torch.empty_like(d["q"]) if out is None else out
    pa.decode(out, d["q"], d["key_cache"], d["value_cache"], case.block_tables, case.context_lens, c.scale,
              max_ctx, ws, partition_size=partition_size, status=case.status)
    torch.cuda.synchronize()
    return out


def _oracle_full(wl, vh):
    c = wl.cfg
    return c_oracle.decode(vh["q"], vh["key_cache"], vh["value_cache"], wl.block_tables, wl.context_lens, c.scale,
                           c.dtype, c.num_kv_heads)


def test_tiny_config_fp32():
    wl = build_workload(get_config("tiny"), seed=0)
    vh = host_values(wl)
    case = DeviceCase(wl, vh)
    pa = _pa()
    d = case.dev
    pa.reshape_and_cache(d["key"], d["value"], d["key_cache"], d["value_cache"], case.slot_mapping)
    out = _decode(case)
    kc, vc = R.reshape_and_cache(vh["key"], vh["value"], vh["key_cache"], vh["value_cache"], wl.slot_mapping)
    c = wl.cfg
    ref = R.decode(vh["q"], kc, vc, wl.block_tables, wl.context_lens, c.scale, c.dtype, c.num_kv_heads)
    compare(out_f64(out), ref, "f32", "tiny")
    assert int(case.status.item()) == 0


EDGE_CTX = (0, 1, 15, 16, 17, 31, 33, 100, 511, 512, 513, 700)
SHAPES = [(28, 4), (8, 8), (16, 2), (32, 2), (48, 2)]   # G = 7, 1, 8, 16 (two n-tiles), 24 (SIMT)


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
@pytest.mark.parametrize("heads", SHAPES, ids=lambda h: f"{h[0]}x{h[1]}")
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("P", [16, 64, 512, 0])
def test_small_cases_every_element(dtype, heads, D, P):
    Hq, Hkv = heads
    cfg = get_config("qwen_layer", dtype=dtype, num_heads=Hq, num_kv_heads=Hkv, head_dim=D, num_blocks=160,
                     ctx_kind="fixed", ctx_args=EDGE_CTX)
    wl = build_workload(cfg, seed=D + Hq + P)
    vh = host_values(wl)
    case = DeviceCase(wl, vh)
    out = _decode(case, partition_size=P)
    compare(out_f64(out), _oracle_full(wl, vh), dtype, f"{dtype} {heads} D={D} P={P}")
    assert int(case.status.item()) == 0


@pytest.mark.parametrize("dtype", ["f32", "f16", "bf16"])
def test_fp32_and_simt_paths_long_context(dtype):
    cfg = get_config("qwen_layer", dtype=dtype, num_heads=12, num_kv_heads=4, head_dim=64, num_blocks=400,
                     ctx_kind="fixed", ctx_args=(1500, 3, 4000, 700))
    wl = build_workload(cfg, seed=5)
    vh = host_values(wl)
    case = DeviceCase(wl, vh)
    out = _decode(case, partition_size=256)
    compare(out_f64(out), _oracle_full(wl, vh), dtype, f"{dtype} long")


def test_output_independent_of_physical_placement():
    """Same logical K/V at different physical blocks: bitwise identical output."""
    import torch

    cfg = get_config("qwen_layer", dtype="bf16", num_blocks=600, ctx_kind="fixed",
                     ctx_args=(5, 300, 1024, 2000, 17))
    wl = build_workload(cfg, seed=1)
    vh = host_values(wl)
    a = _decode(DeviceCase(wl, vh))
    perm = np.random.default_rng(9).permutation(cfg.num_blocks)
    kc2 = np.empty_like(vh["key_cache"])
    vc2 = np.empty_like(vh["value_cache"])
    kc2[perm] = vh["key_cache"]
    vc2[perm] = vh["value_cache"]
    bt2 = np.where(wl.block_tables >= 0, perm[np.maximum(wl.block_tables, 0)], -1).astype(np.int32)
    wl2 = build_workload(cfg, seed=1)
    wl2.block_tables = bt2
    vh2 = dict(vh, key_cache=kc2, value_cache=vc2)
    b = _decode(DeviceCase(wl2, vh2))
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_repeat_runs_bitwise_identical():
    import torch

    wl = build_workload(get_config("churned256"), seed=3, num_seqs=64)
    case = DeviceCase(wl, device_draw=True)
    a = _decode(case)
    b = _decode(case)
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_bad_block_id_flagged_and_skipped():
    """An out-of-pool block id sets the status bit; that block contributes nothing, the rest is exact."""
    cfg = get_config("qwen_layer", dtype="f16", num_blocks=64, ctx_kind="fixed", ctx_args=(40, 100))
    wl = build_workload(cfg, seed=2)
    vh = host_values(wl)
    wl.block_tables[1, 2] = 5000
    case = DeviceCase(wl, vh)
    out = out_f64(_decode(case, partition_size=64))
    pa = _pa()
    assert int(case.status.item()) & pa.PA_ERR_OUT_OF_RANGE
    c = wl.cfg
    ref0 = c_oracle.decode(vh["q"][:1], vh["key_cache"], vh["value_cache"], wl.block_tables[:1],
                           wl.context_lens[:1], c.scale, c.dtype, c.num_kv_heads)
    compare(out[:1], ref0, "f16", "unaffected sequence")
    # sequence 1 without the bad block's 16 tokens: rebuild it as the oracle's own case
    keep = [j for j in range(7) if j != 2]
    toks = [i for j in keep for i in range(16 * j, min(16 * j + 16, 100))]
    kv = lambda pool: np.stack([pool[wl.block_tables[1, i // 16], :, i % 16] for i in toks], axis=1)
    K, V = kv(vh["key_cache"]), kv(vh["value_cache"])
    G = c.num_heads // c.num_kv_heads
    ref1 = np.stack([R.attention_f64(vh["q"][1, h].astype(np.float64), K[h // G].astype(np.float64),
                                     V[h // G].astype(np.float64), c.scale) for h in range(c.num_heads)])
    compare(out[1], ref1, "f16", "sequence with the bad block")


def test_context_above_bound_is_clamped_and_flagged():
    cfg = get_config("qwen_layer", dtype="f16", num_blocks=64, ctx_kind="fixed", ctx_args=(40, 100))
    wl = build_workload(cfg, seed=8)
    vh = host_values(wl)
    case = DeviceCase(wl, vh)
    out = out_f64(_decode(case, max_ctx=64))        # context 100 > 64
    pa = _pa()
    assert int(case.status.item()) & pa.PA_ERR_OUT_OF_RANGE
    wl.context_lens[1] = 64
    compare(out, _oracle_full(wl, vh), "f16", "clamped")


def _seq_sample(wl, n=12, seed=0):
    rng = np.random.default_rng(seed)
    cl = wl.context_lens
    pick = {int(np.argmax(cl)), int(np.argmin(cl))}
    if wl.copy_pairs.size:
        pick.update(range(wl.num_seqs - 3, wl.num_seqs))          # copy-on-write forks
    while len(pick) < min(n, wl.num_seqs):
        pick.add(int(rng.integers(0, wl.num_seqs)))
    return sorted(pick)


@pytest.mark.parametrize("name", ["qwen_layer", "long32k", "churned256", "shared_prefix"])
def test_full_size_step_every_sequence(name):
    """One whole step at full size (copy-on-write, append, decode): every (sequence, head) output element against
    the oracle, with the tolerance and with the sharper check against the oracle rounded to the storage dtype."""
    import torch

    pa = _pa()
    wl = build_workload(get_config(name), seed=0)
    case = DeviceCase(wl, device_draw=True)
    seqs = list(range(wl.num_seqs))
    sub = case.host_subproblem(seqs)                      # pre-step host copy
    d = case.dev
    if wl.copy_pairs.size:
        pa.copy_blocks(d["key_cache"], d["value_cache"], case.copy_pairs, status=case.status)
    pa.reshape_and_cache(d["key"], d["value"], d["key_cache"], d["value_cache"], case.slot_mapping,
                         status=case.status)
    out = _decode(case, partition_size=wl.cfg.partition_size)
    assert int(case.status.item()) == 0
    del case, d
    ref = oracle_step(sub, wl.cfg)
    ref_absv = None
    if wl.cfg.dtype == "f16":
        # the same attention weights applied to |V|: the scale of the P-rounding bound
        sub_abs = dict(sub, value_cache=abs_values(sub["value_cache"], "f16"), value=abs_values(sub["value"], "f16"))
        ref_absv = oracle_step(sub_abs, wl.cfg)
        del sub_abs
    del sub
    mabs, mrel = compare(out_f64(out), ref, wl.cfg.dtype, name)
    stats = sharp_check(out, ref, wl.cfg.dtype, ref_absv, name)
    print(f"{name}: {wl.num_seqs} sequences, max abs {mabs:.2e}, max rel {mrel:.2e}, {stats}")
    torch.cuda.synchronize()


def test_extreme_sizes():
    """The largest shapes the workspace and grids see: one 262,144-token context (512 partitions,
    reduce kernel) and 8,192 short sequences (planning kernel, counters beyond the fixed region)."""
    import torch

    pa = _pa()
    # one very long sequence, MQA group of 8
    cfg = get_config("qwen_layer", dtype="bf16", num_heads=8, num_kv_heads=1, head_dim=128, num_blocks=16400,
                     ctx_kind="fixed", ctx_args=(262144,))
    wl = build_workload(cfg, seed=21)
    case = DeviceCase(wl, device_draw=True)
    sub = case.host_subproblem([0])
    out = _decode(case, partition_size=512)
    assert int(case.status.item()) == 0
    compare(out_f64(out), oracle_step(sub, cfg, do_copy=False, do_write=False), "bf16", "262144 tokens")
    del case
    torch.cuda.empty_cache()
    # many short sequences
    cfg = get_config("qwen_layer", dtype="f16", num_blocks=8192 * 3 + 8, ctx_kind="uniform", ctx_args=(1, 40))
    wl = build_workload(cfg, seed=22, num_seqs=8192)
    case = DeviceCase(wl, device_draw=True)
    seqs = _seq_sample(wl, n=24, seed=3)
    sub = case.host_subproblem(seqs)
    out = _decode(case, partition_size=16)
    assert int(case.status.item()) == 0
    compare(out_f64(out)[seqs], oracle_step(sub, cfg, do_copy=False, do_write=False), "f16", "8192 sequences")
