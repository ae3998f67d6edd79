"""GPU parity of the cache write and the copy-on-write block copy: bit-exact against the oracle."""

import numpy as np
import pytest

from oracle import reference as R
from parity import DeviceCase, to_host
from workloads import build_workload, get_config, host_values

pytestmark = pytest.mark.gpu


def _pa():
    import paged_kv_cache_362_b200 as pa
    return pa


CASES = [("f32", 64, 2), ("f32", 128, 4), ("f16", 64, 1), ("f16", 128, 4), ("bf16", 64, 2), ("bf16", 128, 8)]


@pytest.mark.parametrize("dtype,D,Hkv", CASES)
def test_reshape_and_cache_bit_exact(dtype, D, Hkv):
    import torch

    cfg = get_config("tiny", dtype=dtype, head_dim=D, num_kv_heads=Hkv, num_heads=Hkv * 2, num_blocks=96,
                     ctx_kind="fixed", ctx_args=(1, 15, 16, 17, 37, 200, 512, 33))
    wl = build_workload(cfg, seed=11, pad_tokens=5)
    vh = host_values(wl)
    case = DeviceCase(wl, vh)
    pa = _pa()
    d = case.dev
    pa.reshape_and_cache(d["key"], d["value"], d["key_cache"], d["value_cache"], case.slot_mapping,
                         status=case.status)
    torch.cuda.synchronize()
    kc, vc = R.reshape_and_cache(vh["key"], vh["value"], vh["key_cache"], vh["value_cache"], wl.slot_mapping)
    assert np.array_equal(R.bits_view(to_host(d["key_cache"], dtype)), R.bits_view(kc))
    assert np.array_equal(R.bits_view(to_host(d["value_cache"], dtype)), R.bits_view(vc))
    assert int(case.status.item()) == 0


def test_reshape_and_cache_out_of_range_slot_is_skipped_and_flagged():
    import torch

    cfg = get_config("tiny", dtype="f16", head_dim=128)
    wl = build_workload(cfg, seed=2)
    vh = host_values(wl)
    wl.slot_mapping[1] = wl.num_blocks * 16 + 3      # past the pool
    wl.slot_mapping[2] = -7                           # padding
    case = DeviceCase(wl, vh)
    pa = _pa()
    d = case.dev
    pa.reshape_and_cache(d["key"], d["value"], d["key_cache"], d["value_cache"], case.slot_mapping,
                         status=case.status)
    torch.cuda.synchronize()
    assert int(case.status.item()) & pa.PA_ERR_OUT_OF_RANGE
    ok = wl.slot_mapping.copy()
    ok[1] = -1
    kc, vc = R.reshape_and_cache(vh["key"], vh["value"], vh["key_cache"], vh["value_cache"], ok)
    assert np.array_equal(R.bits_view(to_host(d["key_cache"], "f16")), R.bits_view(kc))
    assert np.array_equal(R.bits_view(to_host(d["value_cache"], "f16")), R.bits_view(vc))


@pytest.mark.parametrize("dtype,D,Hkv", CASES)
def test_copy_blocks_bit_exact(dtype, D, Hkv):
    import torch

    cfg = get_config("tiny", dtype=dtype, head_dim=D, num_kv_heads=Hkv, num_heads=Hkv, num_blocks=40)
    wl = build_workload(cfg, seed=4)
    vh = host_values(wl)
    pairs = np.array([[1, 3], [1, 0], [5, 39], [7, 8], [20, 21]], dtype=np.int64)
    case = DeviceCase(wl, vh)
    pa = _pa()
    pa.check_copy_pairs(pairs, wl.num_blocks)
    d = case.dev
    pa.copy_blocks(d["key_cache"], d["value_cache"], torch.from_numpy(pairs).cuda(), status=case.status)
    torch.cuda.synchronize()
    kc, vc = R.copy_blocks(vh["key_cache"], vh["value_cache"], pairs)
    assert np.array_equal(R.bits_view(to_host(d["key_cache"], dtype)), R.bits_view(kc))
    assert np.array_equal(R.bits_view(to_host(d["value_cache"], dtype)), R.bits_view(vc))
    assert int(case.status.item()) == 0


def test_copy_blocks_out_of_range_pair_is_skipped_and_flagged():
    import torch

    cfg = get_config("tiny", dtype="bf16", head_dim=64)
    wl = build_workload(cfg, seed=6)
    vh = host_values(wl)
    pairs = np.array([[2, 4], [32, 5], [6, -1], [9, 10]], dtype=np.int64)
    case = DeviceCase(wl, vh)
    pa = _pa()
    d = case.dev
    pa.copy_blocks(d["key_cache"], d["value_cache"], torch.from_numpy(pairs).cuda(), status=case.status)
    torch.cuda.synchronize()
    assert int(case.status.item()) & pa.PA_ERR_OUT_OF_RANGE
    kc, vc = R.copy_blocks(vh["key_cache"], vh["value_cache"], pairs[[0, 3]])
    assert np.array_equal(R.bits_view(to_host(d["key_cache"], "bf16")), R.bits_view(kc))
    assert np.array_equal(R.bits_view(to_host(d["value_cache"], "bf16")), R.bits_view(vc))


def test_full_size_churned256_write():
    """256 appended tokens into the fragmented 80,000-block pool: exactly the addressed rows change."""
    import torch

    wl = build_workload(get_config("churned256"), seed=0)
    case = DeviceCase(wl, device_draw=True)
    pa = _pa()
    d = case.dev
    kb, vb = d["key_cache"].clone(), d["value_cache"].clone()
    pa.reshape_and_cache(d["key"], d["value"], d["key_cache"], d["value_cache"], case.slot_mapping,
                         status=case.status)
    torch.cuda.synchronize()
    assert int(case.status.item()) == 0
    s = case.slot_mapping
    blk, off = s // 16, s % 16
    for pool, before, src in ((d["key_cache"], kb, d["key"]), (d["value_cache"], vb, d["value"])):
        assert torch.equal(pool[blk, :, off, :].view(torch.int16), src.view(torch.int16))
        changed = (pool.view(torch.int16) != before.view(torch.int16)).any(dim=-1).nonzero()
        written = set((int(b), int(o)) for b, o in zip(blk.tolist(), off.tolist()))
        assert all((int(b), int(o)) in written for b, _, o in changed.tolist())


def test_full_size_shared_prefix_copy():
    """The 64 copy-on-write clones of the shared partial block, in the full-size pool."""
    import torch

    wl = build_workload(get_config("shared_prefix"), seed=0)
    case = DeviceCase(wl, device_draw=True)
    pa = _pa()
    pa.check_copy_pairs(wl.copy_pairs, wl.num_blocks)
    d = case.dev
    kb, vb = d["key_cache"].clone(), d["value_cache"].clone()
    pa.copy_blocks(d["key_cache"], d["value_cache"], case.copy_pairs, status=case.status)
    torch.cuda.synchronize()
    assert int(case.status.item()) == 0
    src, dst = case.copy_pairs[:, 0], case.copy_pairs[:, 1]
    for pool, before in ((d["key_cache"], kb), (d["value_cache"], vb)):
        assert torch.equal(pool[dst].view(torch.int16), before[src].view(torch.int16))
        mask = torch.ones(pool.shape[0], dtype=torch.bool, device=pool.device)
        mask[dst] = False
        assert torch.equal(pool[mask].view(torch.int16), before[mask].view(torch.int16))
