"""A decode loop driven by the host block manager, on the GPU, against the fp64 oracle.

Prompts are written with pa_reshape_and_cache through the manager's slot
mappings, sequences fork (a shared prefix ending inside a block), and every
decode step appends one token per sequence: the manager's copy-on-write pairs
go to pa_copy_blocks, the new tokens to pa_reshape_and_cache, its block tables
to pa_decode.  A host mirror of the pools follows the same steps with the
oracle's scatter and copy; the pools must stay bit-identical and every decode
must match the oracle.
"""

import numpy as np
import pytest

from oracle import c_oracle
from oracle import reference as R
from parity import compare, out_f64, to_device, to_host

pytestmark = pytest.mark.gpu


def test_decode_loop_with_forks_and_copy_on_write():
    import torch

    import paged_kv_cache_362_b200 as pa

    rng = np.random.default_rng(11)
    NB, Hkv, Hq, D, dt = 128, 4, 28, 128, "f16"
    scale = 1.0 / np.sqrt(D)
    bm = pa.BlockManager(NB, 16)
    shape = (NB, Hkv, 16, D)
    kc_h = rng.standard_normal(shape).astype(np.float16)
    vc_h = rng.standard_normal(shape).astype(np.float16)
    kc, vc = to_device(kc_h, dt), to_device(vc_h, dt)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")

    def write(slots, n):
        nonlocal kc_h, vc_h
        k = rng.standard_normal((n, Hkv, D)).astype(np.float16)
        v = rng.standard_normal((n, Hkv, D)).astype(np.float16)
        pa.reshape_and_cache(to_device(k, dt), to_device(v, dt), kc, vc,
                             torch.from_numpy(slots).cuda(), status=status)
        kc_h, vc_h = R.reshape_and_cache(k, v, kc_h, vc_h, slots)

    # prompts, then forks of sequence 0 (40 tokens: its third block is shared and partly filled)
    for sid, n in ((0, 40), (1, 100), (2, 17)):
        write(bm.add_sequence(sid, n), n)
    bm.fork(0, 3)
    bm.fork(0, 4)
    live = [0, 1, 2, 3, 4]
    ws = pa.make_workspace(len(live), Hq, Hkv, D, 4096)
    copies_seen = 0
    for step in range(4):
        slots, pairs = bm.append_tokens(live)
        copies_seen += len(pairs)
        if len(pairs):
            pa.copy_blocks(kc, vc, torch.from_numpy(np.ascontiguousarray(pairs)).cuda(), status=status)
            kc_h, vc_h = R.copy_blocks(kc_h, vc_h, pairs)
        write(slots, len(live))
        bt, cl = bm.block_tables(live, 64)
        q = rng.standard_normal((len(live), Hq, D)).astype(np.float16)
        out = torch.empty((len(live), Hq, D), dtype=torch.float16, device="cuda")
        pa.decode(out, to_device(q, dt), kc, vc, torch.from_numpy(bt).cuda(), torch.from_numpy(cl).cuda(), scale,
                  int(cl.max()), ws, status=status)
        torch.cuda.synchronize()
        ref = c_oracle.decode(q, kc_h, vc_h, bt, cl, scale, dt, Hkv)
        compare(out_f64(out), ref, dt, f"step {step}")
    assert int(status.item()) == 0
    # the forks' first appends cloned the shared partial block: one copy per fork, then none
    assert copies_seen == 2
    assert np.array_equal(to_host(kc, dt).view(np.uint16), kc_h.view(np.uint16))
    assert np.array_equal(to_host(vc, dt).view(np.uint16), vc_h.view(np.uint16))
    for sid in live:
        bm.free_sequence(sid)
    assert bm.num_free_blocks == NB


def test_swap_out_and_in_through_pinned_host_memory():
    """A request is evicted to pinned host pools, its device blocks are reused, it comes back intact."""
    import torch

    import paged_kv_cache_362_b200 as pa

    rng = np.random.default_rng(5)
    NB, NH, Hkv, Hq, D, dt = 64, 32, 4, 28, 128, "bf16"
    scale = 1.0 / np.sqrt(D)
    bm = pa.BlockManager(NB, 16, NH)
    shape = (NB, Hkv, 16, D)
    # N(0, 1) values as bf16 bit patterns (the top half of the fp32 bits)
    bits = lambda s: (rng.standard_normal(s).astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    kc_h, vc_h = bits(shape), bits(shape)
    kc, vc = to_device(kc_h, dt), to_device(vc_h, dt)
    hk = torch.empty((NH, Hkv, 16, D), dtype=torch.bfloat16).pin_memory()
    hv = torch.empty((NH, Hkv, 16, D), dtype=torch.bfloat16).pin_memory()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    for sid, n in ((1, 300), (2, 70)):
        bm.add_sequence(sid, n)
    bm.fork(1, 3)
    bm.append_tokens([3])                       # 3 clones 1's partial block: it owns that one, shares the rest
    bt0, cl0 = bm.block_tables([1, 2, 3], 32)
    q = bits((3, Hq, D))
    before = torch.empty((3, Hq, D), dtype=torch.bfloat16, device="cuda")
    ws = pa.make_workspace(3, Hq, Hkv, D, 512)
    q_d = to_device(q, dt)
    pa.decode(before, q_d, kc, vc, torch.from_numpy(bt0).cuda(), torch.from_numpy(cl0).cuda(), scale, 512, ws)
    # evict 1 and 2; their private blocks go to the host pools
    moved = {}
    for sid in (1, 2):
        pairs = bm.swap_out(sid)
        moved[sid] = pairs
        pa.swap_blocks(kc, vc, hk, hv, torch.from_numpy(pairs).cuda(), status=status)
    torch.cuda.synchronize()
    for sid, pairs in moved.items():
        for d, h in pairs.tolist():
            assert np.array_equal(hk[h].view(torch.int16).numpy().view(np.uint16), kc_h[d])
            assert np.array_equal(hv[h].view(torch.int16).numpy().view(np.uint16), vc_h[d])
    # 1's shared blocks stayed for 3; the freed blocks are overwritten by a new request
    assert len(moved[1]) < bm.sequence_blocks(1)
    slots = bm.add_sequence(9, 16 * bm.num_free_blocks)
    junk = torch.zeros((len(slots), Hkv, D), dtype=torch.bfloat16, device="cuda")
    pa.reshape_and_cache(junk, junk, kc, vc, torch.from_numpy(slots).cuda(), status=status)
    bm.free_sequence(9)
    # bring them back (pinned pairs this time) and decode again: the same bits as before the eviction
    for sid in (1, 2):
        pairs = torch.from_numpy(bm.swap_in(sid)).pin_memory()
        pa.swap_blocks(hk, hv, kc, vc, pairs, status=status)
    bt1, cl1 = bm.block_tables([1, 2, 3], 32)
    after = torch.empty_like(before)
    pa.decode(after, q_d, kc, vc, torch.from_numpy(bt1).cuda(), torch.from_numpy(cl1).cuda(), scale, 512, ws)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert torch.equal(before.view(torch.int16), after.view(torch.int16))
    # and the result is the oracle's on the original pools through the original tables
    ref = c_oracle.decode(q, kc_h, vc_h, bt0, cl0, scale, dt, Hkv)
    compare(out_f64(after), ref, dt, "after swap round trip")
