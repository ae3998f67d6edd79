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
