"""Block sizes 8, 16 and 32, on pools whose unread slots hold NaN, against the fp64 oracle.

The pages call the block size a trade-off: smaller blocks waste fewer slots in
a sequence's last block, larger ones mean shorter tables and fewer, larger
reads; 16 is the default ("PagedAttention" digest, "Misconceptions").  The
kernels step through 16-token tiles whatever the block size: a tile is one
block, two 8-token blocks or half a 32-token block.  These tests run the
edge lengths around both block boundaries and tile boundaries.

Every pool here has NaN in each slot that no sequence reads -- the tail of a
sequence's last block, blocks no table names -- as a fresh allocation may: the
oracle never reads them, and neither must any result of the kernels.
"""

import numpy as np
import pytest

from oracle import c_oracle
from oracle import reference as R
from parity import DeviceCase, compare, oracle_step, out_f64, to_device, to_host
from workloads import build_workload, get_config, host_values, poison_unread_slots

pytestmark = pytest.mark.gpu

BS_CTX = (0, 1, 7, 8, 9, 15, 16, 17, 24, 25, 31, 32, 33, 40, 100, 511, 512, 513, 700)
SHAPES = [(28, 4), (8, 8), (32, 2), (48, 2)]   # G = 7, 1, 16 (two n-tiles), 24 (SIMT)


def _pa():
    import paged_kv_cache_362_b200 as pa
    return pa


def _cfg(bs, dtype, Hq, Hkv, D, ctx=BS_CTX, name="qwen_layer", extra=64):
    need = sum(-(-c // bs) for c in ctx)
    return get_config(name, dtype=dtype, num_heads=Hq, num_kv_heads=Hkv, head_dim=D, block_size=bs,
                      num_blocks=need + extra, ctx_kind="fixed", ctx_args=tuple(ctx), partition_size=0)


def _decode(case, P=0):
    import torch

    pa = _pa()
    wl, d = case.wl, case.dev
    c = wl.cfg
    ws = pa.make_workspace(wl.num_seqs, c.num_heads, c.num_kv_heads, c.head_dim, wl.max_context_len, P)
    out = torch.empty_like(d["q"])
    pa.decode(out, d["q"], d["key_cache"], d["value_cache"], case.block_tables, case.context_lens, c.scale,
              wl.max_context_len, ws, partition_size=P, status=case.status)
    torch.cuda.synchronize()
    return out


def _oracle(wl, vh):
    c = wl.cfg
    return c_oracle.decode(vh["q"], vh["key_cache"], vh["value_cache"], wl.block_tables, wl.context_lens, c.scale,
                           c.dtype, c.num_kv_heads)


def _poisoned_case(cfg, seed):
    wl = build_workload(cfg, seed=seed)
    vh = host_values(wl)
    n = poison_unread_slots(wl, vh)
    assert n > 0
    return wl, vh, DeviceCase(wl, vh)


@pytest.mark.parametrize("bs", [8, 16, 32])
@pytest.mark.parametrize("dtype", ["f16", "bf16"])
@pytest.mark.parametrize("heads", SHAPES, ids=lambda h: f"{h[0]}x{h[1]}")
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("P", [16, 0])
def test_every_element_nan_in_unread_slots(bs, dtype, heads, D, P):
    Hq, Hkv = heads
    wl, vh, case = _poisoned_case(_cfg(bs, dtype, Hq, Hkv, D), seed=bs + D + Hq + P)
    out = _decode(case, P)
    assert int(case.status.item()) == 0
    compare(out_f64(out), _oracle(wl, vh), dtype, f"bs={bs} {dtype} {heads} D={D} P={P}")


@pytest.mark.parametrize("bs", [8, 16, 32])
@pytest.mark.parametrize("heads,D", [((4, 2), 64), ((8, 8), 128)])
@pytest.mark.parametrize("P", [16, 0])
def test_fp32_nan_in_unread_slots(bs, heads, D, P):
    Hq, Hkv = heads
    wl, vh, case = _poisoned_case(_cfg(bs, "f32", Hq, Hkv, D), seed=3 * bs + P)
    out = _decode(case, P)
    assert int(case.status.item()) == 0
    compare(out_f64(out), _oracle(wl, vh), "f32", f"f32 bs={bs} {heads} P={P}")


@pytest.mark.parametrize("bs", [8, 32])
@pytest.mark.parametrize("P", [512, 0])
def test_long_contexts(bs, P):
    """Many partitions (fused merge and the reduce kernel) with 8- and 32-token blocks."""
    wl, vh, case = _poisoned_case(_cfg(bs, "bf16", 28, 4, 128, ctx=(20000, 3, 4097, 9000)), seed=bs + P)
    out = _decode(case, P)
    assert int(case.status.item()) == 0
    compare(out_f64(out), _oracle(wl, vh), "bf16", f"long bs={bs} P={P}")


@pytest.mark.parametrize("bs,bad_entry,dropped", [(8, 5, range(32, 48)), (8, 4, range(32, 48)),
                                                  (32, 1, range(32, 64)), (16, 2, range(32, 48))])
def test_bad_block_drops_its_tile(bs, bad_entry, dropped):
    """An out-of-pool id sets the status bit; the 16-token tile(s) holding it contribute nothing."""
    cfg = _cfg(bs, "f16", 28, 4, 128, ctx=(40, 100))
    wl = build_workload(cfg, seed=2)
    vh = host_values(wl)
    poison_unread_slots(wl, vh)
    wl.block_tables[1, bad_entry] = wl.num_blocks + 1000
    case = DeviceCase(wl, vh)
    out = out_f64(_decode(case, 64))
    pa = _pa()
    assert int(case.status.item()) & pa.PA_ERR_OUT_OF_RANGE
    c = wl.cfg
    ref0 = c_oracle.decode(vh["q"][:1], vh["key_cache"], vh["value_cache"], wl.block_tables[:1],
                           wl.context_lens[:1], c.scale, c.dtype, c.num_kv_heads)
    compare(out[:1], ref0, "f16", "unaffected sequence")
    toks = [i for i in range(100) if i not in dropped]
    kv = lambda pool: np.stack([pool[wl.block_tables[1, i // bs], :, i % bs] for i in toks], axis=1)
    K, V = kv(vh["key_cache"]), kv(vh["value_cache"])
    G = c.num_heads // c.num_kv_heads
    ref1 = np.stack([R.attention_f64(vh["q"][1, h].astype(np.float64), K[h // G].astype(np.float64),
                                     V[h // G].astype(np.float64), c.scale) for h in range(c.num_heads)])
    compare(out[1], ref1, "f16", "sequence with the bad block")


@pytest.mark.parametrize("bs", [8, 32])
@pytest.mark.parametrize("dtype", ["f32", "f16", "bf16"])
def test_cache_ops_bit_exact(bs, dtype):
    """Append, copy-on-write clone and swap to pinned host memory with 8- and 32-token blocks."""
    import torch

    pa = _pa()
    cfg = _cfg(bs, dtype, 8, 4, 128, ctx=(1, 7, 8, 9, 33, 200, 512, 31))
    wl = build_workload(cfg, seed=bs, pad_tokens=3)
    vh = host_values(wl)
    case = DeviceCase(wl, vh)
    d = case.dev
    pa.reshape_and_cache(d["key"], d["value"], d["key_cache"], d["value_cache"], case.slot_mapping,
                         status=case.status)
    kc, vc = R.reshape_and_cache(vh["key"], vh["value"], vh["key_cache"], vh["value_cache"], wl.slot_mapping)
    free = sorted(set(range(wl.num_blocks)) - set(int(x) for x in wl.block_tables.ravel()))
    pairs = np.array([[wl.block_tables[5, 0], free[0]], [wl.block_tables[6, 3], free[1]]], dtype=np.int64)
    pa.copy_blocks(d["key_cache"], d["value_cache"], torch.from_numpy(pairs).cuda(), status=case.status)
    kc, vc = R.copy_blocks(kc, vc, pairs)
    torch.cuda.synchronize()
    assert np.array_equal(R.bits_view(to_host(d["key_cache"], dtype)), R.bits_view(kc))
    assert np.array_equal(R.bits_view(to_host(d["value_cache"], dtype)), R.bits_view(vc))
    # whole blocks to pinned host pools and back into other device blocks
    hk = torch.empty((4,) + tuple(d["key_cache"].shape[1:]), dtype=d["key_cache"].dtype).pin_memory()
    hv = torch.empty_like(hk).pin_memory()
    out_pairs = torch.tensor([[int(wl.block_tables[7, 0]), 2], [int(wl.block_tables[6, 1]), 0]], dtype=torch.int64)
    pa.swap_blocks(d["key_cache"], d["value_cache"], hk, hv, out_pairs.cuda(), status=case.status)
    back = torch.tensor([[2, free[2]], [0, free[3]]], dtype=torch.int64).pin_memory()
    pa.swap_blocks(hk, hv, d["key_cache"], d["value_cache"], back, status=case.status)
    torch.cuda.synchronize()
    kc, vc = R.copy_blocks(kc, vc, np.array([[wl.block_tables[7, 0], free[2]], [wl.block_tables[6, 1], free[3]]]))
    assert np.array_equal(R.bits_view(to_host(d["key_cache"], dtype)), R.bits_view(kc))
    assert np.array_equal(R.bits_view(to_host(d["value_cache"], dtype)), R.bits_view(vc))
    assert int(case.status.item()) == 0


@pytest.mark.parametrize("bs", [8, 32])
def test_full_size_churned256_sampled(bs):
    """The churned 256-sequence step (append, then decode) with 8- and 32-token blocks, at full size, with
    NaN in every unread slot: sampled sequences against the oracle."""
    import torch

    pa = _pa()
    cfg = get_config("churned256", block_size=bs, num_blocks=80000 * 16 // bs)
    wl = build_workload(cfg, seed=0)
    case = DeviceCase(wl, device_draw=True)
    case.poison_unread()
    cl = wl.context_lens
    rng = np.random.default_rng(bs)
    seqs = sorted({int(np.argmax(cl)), int(np.argmin(cl))} | {int(x) for x in rng.integers(0, wl.num_seqs, 10)})
    sub = case.host_subproblem(seqs)
    d = case.dev
    pa.reshape_and_cache(d["key"], d["value"], d["key_cache"], d["value_cache"], case.slot_mapping,
                         status=case.status)
    out = _decode(case, cfg.partition_size)
    assert int(case.status.item()) == 0
    ref = oracle_step(sub, cfg)
    compare(out_f64(out)[seqs], ref, cfg.dtype, f"churned256 bs={bs}")
    torch.cuda.synchronize()


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_prefill_nan_in_unread_slots(dtype):
    """Paged prefill reads only slots inside the context, whatever the rest of its last block holds."""
    import torch

    pa = _pa()
    rng = np.random.default_rng(19)
    ctxs, chunks = [1, 15, 17, 64, 300, 129, 40], [1, 15, 16, 33, 300, 1, 40]
    Hq, Hkv, D = 28, 4, 128
    nb = sum(-(-c // 16) for c in ctxs) + 4
    perm = rng.permutation(nb)
    bt = np.full((len(ctxs), max(-(-c // 16) for c in ctxs)), -1, dtype=np.int32)
    k = 0
    extent = np.zeros(nb, dtype=np.int64)
    for b, c in enumerate(ctxs):
        for j in range(-(-c // 16)):
            bt[b, j] = perm[k]
            extent[perm[k]] = min(16, c - 16 * j)
            k += 1
    draw = lambda s: (rng.standard_normal(s).astype(np.float16) if dtype == "f16"
                      else (rng.standard_normal(s).astype(np.float32).view(np.uint32) >> 16).astype(np.uint16))
    kc, vc = draw((nb, Hkv, 16, D)), draw((nb, Hkv, 16, D))
    blk, off = np.nonzero(np.arange(16)[None, :] >= extent[:, None])
    nan = np.float16(np.nan) if dtype == "f16" else np.uint16(0x7FC0)
    kc[blk, :, off, :] = nan
    vc[blk, :, off, :] = nan
    qs = np.concatenate([[0], np.cumsum(chunks)]).astype(np.int32)
    q = draw((int(qs[-1]), Hq, D))
    cl = np.array(ctxs, dtype=np.int32)
    tdt = torch.float16 if dtype == "f16" else torch.bfloat16
    out = torch.empty(q.shape, dtype=tdt, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    scale = 1.0 / np.sqrt(D)
    pa.prefill(out, to_device(q, dtype), to_device(kc, dtype), to_device(vc, dtype), torch.from_numpy(bt).cuda(),
               torch.from_numpy(qs).cuda(), torch.from_numpy(cl).cuda(), scale, int(max(chunks)), status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    compare(out_f64(out), c_oracle.prefill(q, kc, vc, bt, qs, cl, scale, dtype, Hkv), dtype, f"prefill {dtype}")
