"""The oracle checked against what the pages and the mathematics fix (CPU only)."""

import types

import numpy as np
import pytest

import pins
from oracle import c_oracle
from oracle import reference as R


@pytest.mark.parametrize("check", pins.ALL_CHECKS, ids=lambda c: c.__name__)
def test_numpy_oracle_pin(check):
    check(R)


def _c_impl():
    ns = types.SimpleNamespace(**{k: getattr(R, k) for k in dir(R) if not k.startswith("_")})
    ns.decode = c_oracle.decode
    return ns


C_DECODE_CHECKS = [
    pins.check_p3_block_table_walk,
    pins.check_permutation_invariance,
    pins.check_matches_contiguous_sdpa,
    pins.check_single_token_is_v,
    pins.check_zero_query_is_mean,
    pins.check_equal_keys_is_mean,
    pins.check_dominant_key,
    pins.check_empty_context_is_zero,
]


@pytest.mark.parametrize("check", C_DECODE_CHECKS, ids=lambda c: c.__name__)
def test_c_oracle_pin(check):
    check(_c_impl())


@pytest.mark.parametrize("dtype", ["f32", "f16", "bf16"])
def test_c_oracle_equals_numpy_oracle(dtype):
    ctxs = [1, 15, 16, 17, 37, 64, 130]
    q, kc, vc, bt, cl = pins._rand_case(21, len(ctxs), 8, 2, 64, ctxs, NB=40, dtype=dtype)
    a = R.decode(q, kc, vc, bt, cl, 0.125, dtype, 2)
    b = c_oracle.decode(q, kc, vc, bt, cl, 0.125, dtype, 2)
    assert np.abs(a - b).max() < 1e-12
    pairs = [(6, 7), (0, 0), (3, 4)]
    c = c_oracle.decode_pairs(pairs, q, kc, vc, bt, cl, 0.125, dtype, 2)
    for k, (bb, hh) in enumerate(pairs):
        assert np.array_equal(c[k], b[bb, hh])


def test_c_oracle_half_conversion_all_finite_patterns():
    """Every finite binary16 pattern survives the C oracle's upcast exactly (n = 1 -> out = V)."""
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    vals = bits.view(np.float16)
    finite = bits[np.isfinite(vals)]
    D = 64
    n = len(finite) // D
    v = finite[: n * D].view(np.float16).reshape(n, 1, 1, D)
    vc = np.zeros((n, 1, 16, D), dtype=np.float16)
    vc[:, :, :1, :] = v
    kc = np.zeros_like(vc)
    q = np.zeros((n, 1, D), dtype=np.float16)
    bt = np.arange(n, dtype=np.int32)[:, None]
    out = c_oracle.decode(q, kc, vc, bt, np.ones(n, np.int32), 1.0, "f16", 1)
    assert np.array_equal(out[:, 0, :], v[:, 0, 0, :].astype(np.float64))


def test_bf16_upcast_known_patterns():
    pat = np.array([0x3F80, 0xBF80, 0x4049, 0x0001, 0x7F7F, 0x0000, 0x8000], dtype=np.uint16)
    expect = [1.0, -1.0, 3.140625, 2.0 ** -133, 3.3895313892515355e38, 0.0, -0.0]
    got = R.to_f64(pat, "bf16")
    assert list(got) == expect


def test_c_oracle_rejects_out_of_pool_block():
    q, kc, vc, bt, cl = pins._rand_case(22, 2, 2, 1, 16, [5, 20], NB=4)
    bt[1, 1] = 4
    with pytest.raises(IndexError):
        c_oracle.decode(q, kc, vc, bt, cl, 1.0, "f32", 1)
    with pytest.raises(IndexError):
        R.decode(q, kc, vc, bt, cl, 1.0, "f32", 1)


def _relayout(kc, vc, tables, ctx, bs, rng):
    """The same per-sequence K/V rows in a pool of block size ``bs``, blocks placed at random."""
    B = len(ctx)
    nblk = [-(-int(n) // bs) for n in ctx]
    nb = sum(nblk) + 3
    Hkv, D = kc.shape[1], kc.shape[3]
    bs0 = kc.shape[2]
    k2 = rng.standard_normal((nb, Hkv, bs, D)).astype(kc.dtype)
    v2 = rng.standard_normal((nb, Hkv, bs, D)).astype(vc.dtype)
    perm = rng.permutation(nb)
    t2 = np.full((B, max(1, max(nblk))), -1, dtype=np.int32)
    k = 0
    for b in range(B):
        for j in range(nblk[b]):
            t2[b, j] = perm[k]
            k += 1
        for i in range(int(ctx[b])):
            src = tables[b, i // bs0]
            k2[t2[b, i // bs], :, i % bs] = kc[src, :, i % bs0]
            v2[t2[b, i // bs], :, i % bs] = vc[src, :, i % bs0]
    return k2, v2, t2


@pytest.mark.parametrize("bs", [1, 4, 8, 32])
def test_oracle_output_does_not_depend_on_block_size(bs):
    """Paging changes where K/V rows live, not the attention ("PagedAttention" digest, "Why the attention
    kernel works at all"): the same rows in pools of another block size give the same bits."""
    rng = np.random.default_rng(bs)
    ctx = np.array([1, 7, 8, 9, 16, 33, 70], dtype=np.int32)
    Hq, Hkv, D = 6, 2, 16
    # a pool of block size 16 with random rows, then the same rows re-laid at bs
    nb = sum(-(-int(n) // 16) for n in ctx)
    k16 = rng.standard_normal((nb, Hkv, 16, D)).astype(np.float32)
    v16 = rng.standard_normal((nb, Hkv, 16, D)).astype(np.float32)
    t16 = np.full((len(ctx), 5), -1, dtype=np.int32)
    k = 0
    for b, n in enumerate(ctx):
        for j in range(-(-int(n) // 16)):
            t16[b, j] = k
            k += 1
    q = rng.standard_normal((len(ctx), Hq, D)).astype(np.float32)
    kb, vb, tb = _relayout(k16, v16, t16, ctx, bs, rng)
    a = R.decode(q, k16, v16, t16, ctx, 0.25, "f32", Hkv)
    b = R.decode(q, kb, vb, tb, ctx, 0.25, "f32", Hkv)
    assert np.array_equal(a, b)
    c = c_oracle.decode(q, kb, vb, tb, ctx, 0.25, "f32", Hkv)
    assert np.allclose(a, c, rtol=0, atol=1e-12)


@pytest.mark.parametrize("bs", [8, 16, 32])
def test_oracle_never_reads_past_the_context(bs):
    """Slots past a sequence's context (the tail of its last block, unused blocks) may hold NaN: the oracle's
    result is unchanged, bit for bit, and finite."""
    from workloads import build_workload, get_config, host_values, poison_unread_slots, unread_slots

    ctx = (0, 1, 7, 8, 9, 15, 17, 31, 33, 100)
    need = sum(-(-c // bs) for c in ctx)
    cfg = get_config("qwen_layer", dtype="f16", num_heads=8, num_kv_heads=2, head_dim=64, block_size=bs,
                     num_blocks=need + 5, ctx_kind="fixed", ctx_args=ctx)
    wl = build_workload(cfg, seed=bs)
    vh = host_values(wl)
    before = c_oracle.decode(vh["q"], vh["key_cache"], vh["value_cache"], wl.block_tables, wl.context_lens,
                             cfg.scale, "f16", 2)
    n = poison_unread_slots(wl, vh)
    # exactly the slots past each context: block tails plus the 5 unused blocks
    assert n == need * bs - sum(ctx) + 5 * bs
    blk, off = unread_slots(wl)
    for b, c in enumerate(ctx):
        for i in range(c):
            assert not ((blk == wl.block_tables[b, i // bs]) & (off == i % bs)).any()
    after = c_oracle.decode(vh["q"], vh["key_cache"], vh["value_cache"], wl.block_tables, wl.context_lens,
                            cfg.scale, "f16", 2)
    assert np.isfinite(after).all() and np.array_equal(before, after)


def test_unread_slots_keep_copy_sources_whole():
    """A fork's clone is copied from a block no table names; its slots are still read (through the copy),
    so poisoning unread slots must leave copy sources whole: the oracle's step is unchanged."""
    from workloads import build_workload, get_config, host_values, poison_unread_slots, unread_slots
    from parity import oracle_step

    cfg = get_config("shared_prefix", num_heads=8, num_kv_heads=2, head_dim=64, num_blocks=4000)
    wl = build_workload(cfg, seed=4, num_seqs=40)
    assert wl.copy_pairs.size
    blk, _ = unread_slots(wl)
    assert not np.isin(wl.copy_pairs[:, 0], blk).any()
    vh = host_values(wl)
    sub = dict(q=vh["q"], key_cache=vh["key_cache"], value_cache=vh["value_cache"], block_tables=wl.block_tables,
               context_lens=wl.context_lens, key=vh["key"], value=vh["value"], slot_mapping=wl.slot_mapping,
               copy_pairs=wl.copy_pairs)
    before = oracle_step(sub, cfg)
    poison_unread_slots(wl, vh)
    sub.update(key_cache=vh["key_cache"], value_cache=vh["value_cache"])
    after = oracle_step(sub, cfg)
    assert np.isfinite(after).all() and np.array_equal(before, after)
