"""Host-side input generation: tables, slots and copy pairs are well formed (CPU only)."""

import numpy as np
import pytest

from oracle import reference as R
from workloads import CONFIGS, build_workload, get_config, host_values


def _used_blocks(wl):
    bs = wl.cfg.block_size
    out = []
    for b in range(wl.num_seqs):
        n = -(-int(wl.context_lens[b]) // bs)
        out.append(wl.block_tables[b, :n])
    return out


def _check_well_formed(wl, name):
    cfg = wl.cfg
    bs = cfg.block_size
    assert wl.context_lens.dtype == np.int32 and wl.block_tables.dtype == np.int32
    assert wl.slot_mapping.dtype == np.int64
    used = _used_blocks(wl)
    for b, blocks in enumerate(used):
        assert ((blocks >= 0) & (blocks < cfg.num_blocks)).all()
        n = -(-int(wl.context_lens[b]) // bs)
        assert (wl.block_tables[b, n:] == -1).all()
    # appended token b sits at position ctx-1 of sequence b
    for b in range(wl.num_seqs):
        pos = int(wl.context_lens[b]) - 1
        assert wl.slot_mapping[b] == wl.block_tables[b, pos // bs] * bs + pos % bs
    return used


@pytest.mark.parametrize("name", sorted(CONFIGS))
def test_tables_slots_well_formed(name):
    wl = build_workload(get_config(name), seed=0)
    used = _check_well_formed(wl, name)
    if name != "shared_prefix":
        flat = np.concatenate(used)
        assert len(np.unique(flat)) == len(flat), "private blocks must not be shared"


def test_tiny_matches_config_text():
    wl = build_workload(get_config("tiny"), seed=0)
    assert list(wl.context_lens) == [1, 15, 16, 37]
    assert wl.num_blocks == 32 and wl.cfg.num_heads == 4 and wl.cfg.num_kv_heads == 2
    assert wl.cfg.head_dim == 64 and wl.cfg.dtype == "f32" and wl.cfg.scale == 1 / 8


def test_long32k_shape():
    wl = build_workload(get_config("long32k"), seed=0)
    assert (wl.context_lens == 32768).all() and wl.block_tables.shape == (8, 2048)
    assert wl.kv_bytes() == 8 * 32768 * 4 * 128 * 2 * 2


def test_churned_pool_is_fragmented():
    wl = build_workload(get_config("churned256"), seed=0)
    assert wl.num_seqs == 256
    assert 8 <= wl.context_lens.min() and wl.context_lens.max() <= 4096
    assert 200 < np.median(wl.context_lens) < 450
    # consecutive logical blocks land far apart in the pool
    assert wl.info["mean_block_id_gap"] > 1000


def test_shared_prefix_copy_on_write_setup():
    wl = build_workload(get_config("shared_prefix"), seed=0)
    info = wl.info
    pre = info["prefix_blocks"]
    assert len(pre) == 32 and wl.num_seqs == 1024
    for b in range(wl.num_seqs):
        assert list(wl.block_tables[b, :32]) == pre
    pairs = wl.copy_pairs
    assert pairs.shape == (64, 2)
    assert (pairs[:, 0] == info["parent_partial"]).all()
    assert len(np.unique(pairs[:, 1])) == 64
    assert not np.isin(pairs[:, 1], pairs[:, 0]).any()
    forks = np.arange(wl.num_seqs - 64, wl.num_seqs)
    r = info["shared_tokens_in_partial"]
    assert 1 <= r <= 15
    assert (wl.context_lens[forks] == 512 + r + 1).all()
    assert set(wl.block_tables[forks, 32]) == set(pairs[:, 1])
    # each fork's new token goes at offset r of its own clone
    assert (wl.slot_mapping[forks] == wl.block_tables[forks, 32].astype(np.int64) * 16 + r).all()
    regular = np.arange(wl.num_seqs - 64)
    suf = wl.context_lens[regular] - 512
    assert suf.min() >= 16 and suf.max() <= 1024


def test_padding_slots_inserted():
    wl = build_workload(get_config("tiny"), seed=3, pad_tokens=3)
    assert wl.num_tokens == 4 + 3 and (wl.slot_mapping == -1).sum() == 3


def test_identity_placement_is_contiguous():
    wl = build_workload(get_config("qwen_layer"), seed=0, placement="identity")
    flat = np.concatenate(_used_blocks(wl))
    assert np.array_equal(flat, np.arange(len(flat)))


def test_write_then_walk_returns_appended_token():
    """Host logic consistency: the slot of each appended token is where the table walk finds it."""
    wl = build_workload(get_config("tiny"), seed=5, pad_tokens=2)
    v = host_values(wl)
    kc, vc = R.reshape_and_cache(v["key"], v["value"], v["key_cache"], v["value_cache"], wl.slot_mapping)
    real = np.flatnonzero(wl.slot_mapping >= 0)
    for b in range(wl.num_seqs):
        ctx = int(wl.context_lens[b])
        for g in range(wl.cfg.num_kv_heads):
            rows = R.gather_kv(kc, wl.block_tables[b], ctx, g, 16)
            assert np.array_equal(rows[ctx - 1], v["key"][real[b], g])


def test_seeded_generation_is_deterministic():
    a = build_workload(get_config("churned256"), seed=7)
    b = build_workload(get_config("churned256"), seed=7)
    assert np.array_equal(a.block_tables, b.block_tables) and np.array_equal(a.context_lens, b.context_lens)
    c = build_workload(get_config("churned256"), seed=8)
    assert not np.array_equal(a.context_lens, c.context_lens)


@pytest.mark.parametrize("name", ["churned256", "long32k"])
@pytest.mark.parametrize("bs", [8, 32])
def test_block_size_variants_hold_the_same_sequences(name, bs):
    """The block-size sweep compares like with like: the same context lengths, a pool of the same token
    capacity, ceil(ctx / bs) private blocks per sequence, well-formed tables and slots."""
    base = build_workload(get_config(name), seed=0)
    c0 = get_config(name)
    wl = build_workload(get_config(name, block_size=bs, num_blocks=c0.num_blocks * 16 // bs), seed=0)
    assert np.array_equal(wl.context_lens, base.context_lens)
    assert wl.num_blocks * bs == base.num_blocks * 16
    used = _check_well_formed(wl, name)
    flat = np.concatenate(used)
    assert len(np.unique(flat)) == len(flat)
    assert len(flat) == sum(-(-int(c) // bs) for c in wl.context_lens)
