"""Pins for the oracle: checks against what the pages and the mathematics fix.

Each ``check_*`` takes an oracle implementation (a namespace with the
functions of ``oracle.reference``) and raises AssertionError if the
implementation disagrees with the pin.  ``test_oracle_pins.py`` runs them on
the real oracle; ``test_oracle_mutants.py`` plants plausible mistakes in
copies of the oracle and checks that some pin catches each one.
"""

from __future__ import annotations

import json
import math
import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def golden(name: str) -> dict:
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _rand_case(seed, B, Hq, Hkv, D, ctxs, NB, bs=16, dtype="f32", placement=None):
    """Small random paged problem (fp32/f16/bf16 storage) with a seeded placement."""
    from workloads.gen import _normal

    rng = np.random.default_rng(seed)
    nblk = [-(-c // bs) for c in ctxs]
    MB = max(1, max(nblk))
    perm = rng.permutation(NB) if placement is None else np.asarray(placement)
    bt = np.full((B, MB), -1, dtype=np.int32)
    k = 0
    for b in range(B):
        for j in range(nblk[b]):
            bt[b, j] = perm[k]
            k += 1
    q = _normal(rng, (B, Hq, D), dtype)
    kc = _normal(rng, (NB, Hkv, bs, D), dtype)
    vc = _normal(rng, (NB, Hkv, bs, D), dtype)
    return q, kc, vc, bt, np.asarray(ctxs, dtype=np.int32)


def _replace(kc, vc, bt, ctxs, new_perm, bs=16):
    """Move every used block to a new physical id given by new_perm (old -> new)."""
    kc2 = np.zeros_like(kc)
    vc2 = np.zeros_like(vc)
    bt2 = bt.copy()
    for b in range(bt.shape[0]):
        for j in range(-(-int(ctxs[b]) // bs)):
            old = bt[b, j]
            new = new_perm[old]
            kc2[new] = kc[old]
            vc2[new] = vc[old]
            bt2[b, j] = new
    return kc2, vc2, bt2


# ---------------------------------------------------------------------------
# sizes and block rounding
# ---------------------------------------------------------------------------


def check_kv_sizes(impl):
    g = golden("p1_kv_sizes.json")
    assert impl.kv_bytes_per_token(4, 128, 28, 2) == g["kv_bytes_per_token"]
    assert impl.kv_bytes_per_token(4, 128, 1, 2) == g["kv_bytes_per_token_per_layer"]
    gib = g["a40_vllm_kv_tokens"] * impl.kv_bytes_per_token(4, 128, 28, 2) / 2 ** 30
    assert round(gib, 2) == g["a40_vllm_kv_gib"]
    gb = g["conversation_tokens"] * impl.kv_bytes_per_token(4, 128, 28, 2) / 1e9
    assert round(gb, 1) == g["conversation_gb_approx"]
    w = impl.reservation_waste(g["reservation_used_tokens"], g["reservation_tokens"])
    assert round(w, 2) == g["reservation_waste_approx"]


def check_block_rounding(impl):
    g = golden("p2_block_rounding.json")
    bs = g["block_size"]
    assert impl.blocks_needed(g["tokens"], bs) == g["blocks"]
    assert impl.blocks_needed(g["tokens"], bs) * bs == g["slots"]
    for n in range(1, 200):
        w = impl.paged_waste_tokens(n, bs)
        assert 0 <= w <= g["max_waste_tokens"], (n, w)
        assert impl.blocks_needed(n, bs) * bs - n == w
    assert impl.blocks_needed(16, 16) == 1 and impl.blocks_needed(17, 16) == 2
    assert impl.blocks_needed(0, 16) == 0


def check_p3_block_table_walk(impl):
    """Block size 4: A0 -> page 0, A1 -> page 3, A2 -> page 7; 9 tokens, 3 empty slots."""
    g = golden("p3_block_size4.json")
    bs = g["block_size"]
    toks = g["tokens"]
    n = len(toks)
    assert impl.blocks_needed(n, bs) == len(g["logical_to_physical"])
    assert impl.paged_waste_tokens(n, bs) == g["empty_slots_in_last_block"]
    table = np.array([g["logical_to_physical"][f"A{j}"] for j in range(3)], dtype=np.int32)
    # a pool of 12 pages, 1 KV head, 4 slots, D = 2: page p slot o holds (p, o)
    pool = np.zeros((12, 1, bs, 2), dtype=np.float32)
    for p in range(12):
        for o in range(bs):
            pool[p, 0, o] = (p, o)
    rows = impl.gather_kv(pool, table, n, 0, bs)
    for i, tok in enumerate(toks):
        blk = g["block_contents"][f"A{i // bs}"]
        assert blk[i % bs] == tok
        assert tuple(rows[i]) == (g["logical_to_physical"][f"A{i // bs}"], i % bs), (i, rows[i])
    # attention over the request: a key that dominates on token "dog" (page 7, slot 0)
    kc = np.zeros((12, 1, bs, 1), dtype=np.float32)
    vc = np.zeros((12, 1, bs, 1), dtype=np.float32)
    for i in range(n):
        p, o = int(table[i // bs]), i % bs
        vc[p, 0, o, 0] = float(i)
        kc[p, 0, o, 0] = 40.0 if toks[i] == "dog" else 0.0
    q = np.ones((1, 1, 1), dtype=np.float32)
    out = impl.decode(q, kc, vc, table[None, :], np.array([n], np.int32), 1.0, "f32", 1)
    assert abs(out[0, 0, 0] - toks.index("dog")) < 1e-12 * n + 8 * math.exp(-40.0) * n


def check_two_token_closed_form(impl):
    g = golden("two_token_attention.json")
    q = np.array(g["q"], dtype=np.float64)
    k = np.array(g["k"], dtype=np.float64)
    v = np.array(g["v"], dtype=np.float64)
    # put the two tokens in physical block 5 of a 8-block pool (block size 16)
    kc = np.zeros((8, 1, 16, 2), dtype=np.float64)
    vc = np.zeros((8, 1, 16, 2), dtype=np.float64)
    kc[5, 0, :2] = k
    vc[5, 0, :2] = v
    bt = np.array([[5]], dtype=np.int32)
    out = impl.decode(q[None, None, :], kc, vc, bt, np.array([2], np.int32), g["scale"], "f64", 1)
    assert np.abs(out[0, 0] - np.array(g["out"])).max() < g["tol"], out


# ---------------------------------------------------------------------------
# attention invariants
# ---------------------------------------------------------------------------


def check_permutation_invariance(impl):
    """Same logical K/V, different physical placement -> bitwise equal fp64 output."""
    for seed, dtype in ((0, "f32"), (1, "f16"), (2, "bf16")):
        ctxs = [1, 15, 16, 37, 70]
        q, kc, vc, bt, cl = _rand_case(seed, 5, 6, 2, 32, ctxs, NB=40, dtype=dtype)
        a = impl.decode(q, kc, vc, bt, cl, 0.3, dtype, 2)
        perm = np.random.default_rng(100 + seed).permutation(40)
        kc2, vc2, bt2 = _replace(kc, vc, bt, cl, perm)
        b = impl.decode(q, kc2, vc2, bt2, cl, 0.3, dtype, 2)
        assert np.array_equal(a, b), np.abs(a - b).max()


def _sdpa_contiguous(q64, k64, v64, scale, Hkv):
    """torch SDPA (CPU, fp64) on contiguous K/V; GQA by repeating KV heads."""
    import torch
    import torch.nn.functional as F

    Hq = q64.shape[0]
    G = Hq // Hkv
    qt = torch.from_numpy(q64)[None, :, None, :]                 # [1, Hq, 1, D]
    kt = torch.from_numpy(k64).repeat_interleave(G, dim=0)[None]  # [1, Hq, n, D]
    vt = torch.from_numpy(v64).repeat_interleave(G, dim=0)[None]
    return F.scaled_dot_product_attention(qt, kt, vt, scale=scale)[0, :, 0, :].numpy()


def check_matches_contiguous_sdpa(impl):
    """Paged result equals contiguous (unpaged) attention from torch's SDPA."""
    from oracle.reference import to_f64

    for seed, (Hq, Hkv), dtype in ((3, (8, 2), "f32"), (4, (4, 4), "f16"), (5, (7, 1), "bf16"),
                                   (6, (12, 4), "f32")):
        ctxs = [1, 9, 16, 33, 64]
        q, kc, vc, bt, cl = _rand_case(seed, len(ctxs), Hq, Hkv, 16, ctxs, NB=32, dtype=dtype)
        out = impl.decode(q, kc, vc, bt, cl, 0.25, dtype, Hkv)
        for b, n in enumerate(ctxs):
            # contiguous copy of the sequence's K/V, [Hkv, n, D], built by hand
            kcont = np.zeros((Hkv, n, 16))
            vcont = np.zeros((Hkv, n, 16))
            for i in range(n):
                blk = bt[b, i // 16]
                kcont[:, i] = to_f64(kc[blk, :, i % 16], dtype)
                vcont[:, i] = to_f64(vc[blk, :, i % 16], dtype)
            ref = _sdpa_contiguous(to_f64(q[b], dtype), kcont, vcont, 0.25, Hkv)
            assert np.abs(out[b] - ref).max() < 1e-12, (seed, b, np.abs(out[b] - ref).max())


def check_single_token_is_v(impl):
    """n = 1: softmax weight is exactly 1, output is that token's V row."""
    from oracle.reference import to_f64

    for dtype in ("f32", "f16", "bf16"):
        q, kc, vc, bt, cl = _rand_case(7, 3, 4, 2, 16, [1, 1, 1], NB=8, dtype=dtype)
        out = impl.decode(q, kc, vc, bt, cl, 0.7, dtype, 2)
        for b in range(3):
            for h in range(4):
                assert np.array_equal(out[b, h], to_f64(vc[bt[b, 0], h // 2, 0], dtype))


def check_zero_query_is_mean(impl):
    """q = 0: every logit equal, output is the plain mean of the V rows."""
    from oracle.reference import to_f64

    ctxs = [15, 16, 37]
    q, kc, vc, bt, cl = _rand_case(8, 3, 4, 2, 16, ctxs, NB=16)
    q[:] = 0
    out = impl.decode(q, kc, vc, bt, cl, 1.0, "f32", 2)
    for b, n in enumerate(ctxs):
        for h in range(4):
            rows = [to_f64(vc[bt[b, i // 16], h // 2, i % 16], "f32") for i in range(n)]
            assert np.abs(out[b, h] - np.mean(rows, axis=0)).max() < 1e-13


def check_equal_keys_is_mean(impl):
    """All keys equal: output is the mean of V regardless of q."""
    from oracle.reference import to_f64

    q, kc, vc, bt, cl = _rand_case(9, 2, 2, 1, 16, [16, 21], NB=8)
    kc[:] = kc[0, 0, 0]
    out = impl.decode(q, kc, vc, bt, cl, 0.5, "f32", 1)
    for b, n in enumerate([16, 21]):
        rows = [to_f64(vc[bt[b, i // 16], 0, i % 16], "f32") for i in range(n)]
        assert np.abs(out[b, 0] - np.mean(rows, axis=0)).max() < 1e-13
        assert np.abs(out[b, 1] - np.mean(rows, axis=0)).max() < 1e-13


def check_dominant_key(impl):
    """One logit 50 above the rest: output is that token's V row up to e^-50 * n."""
    from oracle.reference import to_f64

    q, kc, vc, bt, cl = _rand_case(10, 1, 1, 1, 8, [37], NB=8)
    q[:] = 0
    q[0, 0, 0] = 1.0
    kc[:, :, :, 0] = 0.0
    star = 29                                  # a token in the last, partial block
    blk = bt[0, star // 16]
    kc[blk, 0, star % 16, 0] = 50.0
    out = impl.decode(q, kc, vc, bt, cl, 1.0, "f32", 1)
    ref = to_f64(vc[blk, 0, star % 16], "f32")
    assert np.abs(out[0, 0] - ref).max() < 37 * 8 * math.exp(-50.0) + 1e-14


def check_empty_context_is_zero(impl):
    q, kc, vc, bt, cl = _rand_case(11, 2, 2, 1, 8, [0, 5], NB=4)
    out = impl.decode(q, kc, vc, bt, cl, 0.5, "f32", 1)
    assert np.array_equal(out[0], np.zeros_like(out[0]))
    assert np.abs(out[1]).max() > 0


def check_split_merge_identity(impl):
    """Partitioned softmax merged by rescaling equals the unsplit result (fp64)."""
    for dtype in ("f32", "bf16"):
        ctxs = [1, 15, 16, 37, 100, 600]
        q, kc, vc, bt, cl = _rand_case(12, len(ctxs), 4, 2, 16, ctxs, NB=60, dtype=dtype)
        full = impl.decode(q, kc, vc, bt, cl, 0.4, dtype, 2)
        for P in (1, 4, 16, 32, 512, 4096):
            for b in range(len(ctxs)):
                for h in range(4):
                    s = impl.decode_split(q, kc, vc, bt, cl, b, h, 0.4, dtype, 2, P)
                    assert np.abs(s - full[b, h]).max() < 1e-12, (P, b, h)


# ---------------------------------------------------------------------------
# cache write and block copy
# ---------------------------------------------------------------------------


def check_reshape_and_cache_hand_example(impl):
    """Three tokens, slots [5, -1, 18] in a 2-block pool (block size 16, 1 head, D = 2)."""
    key = np.array([[[1, 2]], [[3, 4]], [[5, 6]]], dtype=np.float32)
    value = -key
    kc = np.zeros((2, 1, 16, 2), dtype=np.float32)
    vc = np.zeros_like(kc)
    kc2, vc2 = impl.reshape_and_cache(key, value, kc, vc, np.array([5, -1, 18], dtype=np.int64))
    expect_k = np.zeros_like(kc)
    expect_k[0, 0, 5] = (1, 2)      # slot 5  -> block 0, offset 5
    expect_k[1, 0, 2] = (5, 6)      # slot 18 -> block 1, offset 2; token 1 is padding
    assert np.array_equal(kc2, expect_k)
    assert np.array_equal(vc2, -expect_k)
    assert np.array_equal(kc, np.zeros_like(kc))   # inputs untouched


def check_reshape_and_cache_two_heads(impl):
    key = np.arange(2 * 3 * 4, dtype=np.float32).reshape(2, 3, 4)
    value = key + 100
    kc = np.full((3, 3, 16, 4), -1, dtype=np.float32)
    vc = kc.copy()
    kc2, vc2 = impl.reshape_and_cache(key, value, kc, vc, np.array([47, 16], dtype=np.int64))
    assert np.array_equal(kc2[2, :, 15], key[0]) and np.array_equal(vc2[2, :, 15], value[0])
    assert np.array_equal(kc2[1, :, 0], key[1]) and np.array_equal(vc2[1, :, 0], value[1])
    mask = np.ones(kc.shape[:3], bool)
    mask[2, :, 15] = False
    mask[1, :, 0] = False
    assert (kc2[mask] == -1).all()


def check_copy_blocks_hand_example(impl):
    """Clone block 1 into blocks 3 and 0 (copy-on-write of a shared block)."""
    kc = np.arange(4 * 2 * 16 * 2, dtype=np.float32).reshape(4, 2, 16, 2)
    vc = kc * 10
    kc2, vc2 = impl.copy_blocks(kc, vc, np.array([[1, 3], [1, 0]], dtype=np.int64))
    assert np.array_equal(kc2[3], kc[1]) and np.array_equal(kc2[0], kc[1])
    assert np.array_equal(vc2[3], vc[1]) and np.array_equal(vc2[0], vc[1])
    assert np.array_equal(kc2[1], kc[1]) and np.array_equal(kc2[2], kc[2])   # source, bystander intact


ALL_CHECKS = [
    check_kv_sizes,
    check_block_rounding,
    check_p3_block_table_walk,
    check_two_token_closed_form,
    check_permutation_invariance,
    check_matches_contiguous_sdpa,
    check_single_token_is_v,
    check_zero_query_is_mean,
    check_equal_keys_is_mean,
    check_dominant_key,
    check_empty_context_is_zero,
    check_split_merge_identity,
    check_reshape_and_cache_hand_example,
    check_reshape_and_cache_two_heads,
    check_copy_blocks_hand_example,
]
