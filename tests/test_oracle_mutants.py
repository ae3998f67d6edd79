"""Plant plausible mistakes in copies of the oracle and check that a pin catches each.

This is what makes the pins worth trusting: a dropped term, a wrong sign or
index, a transposed operand anywhere in the oracle must fail at least one of
them.  Mistakes are planted only in fresh CPU copies of oracle/reference.py.
"""

import importlib.util
import os

import numpy as np
import pytest

import pins

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _fresh_oracle(tag):
    spec = importlib.util.spec_from_file_location(f"oracle_mutant_{tag}",
                                                  os.path.join(ROOT, "oracle", "reference.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _mutants():
    out = {}

    def add(name):
        def deco(fn):
            out[name] = fn
            return fn
        return deco

    @add("gqa_head_modulo")
    def _(m):
        def decode_one(q, kc, vc, bt, cl, b, h, scale, dtype, hkv):
            # wrong GQA grouping: query head h reads KV head h % Hkv instead of h // G
            bs, ctx, g = kc.shape[2], int(cl[b]), h % hkv
            kb = m.to_f64(m.gather_kv(kc, bt[b], ctx, g, bs), dtype)
            vb = m.to_f64(m.gather_kv(vc, bt[b], ctx, g, bs), dtype)
            return m.attention_f64(m.to_f64(q[b, h], dtype), kb, vb, scale)
        m.decode_one = decode_one

    @add("scale_dropped")
    def _(m):
        orig = m.attention_f64
        m.attention_f64 = lambda q, k, v, scale: orig(q, k, v, 1.0)

    @add("sign_flipped_logits")
    def _(m):
        orig = m.attention_f64
        m.attention_f64 = lambda q, k, v, scale: orig(q, k, v, -scale)

    @add("table_ignored")
    def _(m):
        m.token_slot = lambda row, pos, bs: (pos // bs, pos % bs)

    @add("offset_off_by_one")
    def _(m):
        m.token_slot = lambda row, pos, bs: (int(row[pos // bs]), (pos + 1) % bs)

    @add("last_token_dropped")
    def _(m):
        orig = m.gather_kv
        m.gather_kv = lambda cache, row, ctx, g, bs: orig(cache, row, max(ctx - 1, 0), g, bs)

    @add("k_and_v_swapped")
    def _(m):
        orig = m.attention_f64
        m.attention_f64 = lambda q, k, v, scale: orig(q, v, k, scale)

    @add("softmax_not_normalised")
    def _(m):
        def att(q, k, v, scale):
            n = k.shape[0]
            if n == 0:
                return np.zeros(v.shape[1])
            s = np.array([scale * float(np.dot(q, k[i])) for i in range(n)])
            w = np.exp(s - s.max())
            return (w[:, None] * v).sum(0)
        m.attention_f64 = att

    @add("merge_without_rescale")
    def _(m):
        def merge(parts):
            parts = [p for p in parts if p[1] > 0.0]
            if not parts:
                return None
            return sum(p[2] for p in parts) / sum(p[1] for p in parts)
        m.merge_partials = merge

    @add("write_block_offset_swapped")
    def _(m):
        orig = m.reshape_and_cache

        def rc(key, value, kc, vc, slots):
            bs = kc.shape[2]
            swapped = np.array([(s % bs) * bs + s // bs if s >= 0 else s for s in slots], dtype=np.int64)
            return orig(key, value, kc, vc, swapped)
        m.reshape_and_cache = rc

    @add("write_ignores_padding_rule")
    def _(m):
        orig = m.reshape_and_cache

        def rc(key, value, kc, vc, slots):
            return orig(key, value, kc, vc, np.where(np.asarray(slots) < 0, 0, slots))
        m.reshape_and_cache = rc

    @add("copy_direction_reversed")
    def _(m):
        orig = m.copy_blocks
        m.copy_blocks = lambda kc, vc, pairs: orig(kc, vc, np.asarray(pairs)[:, ::-1])

    @add("kv_bytes_missing_k_or_v")
    def _(m):
        m.kv_bytes_per_token = lambda hkv, d, layers, e: hkv * d * layers * e

    @add("blocks_rounded_down")
    def _(m):
        m.blocks_needed = lambda n, bs: n // bs

    return out


MUTANTS = _mutants()


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_some_pin_catches_mutant(name):
    m = _fresh_oracle(name)
    MUTANTS[name](m)
    caught = []
    for check in pins.ALL_CHECKS:
        try:
            check(m)
        except (AssertionError, IndexError, ValueError):
            caught.append(check.__name__)
    assert caught, f"no pin catches mutant {name}"


def test_unmutated_copy_passes_every_pin():
    m = _fresh_oracle("clean")
    for check in pins.ALL_CHECKS:
        check(m)
