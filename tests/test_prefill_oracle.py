"""Pins of the prefill oracle (oracle/reference.py prefill), CPU only.

Causal prefill has plain special cases the definition fixes: the first prompt
token sees only itself (its output is its own V row), the last row of a whole
prompt is that prompt's decode, and on contiguous K/V the whole thing is
torch's causal scaled-dot-product attention (with GQA by repeating KV heads).
A chunk on top of an existing context equals the rows of the full prefill.
"""

import numpy as np
import pytest
import torch

from oracle import c_oracle
from oracle import reference as R


def _case(rng, B, ctxs, chunks, Hq=8, Hkv=2, D=32, dtype="f32"):
    mb = max(-(-c // 16) for c in ctxs)
    nb = sum(-(-c // 16) for c in ctxs) + 3
    perm = rng.permutation(nb)
    bt = np.full((B, mb), -1, dtype=np.int32)
    k = 0
    for b, c in enumerate(ctxs):
        for j in range(-(-c // 16)):
            bt[b, j] = perm[k]
            k += 1
    kc = rng.standard_normal((nb, Hkv, 16, D)).astype(np.float32)
    vc = rng.standard_normal((nb, Hkv, 16, D)).astype(np.float32)
    qs = np.concatenate([[0], np.cumsum(chunks)]).astype(np.int32)
    q = rng.standard_normal((int(qs[-1]), Hq, D)).astype(np.float32)
    return q, kc, vc, bt, qs, np.array(ctxs, dtype=np.int32)


def _contiguous(cache, bt, b, n):
    return np.stack([cache[bt[b, i // 16], :, i % 16] for i in range(n)], axis=1)   # [Hkv, n, D]


def test_first_token_sees_only_itself_and_last_row_is_the_decode():
    rng = np.random.default_rng(0)
    q, kc, vc, bt, qs, cl = _case(rng, 2, [37, 20], [37, 20])
    out = R.prefill(q, kc, vc, bt, qs, cl, 0.2, "f32", 2)
    G = 4
    for b in range(2):
        first = out[qs[b]]
        for h in range(8):
            assert np.allclose(first[h], vc[bt[b, 0], h // G, 0], atol=1e-12)
        last = out[qs[b + 1] - 1]
        dec = R.decode(q[qs[b + 1] - 1:qs[b + 1]], kc, vc, bt[b:b + 1], cl[b:b + 1], 0.2, "f32", 2)[0]
        assert np.allclose(last, dec, atol=1e-12)


def test_equals_causal_sdpa_on_contiguous_kv():
    rng = np.random.default_rng(1)
    n = 53
    q, kc, vc, bt, qs, cl = _case(rng, 1, [n], [n], Hq=6, Hkv=2, D=16)
    out = R.prefill(q, kc, vc, bt, qs, cl, 0.25, "f32", 2)
    K = torch.from_numpy(_contiguous(kc, bt, 0, n)).double().repeat_interleave(3, dim=0)
    V = torch.from_numpy(_contiguous(vc, bt, 0, n)).double().repeat_interleave(3, dim=0)
    Q = torch.from_numpy(q).double().permute(1, 0, 2)                     # [Hq, n, D]
    ref = torch.nn.functional.scaled_dot_product_attention(Q, K, V, is_causal=True, scale=0.25)
    assert np.allclose(out, ref.permute(1, 0, 2).numpy(), atol=1e-12)


def test_a_chunk_equals_the_rows_of_the_whole_prefill():
    rng = np.random.default_rng(2)
    n, L = 70, 19
    q, kc, vc, bt, qs, cl = _case(rng, 1, [n], [n])
    full = R.prefill(q, kc, vc, bt, qs, cl, 0.3, "f32", 2)
    qs2 = np.array([0, L], dtype=np.int32)
    chunk = R.prefill(q[n - L:], kc, vc, bt, qs2, cl, 0.3, "f32", 2)
    assert np.allclose(chunk, full[n - L:], atol=1e-12)


@pytest.mark.parametrize("dtype", ["f32", "f16"])
def test_c_oracle_agrees(dtype):
    rng = np.random.default_rng(3)
    q, kc, vc, bt, qs, cl = _case(rng, 3, [40, 17, 90], [5, 17, 33])
    if dtype == "f16":
        q, kc, vc = q.astype(np.float16), kc.astype(np.float16), vc.astype(np.float16)
    a = R.prefill(q, kc, vc, bt, qs, cl, 0.2, dtype, 2)
    b = c_oracle.prefill(q, kc, vc, bt, qs, cl, 0.2, dtype, 2)
    assert np.allclose(a, b, atol=1e-12)
