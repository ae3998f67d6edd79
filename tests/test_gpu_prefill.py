"""GPU parity of paged prefill (pa_prefill) against the fp64 oracle.

Whole prompts and chunks on top of an existing context, ragged chunk lengths
(1, 15, 16, 17, ...), GQA groups 1 to 16, head_dim 64 and 128, fp16 and bf16;
every output element is compared.  Also: a bad block id is flagged and
contributes nothing, the result does not depend on where blocks live, NaN in
every pool slot no query reads never reaches a result, and negative and zero
scales.  Chunks that fill a 128-row tile run on the tcgen05 kernel; chunks of
a few tokens (query rows x group < 32) on the mma.sync kernel, and both are
covered.
"""

import numpy as np
import pytest

from oracle import c_oracle
from parity import compare, out_f64, to_device

pytestmark = pytest.mark.gpu


def _case(rng, ctxs, chunks, Hq, Hkv, D, dtype, extra_blocks=3):
    B = len(ctxs)
    mb = max(-(-c // 16) for c in ctxs)
    nb = sum(-(-c // 16) for c in ctxs) + extra_blocks
    perm = rng.permutation(nb)
    bt = np.full((B, mb), -1, dtype=np.int32)
    k = 0
    for b, c in enumerate(ctxs):
        for j in range(-(-c // 16)):
            bt[b, j] = perm[k]
            k += 1
    npdt = np.float16 if dtype == "f16" else np.float32

    def draw(shape):
        x = rng.standard_normal(shape).astype(np.float32)
        return x.astype(np.float16) if dtype == "f16" else (x.view(np.uint32) >> 16).astype(np.uint16)

    kc, vc = draw((nb, Hkv, 16, D)), draw((nb, Hkv, 16, D))
    qs = np.concatenate([[0], np.cumsum(chunks)]).astype(np.int32)
    q = draw((int(qs[-1]), Hq, D))
    del npdt
    return q, kc, vc, bt, qs, np.array(ctxs, dtype=np.int32)


def _run(q, kc, vc, bt, qs, cl, scale, dtype, status=None, workspace=None):
    import torch

    import paged_kv_cache_362_b200 as pa

    out = torch.full(q.shape, float("nan"), dtype=torch.float16 if dtype == "f16" else torch.bfloat16,
                     device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda") if status is None else status
    pa.prefill(out, to_device(q, dtype), to_device(kc, dtype), to_device(vc, dtype), torch.from_numpy(bt).cuda(),
               torch.from_numpy(qs).cuda(), torch.from_numpy(cl).cuda(), scale, int(np.diff(qs).max()), status=st,
               workspace=workspace)
    torch.cuda.synchronize()
    return out, int(st.item())


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
@pytest.mark.parametrize("heads", [(28, 4), (8, 8), (16, 2), (32, 2)], ids=lambda h: f"{h[0]}x{h[1]}")
@pytest.mark.parametrize("D", [64, 128])
def test_prompts_and_chunks_every_element(dtype, heads, D):
    Hq, Hkv = heads
    rng = np.random.default_rng(Hq + D)
    # (context, new tokens): whole prompts, chunks on a context, ragged lengths around 16
    ctxs = [1, 15, 17, 64, 300, 96, 129, 40]
    chunks = [1, 15, 16, 33, 300, 17, 1, 40]
    q, kc, vc, bt, qs, cl = _case(rng, ctxs, chunks, Hq, Hkv, D, dtype)
    scale = 1.0 / np.sqrt(D)
    out, st = _run(q, kc, vc, bt, qs, cl, scale, dtype)
    assert st == 0
    ref = c_oracle.prefill(q, kc, vc, bt, qs, cl, scale, dtype, Hkv)
    compare(out_f64(out), ref, dtype, f"{dtype} {heads} D={D}")


def test_long_chunk_on_long_context():
    rng = np.random.default_rng(7)
    ctxs, chunks = [4096, 2500], [512, 700]
    q, kc, vc, bt, qs, cl = _case(rng, ctxs, chunks, 28, 4, 128, "bf16")
    out, st = _run(q, kc, vc, bt, qs, cl, 1 / np.sqrt(128), "bf16")
    assert st == 0
    ref = c_oracle.prefill(q, kc, vc, bt, qs, cl, 1 / np.sqrt(128), "bf16", 4)
    compare(out_f64(out), ref, "bf16", "long")


def test_placement_does_not_change_the_bits():
    import torch

    rng = np.random.default_rng(9)
    q, kc, vc, bt, qs, cl = _case(rng, [200, 90], [200, 30], 28, 4, 128, "f16")
    a, _ = _run(q, kc, vc, bt, qs, cl, 0.09, "f16")
    perm = rng.permutation(kc.shape[0])
    kc2, vc2 = np.empty_like(kc), np.empty_like(vc)
    kc2[perm], vc2[perm] = kc, vc
    bt2 = np.where(bt >= 0, perm[np.maximum(bt, 0)], -1).astype(np.int32)
    b, _ = _run(q, kc2, vc2, bt2, qs, cl, 0.09, "f16")
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_bad_block_flagged_and_skipped():
    import paged_kv_cache_362_b200 as pa

    rng = np.random.default_rng(4)
    q, kc, vc, bt, qs, cl = _case(rng, [64], [20], 8, 2, 64, "f16")
    bt_bad = bt.copy()
    bt_bad[0, 1] = 10_000            # keys 16..31 are unreachable
    out, st = _run(q, kc, vc, bt_bad, qs, cl, 0.125, "f16")
    assert st & pa.PA_ERR_OUT_OF_RANGE
    # the oracle without those 16 keys: rows see their visible keys except positions 16..31
    from oracle import reference as R

    seqs, pos = R.prefill_rows(qs, cl)
    got = out_f64(out)
    for t, p_ in enumerate(pos):
        keys = [i for i in range(int(p_) + 1) if not 16 <= i < 32]
        K = np.stack([kc[bt[0, i // 16], :, i % 16] for i in keys], axis=1).astype(np.float64)
        V = np.stack([vc[bt[0, i // 16], :, i % 16] for i in keys], axis=1).astype(np.float64)
        ref = np.stack([R.attention_f64(q[t, h].astype(np.float64), K[h // 4], V[h // 4], 0.125) for h in range(8)])
        compare(got[t], ref, "f16", f"row {t}")


def _poison_unread(kc, vc, bt, ctxs):
    """NaN into every slot of the pools that no query of these contexts reads."""
    nan = np.float16("nan") if kc.dtype == np.float16 else np.uint16(0x7FC1)
    used = np.zeros((kc.shape[0], 16), dtype=bool)
    for b, c in enumerate(ctxs):
        for i in range(c):
            used[bt[b, i // 16], i % 16] = True
    blk, off = np.nonzero(~used)
    kc[blk, :, off, :] = nan
    vc[blk, :, off, :] = nan
    return int(blk.size)


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
@pytest.mark.parametrize("heads", [(28, 4), (32, 2)], ids=lambda h: f"{h[0]}x{h[1]}")
def test_nan_in_unread_slots_never_reaches_a_result(dtype, heads):
    Hq, Hkv = heads
    rng = np.random.default_rng(31 + Hq)
    ctxs, chunks = [300, 129, 17, 260, 1000], [300, 100, 17, 3, 333]
    q, kc, vc, bt, qs, cl = _case(rng, ctxs, chunks, Hq, Hkv, 128, dtype, extra_blocks=5)
    ref = c_oracle.prefill(q, kc, vc, bt, qs, cl, 1 / np.sqrt(128), dtype, Hkv)
    assert _poison_unread(kc, vc, bt, ctxs) > 0
    out, st = _run(q, kc, vc, bt, qs, cl, 1 / np.sqrt(128), dtype)
    assert st == 0
    compare(out_f64(out), ref, dtype, f"{dtype} {heads} NaN-filled unread slots")


@pytest.mark.parametrize("heads", [(28, 4), (8, 8), (16, 16)], ids=lambda h: f"{h[0]}x{h[1]}")
def test_short_chunks_take_the_mma_sync_kernel(heads):
    """Chunks of a few tokens per sequence (query rows x group < 32): the 16-query mma.sync kernel."""
    Hq, Hkv = heads
    rng = np.random.default_rng(5 + Hq)
    G = Hq // Hkv
    L = max(1, min(4, 31 // G))
    ctxs = [L, 40, 700, 17]
    chunks = [L, L, 1, L]
    assert max(chunks) * G < 32
    q, kc, vc, bt, qs, cl = _case(rng, ctxs, chunks, Hq, Hkv, 128, "bf16")
    _poison_unread(kc, vc, bt, ctxs)
    out, st = _run(q, kc, vc, bt, qs, cl, 1 / np.sqrt(128), "bf16")
    assert st == 0
    # the oracle reads only the contexts, so the poisoned slots cannot enter it
    ref = c_oracle.prefill(q, kc, vc, bt, qs, cl, 1 / np.sqrt(128), "bf16", Hkv)
    compare(out_f64(out), ref, "bf16", f"short chunks {heads}")


@pytest.mark.parametrize("scale", [-0.0884, 0.0, 0.3])
def test_negative_zero_and_large_scales(scale):
    rng = np.random.default_rng(77)
    ctxs, chunks = [200, 333], [200, 150]
    q, kc, vc, bt, qs, cl = _case(rng, ctxs, chunks, 28, 4, 128, "f16")
    out, st = _run(q, kc, vc, bt, qs, cl, scale, "f16")
    assert st == 0
    ref = c_oracle.prefill(q, kc, vc, bt, qs, cl, scale, "f16", 4)
    compare(out_f64(out), ref, "f16", f"scale {scale}")


def test_bad_block_on_the_diagonal_of_a_tensor_core_tile():
    """A bad id inside the 128-key step that holds the tile's own positions: masked and skipped, the rest exact."""
    import paged_kv_cache_362_b200 as pa
    from oracle import reference as R

    rng = np.random.default_rng(12)
    q, kc, vc, bt, qs, cl = _case(rng, [400], [300], 28, 4, 128, "bf16")
    bt_bad = bt.copy()
    bt_bad[0, 9] = -7                 # keys 144..159
    out, st = _run(q, kc, vc, bt_bad, qs, cl, 0.0884, "bf16")
    assert st & pa.PA_ERR_OUT_OF_RANGE
    got = out_f64(out)
    seqs, pos = R.prefill_rows(qs, cl)
    rows = list(range(0, 300, 7)) + [299]
    for t in rows:
        p_ = int(pos[t])
        keys = [i for i in range(p_ + 1) if not 144 <= i < 160]
        K = np.stack([kc[bt[0, i // 16], :, i % 16] for i in keys], axis=1)
        V = np.stack([vc[bt[0, i // 16], :, i % 16] for i in keys], axis=1)
        K = (K.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
        V = (V.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
        qt = (q[t].astype(np.uint32) << 16).view(np.float32).astype(np.float64)
        ref = np.stack([R.attention_f64(qt[h], K[h // 7], V[h // 7], 0.0884) for h in range(28)])
        compare(got[t], ref, "bf16", f"row {t}")


def test_prefill_kernel_choice():
    """The shape rule: tensor-core tiles when the chunk fills at least a quarter of a 128-row tile."""
    rng = np.random.default_rng(3)
    # both paths on one problem size: identical results within tolerance of the oracle
    for chunks in ([4, 4], [40, 40]):
        q, kc, vc, bt, qs, cl = _case(rng, [100, 64], chunks, 28, 4, 128, "f16")
        out, st = _run(q, kc, vc, bt, qs, cl, 0.0884, "f16")
        assert st == 0
        compare(out_f64(out), c_oracle.prefill(q, kc, vc, bt, qs, cl, 0.0884, "f16", 4), "f16", f"chunks {chunks}")


def _sm_count():
    import torch

    return torch.cuda.get_device_properties(0).multi_processor_count


@pytest.mark.parametrize("ctx_last", [620, 3000], ids=["pieces-mostly-empty", "pieces-of-1-2-tiles"])
def test_split_last_wave_every_element(ctx_last):
    """pa_prefill_ws: 4 chunks of 512 rows x 7 heads = 448 tiles, 3 waves of 148 and 4 tiles split by key
    range into pieces whose partial rows a second kernel merges.  With a short last context most pieces
    hold no key tile (the merge must skip them); with a long one each holds one or two.  Two calls in a
    row on the same workspace, every element against the oracle, the two results bit-identical, and the
    call without a workspace agrees within the tolerance."""
    import torch

    import paged_kv_cache_362_b200 as pa

    rng = np.random.default_rng(ctx_last)
    ctxs, chunks = [1500, 900, 2100, ctx_last], [512, 512, 512, 512]
    q, kc, vc, bt, qs, cl = _case(rng, ctxs, chunks, 28, 4, 128, "bf16")
    need = pa.prefill_workspace_size(4, 28, 4, 128, 512, "bf16")
    if _sm_count() != 148:
        pytest.skip("the split sizes here assume 148 SMs")
    assert need == 4 * 16 * 128 * 132 * 4
    ws = torch.full((need,), 0xFF, dtype=torch.uint8, device="cuda")   # scratch: any contents
    scale = 1.0 / np.sqrt(128)
    ref = c_oracle.prefill(q, kc, vc, bt, qs, cl, scale, "bf16", 4)
    out1, st1 = _run(q, kc, vc, bt, qs, cl, scale, "bf16", workspace=ws)
    out2, st2 = _run(q, kc, vc, bt, qs, cl, scale, "bf16", workspace=ws)
    assert st1 == 0 and st2 == 0
    compare(out_f64(out1), ref, "bf16", f"split, last context {ctx_last}")
    assert torch.equal(out1.view(torch.int16), out2.view(torch.int16))
    out0, st0 = _run(q, kc, vc, bt, qs, cl, scale, "bf16")
    assert st0 == 0
    compare(out_f64(out0), ref, "bf16", f"unsplit, last context {ctx_last}")


def test_split_workspace_too_small_is_rejected():
    import torch

    import paged_kv_cache_362_b200 as pa

    if _sm_count() != 148:
        pytest.skip("the split sizes here assume 148 SMs")
    rng = np.random.default_rng(5)
    q, kc, vc, bt, qs, cl = _case(rng, [600] * 4, [512] * 4, 28, 4, 128, "bf16")
    need = pa.prefill_workspace_size(4, 28, 4, 128, 512, "bf16")
    ws = torch.zeros(need - 16, dtype=torch.uint8, device="cuda")
    with pytest.raises(pa.PagedAttentionError):
        _run(q, kc, vc, bt, qs, cl, 0.088, "bf16", workspace=ws)
