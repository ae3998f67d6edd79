"""The C-ABI library loads, exports every declared symbol, and rejects bad host-side arguments.

CPU only: every call here returns during host-side validation, before any CUDA call.
"""

import ctypes
import glob
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions(header=None):
    """Function names declared in include/*.h (or one header), comments stripped."""
    names = set()
    for h in sorted(glob.glob(os.path.join(ROOT, "include", header or "*.h"))):
        src = re.sub(r"/\*.*?\*/", "", open(h).read(), flags=re.S)
        names.update(re.findall(r"\b(pa_[a-z_0-9]+)\s*\(", src))
    return sorted(names)


def test_header_declares_the_boundary():
    names = _declared_functions("pa.h")
    for n in ("pa_reshape_and_cache", "pa_decode", "pa_decode_workspace_size", "pa_copy_blocks",
              "pa_get_error_string", "pa_swap_blocks", "pa_prefill"):
        assert n in names
    bm = _declared_functions("pa_block_manager.h")
    for n in ("pa_bm_create", "pa_bm_append_tokens", "pa_bm_fork", "pa_bm_swap_out", "pa_bm_block_tables"):
        assert n in bm


def test_library_exports_every_declared_symbol():
    import paged_kv_cache_362_b200 as pa

    lib = ctypes.CDLL(pa.LIB_PATH)
    missing = [n for n in _declared_functions() if not hasattr(lib, n)]
    assert not missing, missing


def test_error_strings_and_version():
    import paged_kv_cache_362_b200 as pa

    assert pa.error_string(0) == "PA_OK"
    for code, word in ((1, "INVALID_ARG"), (2, "UNSUPPORTED"), (4, "OUT_OF_RANGE"), (8, "CUDA"), (16, "TIMEOUT")):
        assert word in pa.error_string(code)
    assert pa.version() >= 100


def test_workspace_size_is_consistent():
    import paged_kv_cache_362_b200 as pa

    lib = pa._lib.LIB
    # invalid arguments -> 0
    assert lib.pa_decode_workspace_size(4, 28, 4, 128, 100, 24) == 0      # not a multiple of 16
    assert lib.pa_decode_workspace_size(4, 28, 4, 128, 100, 1024) == 0    # above 512
    assert lib.pa_decode_workspace_size(-1, 28, 4, 128, 100, 0) == 0
    # one partition -> no partial buffers: header, the fixed 16384-entry merge
    # counter region (int32) and the item list
    counters = 16384 * 4
    small = lib.pa_decode_workspace_size(8, 28, 4, 128, 512, 512)
    assert 256 + counters < small < 256 + counters + 4096
    # the counter region grows with the (sequence, KV head) pairs beyond that
    huge = lib.pa_decode_workspace_size(8192, 32, 8, 128, 16, 16)
    assert huge >= 256 + 8192 * 8 * 4 + 8192 * 8 * 16
    # 32k context, 512-token partitions: 64 partials of (D + 2) floats per (seq, head)
    big = lib.pa_decode_workspace_size(8, 28, 4, 128, 32768, 512)
    assert big >= 8 * 28 * 64 * (128 + 2) * 4
    assert big % 256 == 0


P = ctypes.c_void_p
FAKE = P(0x1000)          # never dereferenced: every call below fails validation first


def _rc(*args):
    import paged_kv_cache_362_b200 as pa

    return pa._lib.LIB.pa_reshape_and_cache(*args)


def test_reshape_and_cache_validation():
    import paged_kv_cache_362_b200 as pa

    ok = dict(key=FAKE, value=FAKE, kc=FAKE, vc=FAKE, slots=FAKE)
    args = lambda **o: [o.get("key", FAKE), o.get("value", FAKE), o.get("kc", FAKE), o.get("vc", FAKE),
                        o.get("slots", FAKE), o.get("T", 4), o.get("NB", 8), o.get("Hkv", 2), o.get("D", 64),
                        o.get("bs", 16), o.get("dt", 1), None, None]
    for bs in (4, 12, 64):                                      # block sizes: 8, 16 and 32 only
        assert _rc(*args(bs=bs)) == pa.PA_ERR_UNSUPPORTED
    for bs in (8, 32):                                          # supported: fails on the null key instead
        assert _rc(*args(bs=bs, key=P(0))) == pa.PA_ERR_INVALID_ARG
    assert _rc(*args(D=96)) == pa.PA_ERR_UNSUPPORTED
    assert _rc(*args(T=-1)) == pa.PA_ERR_INVALID_ARG
    assert _rc(*args(key=P(0))) == pa.PA_ERR_INVALID_ARG
    assert _rc(*args(slots=P(0))) == pa.PA_ERR_INVALID_ARG
    assert _rc(*args(dt=7)) == pa.PA_ERR_INVALID_ARG
    assert _rc(*args(kc=P(0x1008))) == pa.PA_ERR_INVALID_ARG   # not 16-byte aligned
    assert _rc(*args(T=0)) == pa.PA_OK                          # nothing to do
    del ok


def _dec(**o):
    import paged_kv_cache_362_b200 as pa

    a = [o.get("out", FAKE), o.get("q", FAKE), o.get("kc", FAKE), o.get("vc", FAKE), o.get("bt", FAKE),
         o.get("MB", 4), o.get("cl", FAKE), o.get("B", 2), o.get("Hq", 4), o.get("Hkv", 2), o.get("D", 64),
         o.get("bs", 16), o.get("NB", 8), ctypes.c_float(o.get("scale", 0.125)), o.get("maxctx", 64),
         o.get("P", 0), o.get("ws", P(0x100000)), o.get("wsb", 1 << 20), o.get("dt", 1), None, None]
    return pa._lib.LIB.pa_decode(*a)


def test_decode_validation():
    import paged_kv_cache_362_b200 as pa

    assert _dec(Hq=5) == pa.PA_ERR_INVALID_ARG               # Hq not a multiple of Hkv
    for bs in (4, 24, 64):
        assert _dec(bs=bs) == pa.PA_ERR_UNSUPPORTED
    for bs in (8, 32):
        assert _dec(bs=bs, out=P(0)) == pa.PA_ERR_INVALID_ARG
    # pool rows (blocks x KV heads x block size) index the tensor copies in int32
    assert _dec(bs=32, NB=1 << 25) == pa.PA_ERR_UNSUPPORTED
    assert _dec(D=80) == pa.PA_ERR_UNSUPPORTED
    assert _dec(Hkv=256, Hq=256) == pa.PA_ERR_UNSUPPORTED
    assert _dec(P=24) == pa.PA_ERR_INVALID_ARG
    assert _dec(P=1024) == pa.PA_ERR_INVALID_ARG
    assert _dec(out=P(0)) == pa.PA_ERR_INVALID_ARG
    assert _dec(ws=P(0)) == pa.PA_ERR_INVALID_ARG
    assert _dec(ws=P(0x100010)) == pa.PA_ERR_INVALID_ARG     # workspace not 256-byte aligned
    assert _dec(q=P(0x1004)) == pa.PA_ERR_INVALID_ARG
    assert _dec(wsb=16) == pa.PA_ERR_INVALID_ARG             # workspace too small
    assert _dec(scale=float("nan")) == pa.PA_ERR_INVALID_ARG
    assert _dec(maxctx=-1) == pa.PA_ERR_INVALID_ARG
    assert _dec(B=0) == pa.PA_OK


def test_decode_tuned_validation():
    """pa_decode_tuned checks its options on the host before anything else; NULL options are pa_decode."""
    import paged_kv_cache_362_b200 as pa

    f = pa._lib.LIB.pa_decode_tuned

    def dec_t(t, **o):
        a = [o.get("out", FAKE), FAKE, FAKE, FAKE, FAKE, 4, FAKE, o.get("B", 2), 4, 2, 64, 16, 8,
             ctypes.c_float(0.125), 64, 0, P(0x100000), 1 << 20, 1, None, None, None if t is None else ctypes.byref(t)]
        return f(*a)

    for bad in (pa.tuning(shape=5), pa.tuning(shape=-1), pa.tuning(planner=2), pa.tuning(split=-1),
                pa.tuning(order=3), pa.tuning(wait_limit_ns=-5), pa.tuning(stall_first_item=2)):
        assert dec_t(bad) == pa.PA_ERR_INVALID_ARG
    # valid options fall through to pa_decode's own checks
    assert dec_t(pa.tuning(shape="paired"), out=P(0)) == pa.PA_ERR_INVALID_ARG
    assert dec_t(None, B=0) == pa.PA_OK
    assert dec_t(pa.tuning(shape="pair1", planner=1, split=1, order=1, wait_limit_ns=1000), B=0) == pa.PA_OK
    lc = pa._lib.LIB.pa_decode_launch_count_tuned
    assert lc(8, 28, 4, 128, 4096, 512, 1, ctypes.byref(pa.tuning(shape=7))) == -1


def test_decode_planned_validation():
    """pa_decode_planned validates exactly as pa_decode does, on the host, before any launch."""
    import paged_kv_cache_362_b200 as pa

    f = pa._lib.LIB.pa_decode_planned

    def dec_p(**o):
        a = [o.get("out", FAKE), o.get("q", FAKE), FAKE, FAKE, FAKE, 4, FAKE, o.get("B", 2), o.get("Hq", 4), 2,
             o.get("D", 64), o.get("bs", 16), 8, ctypes.c_float(o.get("scale", 0.125)), 64, o.get("P", 0),
             o.get("ws", P(0x100000)), o.get("wsb", 1 << 20), 1, None, None]
        return f(*a)

    assert dec_p(Hq=5) == pa.PA_ERR_INVALID_ARG
    assert dec_p(bs=4) == pa.PA_ERR_UNSUPPORTED
    assert dec_p(D=80) == pa.PA_ERR_UNSUPPORTED
    assert dec_p(P=24) == pa.PA_ERR_INVALID_ARG
    assert dec_p(out=P(0)) == pa.PA_ERR_INVALID_ARG
    assert dec_p(q=P(0x1004)) == pa.PA_ERR_INVALID_ARG
    assert dec_p(ws=P(0x100010)) == pa.PA_ERR_INVALID_ARG
    assert dec_p(wsb=16) == pa.PA_ERR_INVALID_ARG
    assert dec_p(scale=float("nan")) == pa.PA_ERR_INVALID_ARG
    assert dec_p(B=0) == pa.PA_OK
    assert pa._lib.LIB.pa_decode_planned_launch_count(8, 28, 5, 128, 4096, 512, 1) == -1   # Hq % Hkv != 0
    assert pa._lib.LIB.pa_decode_planned_launch_count(8, 28, 4, 80, 4096, 512, 1) == -1    # head_dim


def test_decode_plan_validation():
    """pa_decode_plan checks what it reads (context_lens, sizes, workspace) on the host, before its launch."""
    import paged_kv_cache_362_b200 as pa

    f = pa._lib.LIB.pa_decode_plan

    def plan(**o):
        return f(o.get("cl", FAKE), o.get("B", 2), o.get("Hq", 4), o.get("Hkv", 2), o.get("D", 64), o.get("bs", 16),
                 o.get("MB", 4), o.get("maxctx", 64), o.get("P", 0), o.get("ws", P(0x100000)), o.get("wsb", 1 << 20),
                 None, None)

    assert plan(Hq=5) == pa.PA_ERR_INVALID_ARG
    assert plan(B=-1) == pa.PA_ERR_INVALID_ARG
    assert plan(MB=0) == pa.PA_ERR_INVALID_ARG
    assert plan(maxctx=-1) == pa.PA_ERR_INVALID_ARG
    for bs in (4, 24, 64):
        assert plan(bs=bs) == pa.PA_ERR_UNSUPPORTED
    assert plan(D=80) == pa.PA_ERR_UNSUPPORTED
    assert plan(Hkv=256, Hq=256) == pa.PA_ERR_UNSUPPORTED
    assert plan(P=24) == pa.PA_ERR_INVALID_ARG
    assert plan(P=1024) == pa.PA_ERR_INVALID_ARG
    assert plan(cl=P(0)) == pa.PA_ERR_INVALID_ARG
    assert plan(ws=P(0)) == pa.PA_ERR_INVALID_ARG
    assert plan(ws=P(0x100010)) == pa.PA_ERR_INVALID_ARG
    assert plan(wsb=16) == pa.PA_ERR_INVALID_ARG
    assert plan(B=0, cl=P(0), ws=P(0)) == pa.PA_OK      # nothing to plan: no pointer is read


def test_copy_blocks_validation():
    import paged_kv_cache_362_b200 as pa

    lib = pa._lib.LIB
    assert lib.pa_copy_blocks(FAKE, FAKE, FAKE, -1, 8, 2, 64, 16, 1, None, None) == pa.PA_ERR_INVALID_ARG
    assert lib.pa_copy_blocks(FAKE, FAKE, P(0), 3, 8, 2, 64, 16, 1, None, None) == pa.PA_ERR_INVALID_ARG
    assert lib.pa_copy_blocks(FAKE, FAKE, FAKE, 3, 8, 2, 64, 12, 1, None, None) == pa.PA_ERR_UNSUPPORTED
    assert lib.pa_copy_blocks(FAKE, FAKE, FAKE, 0, 8, 2, 64, 16, 1, None, None) == pa.PA_OK


def test_prefill_and_swap_validation():
    import paged_kv_cache_362_b200 as pa

    lib = pa._lib.LIB
    pf = lambda bs, dt=1, out=FAKE: lib.pa_prefill(out, FAKE, FAKE, FAKE, FAKE, 4, FAKE, FAKE, 2, 4, 2, 64, bs, 8,
                                                   ctypes.c_float(0.125), 16, dt, None, None)
    assert pf(8) == pa.PA_ERR_UNSUPPORTED                   # prefill reads 16-token blocks only
    assert pf(32) == pa.PA_ERR_UNSUPPORTED
    assert pf(16, dt=0) == pa.PA_ERR_UNSUPPORTED            # float32
    assert pf(16, out=P(0)) == pa.PA_ERR_INVALID_ARG
    sw = lambda bs, n=3: lib.pa_swap_blocks(FAKE, FAKE, FAKE, FAKE, P(0), n, 8, 8, 2, 64, bs, 1, None, None)
    assert sw(12) == pa.PA_ERR_UNSUPPORTED
    for bs in (8, 16, 32):
        assert sw(bs) == pa.PA_ERR_INVALID_ARG              # null pairs
        assert sw(bs, n=0) == pa.PA_OK


def test_prefill_workspace_size_and_validation():
    """pa_prefill_ws's workspace: the tiles of the last, partial wave (one CTA per SM; 148 SMs when no
    device can be queried) split into up to 16 pieces; none when the tiles fill whole waves."""
    import paged_kv_cache_362_b200 as pa

    lib = pa._lib.LIB
    n = ctypes.c_size_t(0)

    def size(B, Hq, Hkv, D, L, dt=2):
        rc = lib.pa_prefill_workspace_size(B, Hq, Hkv, D, L, dt, ctypes.byref(n))
        return rc, n.value

    # 4 x 512 queries, 28/4 heads, D 128: 28 tiles x 4 KV heads x 4 = 448 items = 3 x 148 + 4;
    # the 4 are split 16 ways: 4 x 16 x 128 partial rows of 128 + 4 floats
    assert size(4, 28, 4, 128, 512) == (pa.PA_OK, 4 * 16 * 128 * 132 * 4)
    assert size(1, 28, 4, 128, 512)[1] == 0          # 112 items: one wave
    assert size(2, 28, 4, 128, 676)[1] == 0          # 37 tiles x 8 = 296 items: two whole waves
    assert size(4, 28, 4, 128, 4)[1] == 0            # 4 x 7 rows < 32: the mma.sync kernel
    assert size(0, 28, 4, 128, 512) == (pa.PA_OK, 0)
    assert size(4, 28, 4, 96, 512)[0] == pa.PA_ERR_UNSUPPORTED
    assert size(4, 28, 4, 128, 512, dt=0)[0] == pa.PA_ERR_UNSUPPORTED
    assert lib.pa_prefill_workspace_size(4, 28, 4, 128, 512, 2, None) == pa.PA_ERR_INVALID_ARG
    need = size(4, 28, 4, 128, 512)[1]
    ws = lambda wsp, nbytes: lib.pa_prefill_ws(FAKE, FAKE, FAKE, FAKE, FAKE, 256, FAKE, FAKE, 4, 28, 4, 128, 16, 1000,
                                                ctypes.c_float(0.088), 512, wsp, nbytes, 2, None, None)
    assert ws(None, 0) == pa.PA_ERR_INVALID_ARG              # a workspace is needed for these sizes
    assert ws(FAKE, need - 1) == pa.PA_ERR_INVALID_ARG       # too small


def test_host_copy_pair_checker():
    import numpy as np

    import paged_kv_cache_362_b200 as pa

    pa.check_copy_pairs(np.array([[1, 3], [1, 4]]), 8)
    with pytest.raises(ValueError):
        pa.check_copy_pairs(np.array([[1, 3], [2, 3]]), 8)     # repeated dst
    with pytest.raises(ValueError):
        pa.check_copy_pairs(np.array([[1, 3], [3, 4]]), 8)     # dst that is also a src
    with pytest.raises(ValueError):
        pa.check_copy_pairs(np.array([[1, 9]]), 8)


def test_auto_partition_size():
    """partition_size 0: enough items for every SM, and no reduce kernel where one wave of CTAs still fills."""
    import paged_kv_cache_362_b200 as pa

    ws = lambda B, mc, P: pa._lib.LIB.pa_decode_workspace_size(B, 28, 4, 128, mc, P)
    # 32 sequences of up to 2048 tokens: 256-token partitions (8 per sequence, merged by the attention kernel),
    # not the 128 that the item count alone would pick
    assert ws(32, 2048, 0) == ws(32, 2048, 256) != ws(32, 2048, 128)
    # 256 sequences of up to 4096 tokens, 8 of up to 32768: 512
    assert ws(256, 4096, 0) == ws(256, 4096, 512) != ws(256, 4096, 256)
    assert ws(8, 32768, 0) == ws(8, 32768, 512)
    # one sequence of 2048: 64-token partitions, the smallest, since even they give too few items
    assert ws(1, 2048, 0) == ws(1, 2048, 64) != ws(1, 2048, 128)
