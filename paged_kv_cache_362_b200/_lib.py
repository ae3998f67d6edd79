"""ctypes binding of libpa.so: argument marshalling only.

Every step of the path runs in the library's CUDA kernels.  These wrappers
take torch tensors (which provide device memory and the current stream),
check shapes and dtypes, pass raw pointers to the C ABI declared in
include/pa.h, and raise on a non-zero status.  If the library is missing the
import fails loudly; there is no fallback.
"""

from __future__ import annotations

import ctypes
import os

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libpa.so")

PA_OK = 0
PA_ERR_INVALID_ARG = 1
PA_ERR_UNSUPPORTED = 2
PA_ERR_OUT_OF_RANGE = 4
PA_ERR_CUDA = 8
PA_ERR_TIMEOUT = 16
PA_ERR_NO_BLOCKS = 32

PA_F32, PA_F16, PA_BF16 = 0, 1, 2
BLOCK_SIZE = 16


class PagedAttentionError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {error_string(code)} (status {code})")


class DecodeTuning(ctypes.Structure):
    """pa_decode_tuning (include/pa_tuning.h): scheduling alternatives and fault-path test hooks.

    shape: 0 auto, 1 paired, 2 quad, 3 triple, 4 pair1; planner: 1 = always the planning kernel;
    split: 1 = near-equal partitions; order: 1 = all items by size; wait_limit_ns: bound of every wait
    in the attention kernel (0 = 2 s); stall_first_item: 1 = CTA 0 never publishes its first item.
    """

    _fields_ = [("shape", ctypes.c_int32), ("planner", ctypes.c_int32), ("split", ctypes.c_int32),
                ("order", ctypes.c_int32), ("wait_limit_ns", ctypes.c_int64), ("stall_first_item", ctypes.c_int32),
                ("reserved", ctypes.c_int32)]


SHAPES = {"auto": 0, "paired": 1, "quad": 2, "triple": 3, "pair1": 4}


def tuning(shape="auto", planner=0, split=0, order=0, wait_limit_ns=0, stall_first_item=0) -> DecodeTuning:
    return DecodeTuning(SHAPES[shape] if isinstance(shape, str) else int(shape), int(planner), int(split), int(order),
                        int(wait_limit_ns), int(stall_first_item), 0)


# Options that decode() and decode_launch_count() use when the caller gives
# none: None is the library's defaults.  The test suite sets it to run its
# parity cases under each scheduling alternative; nothing else should.
_default_tuning: DecodeTuning | None = None


def set_default_tuning(t: DecodeTuning | None) -> None:
    global _default_tuning
    _default_tuning = t


def _tuning_ptr(t):
    t = _default_tuning if t is None else t
    return None if t is None else ctypes.byref(t)


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is not built; run `python paged_kv_cache_362_b200/build.py`")
    lib = ctypes.CDLL(LIB_PATH)
    for sym in ("pa_reshape_and_cache", "pa_decode_workspace_size", "pa_decode", "pa_decode_launch_count",
                "pa_copy_blocks", "pa_get_error_string", "pa_version", "pa_bm_create", "pa_bm_append_tokens",
                "pa_prefill", "pa_swap_blocks", "pa_decode_tuned", "pa_decode_launch_count_tuned", "pa_prefill_ws",
                "pa_prefill_workspace_size", "pa_decode_plan", "pa_decode_planned", "pa_decode_planned_launch_count"):
        if not hasattr(lib, sym):
            raise ImportError(f"{LIB_PATH} lacks {sym} (stale build); run `python paged_kv_cache_362_b200/build.py`")
    p, i32, i64, f32, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t
    lib.pa_reshape_and_cache.argtypes = [p, p, p, p, p, i64, i32, i32, i32, i32, ctypes.c_int, p, p]
    lib.pa_reshape_and_cache.restype = ctypes.c_int
    lib.pa_decode_workspace_size.argtypes = [i32, i32, i32, i32, i32, i32]
    lib.pa_decode_workspace_size.restype = sz
    lib.pa_decode.argtypes = [p, p, p, p, p, i32, p, i32, i32, i32, i32, i32, i32, f32, i32, i32, p, sz,
                              ctypes.c_int, p, p]
    lib.pa_decode.restype = ctypes.c_int
    lib.pa_decode_launch_count.argtypes = [i32, i32, i32, i32, i32, i32, ctypes.c_int]
    lib.pa_decode_launch_count.restype = i32
    # scheduling options and fault-path test hooks (pa_tuning.h)
    lib.pa_decode_tuned.argtypes = lib.pa_decode.argtypes + [ctypes.POINTER(DecodeTuning)]
    lib.pa_decode_tuned.restype = ctypes.c_int
    lib.pa_decode_planned.argtypes = lib.pa_decode.argtypes
    lib.pa_decode_planned.restype = ctypes.c_int
    lib.pa_decode_plan.argtypes = [p, i32, i32, i32, i32, i32, i32, i32, i32, p, sz, p, p]
    lib.pa_decode_plan.restype = ctypes.c_int
    lib.pa_decode_planned_launch_count.argtypes = [i32, i32, i32, i32, i32, i32, ctypes.c_int]
    lib.pa_decode_planned_launch_count.restype = i32
    lib.pa_decode_launch_count_tuned.argtypes = [i32, i32, i32, i32, i32, i32, ctypes.c_int,
                                                 ctypes.POINTER(DecodeTuning)]
    lib.pa_decode_launch_count_tuned.restype = i32
    lib.pa_copy_blocks.argtypes = [p, p, p, i32, i32, i32, i32, i32, ctypes.c_int, p, p]
    lib.pa_copy_blocks.restype = ctypes.c_int
    # host block manager (pa_block_manager.h)
    lib.pa_bm_create.argtypes = [i32, i32, i32]
    lib.pa_bm_create.restype = p
    lib.pa_bm_destroy.argtypes = [p]
    lib.pa_bm_destroy.restype = None
    for fn in ("pa_bm_num_blocks", "pa_bm_num_free_blocks", "pa_bm_num_sequences", "pa_bm_num_free_host_blocks"):
        getattr(lib, fn).argtypes = [p]
        getattr(lib, fn).restype = i32
    lib.pa_bm_ref_count.argtypes = [p, i32]
    lib.pa_bm_ref_count.restype = i32
    lib.pa_bm_add_sequence.argtypes = [p, i64, i32, p]
    lib.pa_bm_add_sequence.restype = ctypes.c_int
    lib.pa_bm_fork.argtypes = [p, i64, i64]
    lib.pa_bm_fork.restype = ctypes.c_int
    lib.pa_bm_append_tokens.argtypes = [p, p, i32, p, p, p]
    lib.pa_bm_append_tokens.restype = ctypes.c_int
    lib.pa_bm_free_sequence.argtypes = [p, i64]
    lib.pa_bm_free_sequence.restype = ctypes.c_int
    for fn in ("pa_bm_swap_out", "pa_bm_swap_in"):
        getattr(lib, fn).argtypes = [p, i64, p, p]
        getattr(lib, fn).restype = ctypes.c_int
    lib.pa_bm_is_swapped.argtypes = [p, i64]
    lib.pa_bm_is_swapped.restype = i32
    lib.pa_prefill.argtypes = [p, p, p, p, p, i32, p, p, i32, i32, i32, i32, i32, i32, f32, i32, ctypes.c_int, p, p]
    lib.pa_prefill.restype = ctypes.c_int
    lib.pa_prefill_ws.argtypes = [p, p, p, p, p, i32, p, p, i32, i32, i32, i32, i32, i32, f32, i32, p, sz,
                                  ctypes.c_int, p, p]
    lib.pa_prefill_ws.restype = ctypes.c_int
    lib.pa_prefill_workspace_size.argtypes = [i32, i32, i32, i32, i32, ctypes.c_int, ctypes.POINTER(sz)]
    lib.pa_prefill_workspace_size.restype = ctypes.c_int
    lib.pa_swap_blocks.argtypes = [p, p, p, p, p, i32, i32, i32, i32, i32, i32, ctypes.c_int, p, p]
    lib.pa_swap_blocks.restype = ctypes.c_int
    lib.pa_bm_block_tables.argtypes = [p, p, i32, i32, p, p]
    lib.pa_bm_block_tables.restype = ctypes.c_int
    lib.pa_bm_sequence_blocks.argtypes = [p, i64]
    lib.pa_bm_sequence_blocks.restype = i32
    lib.pa_bm_sequence_length.argtypes = [p, i64]
    lib.pa_bm_sequence_length.restype = i64
    lib.pa_get_error_string.argtypes = [ctypes.c_int]
    lib.pa_get_error_string.restype = ctypes.c_char_p
    lib.pa_version.argtypes = []
    lib.pa_version.restype = i32
    return lib


LIB = _load()


def error_string(code: int) -> str:
    return LIB.pa_get_error_string(int(code)).decode()


def version() -> int:
    return int(LIB.pa_version())


def _check(code: int, where: str):
    if code != PA_OK:
        raise PagedAttentionError(code, where)


def _dtype_code(t) -> int:
    import torch

    return {torch.float32: PA_F32, torch.float16: PA_F16, torch.bfloat16: PA_BF16}[t.dtype]


def _stream(stream):
    import torch

    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t):
    return ctypes.c_void_p(0 if t is None else t.data_ptr())


def reshape_and_cache(key, value, key_cache, value_cache, slot_mapping, status=None, stream=None):
    """Write each token's K/V into its slot (pa_reshape_and_cache).

    key, value [T, Hkv, D]; key_cache, value_cache [NB, Hkv, block_size, D] (block_size 8, 16 or 32);
    slot_mapping int64 [T] (negative = skip); status: optional int32 device tensor.
    """
    assert key.is_contiguous() and value.is_contiguous() and key_cache.is_contiguous() and value_cache.is_contiguous()
    assert slot_mapping.dtype.is_floating_point is False and slot_mapping.element_size() == 8
    T, Hkv, D = key.shape
    NB, bs = key_cache.shape[0], key_cache.shape[2]
    assert value.shape == key.shape and key_cache.shape == (NB, Hkv, bs, D) == value_cache.shape
    assert key.dtype == value.dtype == key_cache.dtype == value_cache.dtype
    _check(LIB.pa_reshape_and_cache(_ptr(key), _ptr(value), _ptr(key_cache), _ptr(value_cache), _ptr(slot_mapping),
                                    T, NB, Hkv, D, bs, _dtype_code(key), _ptr(status), _stream(stream)),
           "pa_reshape_and_cache")


def decode_workspace_size(num_seqs, num_heads, num_kv_heads, head_dim, max_context_len, partition_size=0) -> int:
    n = int(LIB.pa_decode_workspace_size(num_seqs, num_heads, num_kv_heads, head_dim, max_context_len,
                                         partition_size))
    if n == 0:
        raise PagedAttentionError(PA_ERR_INVALID_ARG, "pa_decode_workspace_size")
    return n


def decode_launch_count(num_seqs, num_heads, num_kv_heads, head_dim, max_context_len, partition_size=0,
                        dtype="f16", tuning=None, planned=False) -> int:
    """Kernels one pa_decode (planned: pa_decode_planned) call enqueues for these sizes on the current device."""
    code = {"f32": 0, "f16": 1, "bf16": 2}[dtype]
    if planned:
        assert tuning is None, "a planned decode takes no tuning"
        n = int(LIB.pa_decode_planned_launch_count(num_seqs, num_heads, num_kv_heads, head_dim, max_context_len,
                                                   partition_size, code))
    else:
        n = int(LIB.pa_decode_launch_count_tuned(num_seqs, num_heads, num_kv_heads, head_dim, max_context_len,
                                                 partition_size, code, _tuning_ptr(tuning)))
    if n < 0:
        raise PagedAttentionError(PA_ERR_INVALID_ARG, "pa_decode_launch_count")
    return n


def make_workspace(num_seqs, num_heads, num_kv_heads, head_dim, max_context_len, partition_size=0, device=None):
    import torch

    n = decode_workspace_size(num_seqs, num_heads, num_kv_heads, head_dim, max_context_len, partition_size)
    # zero-filled: pa_decode keeps merge counters in it that must start at zero
    return torch.zeros(n, dtype=torch.uint8, device=device or "cuda")


def decode_plan(block_tables, context_lens, num_heads, num_kv_heads, head_dim, block_size, max_context_len,
                workspace, partition_size=0, status=None, stream=None):
    """The work list of a decode step into ``workspace`` (pa_decode_plan), for ``decode(..., planned=True)``.

    Sizes are those the planned decodes will pass: B = context_lens.shape[0] sequences, block_tables
    [B, max_blocks_per_seq].  Only context_lens is read.
    """
    assert context_lens.dtype.itemsize == 4 and context_lens.is_contiguous() and workspace.is_contiguous()
    B = context_lens.shape[0]
    assert block_tables.shape[0] == B
    _check(LIB.pa_decode_plan(_ptr(context_lens), B, num_heads, num_kv_heads, head_dim, block_size,
                              block_tables.shape[1], int(max_context_len), int(partition_size), _ptr(workspace),
                              workspace.numel() * workspace.element_size(), _ptr(status), _stream(stream)),
           "pa_decode_plan")


def decode(out, q, key_cache, value_cache, block_tables, context_lens, scale, max_context_len, workspace,
           partition_size=0, status=None, stream=None, tuning=None, planned=False):
    """One decode step of paged attention (pa_decode); writes ``out`` [B, Hq, D].

    The block size (8, 16 or 32 tokens) is the pools' dimension 2.  ``tuning`` (a DecodeTuning) selects a
    scheduling alternative or a test hook (pa_decode_tuned); None is the library's default schedule.
    ``planned`` decodes with the plan decode_plan left in ``workspace`` (pa_decode_planned; no tuning).
    """
    B, Hq, D = q.shape
    NB, Hkv, bs = key_cache.shape[0], key_cache.shape[1], key_cache.shape[2]
    assert out.shape == q.shape and out.dtype == q.dtype == key_cache.dtype == value_cache.dtype
    assert key_cache.shape == (NB, Hkv, bs, D) == value_cache.shape
    assert block_tables.dtype.itemsize == 4 and context_lens.dtype.itemsize == 4
    assert block_tables.shape[0] == B and context_lens.shape == (B,)
    for t in (out, q, key_cache, value_cache, block_tables, context_lens, workspace):
        assert t.is_contiguous()
    if planned:
        assert tuning is None, "a planned decode takes no tuning"
        _check(LIB.pa_decode_planned(_ptr(out), _ptr(q), _ptr(key_cache), _ptr(value_cache), _ptr(block_tables),
                                     block_tables.shape[1], _ptr(context_lens), B, Hq, Hkv, D, bs, NB, float(scale),
                                     int(max_context_len), int(partition_size), _ptr(workspace),
                                     workspace.numel() * workspace.element_size(), _dtype_code(q), _ptr(status),
                                     _stream(stream)),
               "pa_decode_planned")
        return
    _check(LIB.pa_decode_tuned(_ptr(out), _ptr(q), _ptr(key_cache), _ptr(value_cache), _ptr(block_tables),
                               block_tables.shape[1], _ptr(context_lens), B, Hq, Hkv, D, bs, NB, float(scale),
                               int(max_context_len), int(partition_size), _ptr(workspace),
                               workspace.numel() * workspace.element_size(), _dtype_code(q), _ptr(status),
                               _stream(stream), _tuning_ptr(tuning)),
           "pa_decode")


def prefill_workspace_size(num_seqs, num_heads, num_kv_heads, head_dim, max_query_len, dtype="bf16") -> int:
    """Bytes of workspace pa_prefill_ws needs for these sizes on the current device (may be 0)."""
    n = ctypes.c_size_t(0)
    if isinstance(dtype, str):
        code = {"f32": PA_F32, "f16": PA_F16, "bf16": PA_BF16}[dtype]
    else:
        import torch

        code = {torch.float32: PA_F32, torch.float16: PA_F16, torch.bfloat16: PA_BF16}[dtype]
    _check(LIB.pa_prefill_workspace_size(num_seqs, num_heads, num_kv_heads, head_dim, max_query_len, code,
                                         ctypes.byref(n)), "pa_prefill_workspace_size")
    return int(n.value)


def prefill(out, q, key_cache, value_cache, block_tables, query_start, context_lens, scale, max_query_len,
            status=None, stream=None, workspace=None):
    """Causal attention of each sequence's new query rows over its paged cache (pa_prefill).

    q, out [T, Hq, D]; query_start int32 [B + 1]; context_lens int32 [B] (the new tokens included,
    already written with reshape_and_cache).  With a workspace (a uint8 device tensor of at least
    prefill_workspace_size(...) bytes, scratch) the call is pa_prefill_ws, which splits the tensor-core
    kernel's last partial wave.
    """
    T, Hq, D = q.shape
    NB, Hkv, bs = key_cache.shape[0], key_cache.shape[1], key_cache.shape[2]
    assert out.shape == q.shape and out.dtype == q.dtype == key_cache.dtype == value_cache.dtype
    assert key_cache.shape == value_cache.shape
    assert block_tables.dtype.itemsize == 4 and context_lens.dtype.itemsize == 4 and query_start.dtype.itemsize == 4
    B = context_lens.shape[0]
    assert query_start.shape == (B + 1,) and block_tables.shape[0] == B
    for t in (out, q, key_cache, value_cache, block_tables, query_start, context_lens):
        assert t.is_contiguous()
    if workspace is None:
        _check(LIB.pa_prefill(_ptr(out), _ptr(q), _ptr(key_cache), _ptr(value_cache), _ptr(block_tables),
                              block_tables.shape[1], _ptr(query_start), _ptr(context_lens), B, Hq, Hkv, D, bs, NB,
                              float(scale), int(max_query_len), _dtype_code(q), _ptr(status), _stream(stream)),
               "pa_prefill")
        return
    assert workspace.is_contiguous()
    _check(LIB.pa_prefill_ws(_ptr(out), _ptr(q), _ptr(key_cache), _ptr(value_cache), _ptr(block_tables),
                             block_tables.shape[1], _ptr(query_start), _ptr(context_lens), B, Hq, Hkv, D, bs, NB,
                             float(scale), int(max_query_len), _ptr(workspace),
                             workspace.numel() * workspace.element_size(), _dtype_code(q), _ptr(status),
                             _stream(stream)),
           "pa_prefill_ws")


def copy_blocks(key_cache, value_cache, block_pairs, status=None, stream=None):
    """Copy-on-write clone of whole blocks (pa_copy_blocks); block_pairs int64 [N, 2] on the device."""
    assert key_cache.is_contiguous() and value_cache.is_contiguous() and block_pairs.is_contiguous()
    assert block_pairs.element_size() == 8 and block_pairs.dim() == 2 and block_pairs.shape[1] == 2
    NB, Hkv, bs, D = key_cache.shape
    _check(LIB.pa_copy_blocks(_ptr(key_cache), _ptr(value_cache), _ptr(block_pairs), block_pairs.shape[0], NB, Hkv,
                              D, bs, _dtype_code(key_cache), _ptr(status), _stream(stream)),
           "pa_copy_blocks")


def swap_blocks(src_key_cache, src_value_cache, dst_key_cache, dst_value_cache, block_pairs, status=None,
                stream=None):
    """Whole blocks between two pools (pa_swap_blocks); either side may be pinned host memory.

    block_pairs int64 [N, 2] (src block, dst block), on the device or in pinned host memory.
    """
    for t in (src_key_cache, src_value_cache, dst_key_cache, dst_value_cache, block_pairs):
        assert t.is_contiguous()
        assert t.is_cuda or t.is_pinned(), "pools and pairs must be device memory or pinned host memory"
    assert block_pairs.element_size() == 8 and block_pairs.dim() == 2 and block_pairs.shape[1] == 2
    assert src_key_cache.dtype == dst_key_cache.dtype == src_value_cache.dtype == dst_value_cache.dtype
    NBs, Hkv, bs, D = src_key_cache.shape
    NBd = dst_key_cache.shape[0]
    assert dst_key_cache.shape[1:] == src_key_cache.shape[1:]
    _check(LIB.pa_swap_blocks(_ptr(src_key_cache), _ptr(src_value_cache), _ptr(dst_key_cache), _ptr(dst_value_cache),
                              _ptr(block_pairs), block_pairs.shape[0], NBs, NBd, Hkv, D, bs,
                              _dtype_code(src_key_cache), _ptr(status), _stream(stream)),
           "pa_swap_blocks")


def check_copy_pairs(pairs_host, num_blocks: int) -> None:
    """Host-side validation of copy pairs (ids in range, no repeated dst, no dst that is also a src)."""
    import numpy as np

    pr = np.asarray(pairs_host).reshape(-1, 2)
    if pr.size and (pr.min() < 0 or pr.max() >= num_blocks):
        raise ValueError("copy pair id outside the pool")
    dst = pr[:, 1]
    if len(np.unique(dst)) != len(dst):
        raise ValueError("a destination block repeats")
    if np.isin(dst, pr[:, 0]).any():
        raise ValueError("a destination block is also a source")


class BlockManager:
    """Host block manager (pa_block_manager.h): allocation, sharing, copy-on-write, slot mappings.

    Arrays in and out are NumPy (host); ``append_tokens`` returns the slot
    mapping for pa_reshape_and_cache and the copy pairs for pa_copy_blocks.
    """

    def __init__(self, num_blocks: int, block_size: int = BLOCK_SIZE, num_host_blocks: int = 0):
        self._h = LIB.pa_bm_create(num_blocks, block_size, num_host_blocks)
        if not self._h:
            raise PagedAttentionError(PA_ERR_INVALID_ARG, "pa_bm_create")
        self.block_size = block_size

    def close(self):
        if self._h:
            LIB.pa_bm_destroy(self._h)
            self._h = None

    def __del__(self):
        self.close()

    @property
    def num_blocks(self) -> int:
        return int(LIB.pa_bm_num_blocks(self._h))

    @property
    def num_free_blocks(self) -> int:
        return int(LIB.pa_bm_num_free_blocks(self._h))

    @property
    def num_sequences(self) -> int:
        return int(LIB.pa_bm_num_sequences(self._h))

    @property
    def num_free_host_blocks(self) -> int:
        return int(LIB.pa_bm_num_free_host_blocks(self._h))

    def is_swapped(self, seq_id: int) -> bool:
        return int(LIB.pa_bm_is_swapped(self._h, seq_id)) == 1

    def _swap(self, fn, seq_id: int, where: str):
        import numpy as np

        pairs = np.empty((max(self.sequence_blocks(seq_id), 1), 2), dtype=np.int64)
        k = ctypes.c_int32(0)
        _check(fn(self._h, seq_id, pairs.ctypes.data, ctypes.byref(k)), where)
        return pairs[:k.value].copy()

    def swap_out(self, seq_id: int):
        """(device block, host block) pairs for swap_blocks(device pools -> host pools)."""
        return self._swap(LIB.pa_bm_swap_out, seq_id, "pa_bm_swap_out")

    def swap_in(self, seq_id: int):
        """(host block, device block) pairs for swap_blocks(host pools -> device pools)."""
        return self._swap(LIB.pa_bm_swap_in, seq_id, "pa_bm_swap_in")

    def ref_count(self, block: int) -> int:
        return int(LIB.pa_bm_ref_count(self._h, block))

    def sequence_blocks(self, seq_id: int) -> int:
        return int(LIB.pa_bm_sequence_blocks(self._h, seq_id))

    def sequence_length(self, seq_id: int) -> int:
        return int(LIB.pa_bm_sequence_length(self._h, seq_id))

    def add_sequence(self, seq_id: int, num_tokens: int):
        import numpy as np

        slots = np.empty(num_tokens, dtype=np.int64)
        _check(LIB.pa_bm_add_sequence(self._h, seq_id, num_tokens, slots.ctypes.data if num_tokens else None),
               "pa_bm_add_sequence")
        return slots

    def fork(self, parent_id: int, child_id: int) -> None:
        _check(LIB.pa_bm_fork(self._h, parent_id, child_id), "pa_bm_fork")

    def append_tokens(self, seq_ids):
        """(slot_mapping int64 [n], copy_pairs int64 [k, 2]) for one new token per listed sequence."""
        import numpy as np

        ids = np.ascontiguousarray(seq_ids, dtype=np.int64)
        n = ids.shape[0]
        slots = np.empty(n, dtype=np.int64)
        pairs = np.empty((max(n, 1), 2), dtype=np.int64)
        k = ctypes.c_int32(0)
        _check(LIB.pa_bm_append_tokens(self._h, ids.ctypes.data, n, slots.ctypes.data, pairs.ctypes.data,
                                       ctypes.byref(k)), "pa_bm_append_tokens")
        return slots, pairs[:k.value].copy()

    def free_sequence(self, seq_id: int) -> None:
        _check(LIB.pa_bm_free_sequence(self._h, seq_id), "pa_bm_free_sequence")

    def block_tables(self, seq_ids, max_blocks_per_seq: int):
        """(block_tables int32 [n, max_blocks_per_seq] padded with -1, context_lens int32 [n])."""
        import numpy as np

        ids = np.ascontiguousarray(seq_ids, dtype=np.int64)
        n = ids.shape[0]
        bt = np.empty((n, max_blocks_per_seq), dtype=np.int32)
        cl = np.empty(n, dtype=np.int32)
        _check(LIB.pa_bm_block_tables(self._h, ids.ctypes.data, n, max_blocks_per_seq, bt.ctypes.data,
                                      cl.ctypes.data), "pa_bm_block_tables")
        return bt, cl

