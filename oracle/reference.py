"""NumPy fp64 oracle -- test infrastructure only (see the package docstring).

Data layout read here (the layout the library defines, restated with explicit
index arithmetic, not shared code):

* key_cache, value_cache: ``[num_blocks, num_kv_heads, block_size, head_dim]``
  row-major; the K (or V) vector of token ``i`` of a sequence whose logical
  block ``i // block_size`` lives at physical block ``blk`` is
  ``cache[blk, kv_head, i % block_size, :]``.
* block_tables int32 ``[num_seqs, max_blocks_per_seq]``, context_lens int32
  ``[num_seqs]``, slot_mapping int64 ``[num_tokens]`` (slot = blk * block_size +
  offset, ``< 0`` = skip), copy pairs int64 ``[n, 2]`` (src, dst).
* q ``[num_seqs, num_heads, head_dim]``; query head ``h`` reads KV head
  ``h // (num_heads // num_kv_heads)``.

Storage dtypes: "f32", "f16" and "bf16" (bf16 held as uint16 bit patterns).
All attention arithmetic is fp64 on the exactly upcast stored values.
"""

from __future__ import annotations

import numpy as np

# ---------------------------------------------------------------------------
# dtype handling (exact upcasts)
# ---------------------------------------------------------------------------


def to_f64(x: np.ndarray, dtype: str) -> np.ndarray:
    """Exact upcast of stored values to float64 (bf16 = top half of an f32)."""
    if dtype == "bf16":
        u = np.asarray(x, dtype=np.uint16).astype(np.uint32) << 16
        return u.view(np.float32).astype(np.float64)
    return np.asarray(x).astype(np.float64)


def bits_view(x: np.ndarray) -> np.ndarray:
    """Raw bit pattern view for bit-exact comparison of any storage dtype."""
    x = np.ascontiguousarray(x)
    return x.view({2: np.uint16, 4: np.uint32, 8: np.uint64}[x.dtype.itemsize])


# ---------------------------------------------------------------------------
# Closed-form sizes ("PagedAttention, Visualized", Part 2; "PagedAttention",
# section "PagedAttention in one picture")
# ---------------------------------------------------------------------------


def kv_bytes_per_token(num_kv_heads: int, head_dim: int, num_layers: int, elt_bytes: int) -> int:
    """Bytes of K and V one token keeps: 2 (K and V) x width x layers x element size.

    "PagedAttention, Visualized", Part 2: for Qwen2.5-7B the width is 512
    (4 KV heads x 128 dims), 28 layers, 2-byte FP16 elements.
    """
    return 2 * num_kv_heads * head_dim * num_layers * elt_bytes


def blocks_needed(num_tokens: int, block_size: int) -> int:
    """Blocks a request of ``num_tokens`` tokens holds: allocation rounds up to whole blocks.

    "PagedAttention", section "PagedAttention in one picture": 47 tokens take
    three 16-token blocks (48 slots); waste is below one block.
    """
    return -(-num_tokens // block_size)


def reservation_waste(used_tokens: int, reserved_tokens: int) -> float:
    """Fraction of a contiguous worst-case reservation left unused.

    "PagedAttention, Visualized", Part 3: 500 used of a 32,768-token reservation.
    """
    return 1.0 - used_tokens / reserved_tokens


def paged_waste_tokens(num_tokens: int, block_size: int) -> int:
    """Slots allocated but unused under paging (only the last block's tail)."""
    return blocks_needed(num_tokens, block_size) * block_size - num_tokens


# ---------------------------------------------------------------------------
# Block-table walk ("PagedAttention", section "PagedAttention in one picture":
# logical block j of a request lives at physical block table[j]; the first 16
# tokens go in logical block 0, the next 16 in logical block 1, and so on)
# ---------------------------------------------------------------------------


def token_slot(block_table_row: np.ndarray, pos: int, block_size: int) -> tuple[int, int]:
    """(physical block, offset in block) holding token position ``pos``."""
    logical = pos // block_size
    return int(block_table_row[logical]), pos % block_size


def gather_kv(cache: np.ndarray, block_table_row: np.ndarray, ctx: int, kv_head: int,
              block_size: int) -> np.ndarray:
    """The ``ctx`` K (or V) vectors of one sequence and KV head, in logical order.

    Walks the block table entry by entry and gathers each token's vector from
    wherever its block physically lives ("PagedAttention", section
    "PagedAttention in one picture").  Raises IndexError on an out-of-pool id.
    """
    num_blocks = cache.shape[0]
    rows = []
    for pos in range(ctx):
        blk, off = token_slot(block_table_row, pos, block_size)
        if not (0 <= blk < num_blocks):
            raise IndexError(f"block id {blk} outside pool of {num_blocks}")
        rows.append(cache[blk, kv_head, off, :])
    if not rows:
        return cache[:0, kv_head, 0, :]
    return np.stack(rows)


# ---------------------------------------------------------------------------
# Attention: the plain definition.  PagedAttention does not change the math;
# attention gives the same logits whether K/V are contiguous or scattered
# ("PagedAttention", section "Misconceptions").
# ---------------------------------------------------------------------------


def attention_f64(q: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float) -> np.ndarray:
    """softmax(scale * q . k_i) weighted sum of v_i, all in fp64.

    q [D], k [n, D], v [n, D] (float64).  An empty context (n = 0) gives a zero
    vector (the library's convention for a sequence with no tokens).
    """
    n = k.shape[0]
    if n == 0:
        return np.zeros(v.shape[1] if v.ndim == 2 else q.shape[0], dtype=np.float64)
    logits = np.empty(n, dtype=np.float64)
    for i in range(n):
        logits[i] = scale * float(np.dot(q, k[i]))
    m = logits.max()
    w = np.exp(logits - m)
    w /= w.sum()
    out = np.zeros(v.shape[1], dtype=np.float64)
    for i in range(n):
        out += w[i] * v[i]
    return out


def decode_one(q: np.ndarray, key_cache: np.ndarray, value_cache: np.ndarray,
               block_tables: np.ndarray, context_lens: np.ndarray, b: int, h: int,
               scale: float, dtype: str, num_kv_heads: int) -> np.ndarray:
    """Decode output of sequence ``b``, query head ``h`` (fp64 [D])."""
    num_heads = q.shape[1]
    group = num_heads // num_kv_heads
    kv_head = h // group
    bs = key_cache.shape[2]
    ctx = int(context_lens[b])
    kb = to_f64(gather_kv(key_cache, block_tables[b], ctx, kv_head, bs), dtype)
    vb = to_f64(gather_kv(value_cache, block_tables[b], ctx, kv_head, bs), dtype)
    return attention_f64(to_f64(q[b, h], dtype), kb, vb, scale)


def decode(q: np.ndarray, key_cache: np.ndarray, value_cache: np.ndarray,
           block_tables: np.ndarray, context_lens: np.ndarray, scale: float, dtype: str,
           num_kv_heads: int) -> np.ndarray:
    """Paged decode attention for every sequence and query head (fp64 [B, Hq, D])."""
    B, Hq, D = q.shape
    out = np.zeros((B, Hq, D), dtype=np.float64)
    for b in range(B):
        for h in range(Hq):
            out[b, h] = decode_one(q, key_cache, value_cache, block_tables, context_lens, b, h,
                                   scale, dtype, num_kv_heads)
    return out


def prefill_rows(query_start: np.ndarray, context_lens: np.ndarray):
    """For every new query row: (sequence, position).  Row i of sequence b (of L
    new tokens, n tokens in the cache in all) sits at position n - L + i."""
    seqs, pos = [], []
    for b in range(len(context_lens)):
        L = int(query_start[b + 1] - query_start[b])
        n = int(context_lens[b])
        for i in range(L):
            seqs.append(b)
            pos.append(n - L + i)
    return np.array(seqs, dtype=np.int64), np.array(pos, dtype=np.int64)


def prefill(q: np.ndarray, key_cache: np.ndarray, value_cache: np.ndarray, block_tables: np.ndarray,
            query_start: np.ndarray, context_lens: np.ndarray, scale: float, dtype: str,
            num_kv_heads: int) -> np.ndarray:
    """Causal attention of each new query row over the cache up to its own position (fp64 [T, Hq, D]).

    By definition the row at position p sees exactly the keys 0 .. p: it is the
    decode of a sequence whose context is the first p + 1 tokens.
    """
    seqs, pos = prefill_rows(query_start, context_lens)
    return decode(q, key_cache, value_cache, block_tables[seqs], (pos + 1).astype(np.int32), scale, dtype,
                  num_kv_heads)


# ---------------------------------------------------------------------------
# Split-context partitions and their merge.  Softmax over a union of disjoint
# token sets can be rebuilt from each set's (max, sum of exp, unnormalised
# weighted sum): rescale each by exp(max_p - max) and add.
# ---------------------------------------------------------------------------


def partition_partial(q: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float):
    """(m, l, acc) of one partition: max logit, sum of exp(logit - m), sum of exp(logit - m) v."""
    n = k.shape[0]
    if n == 0:
        return -np.inf, 0.0, np.zeros(v.shape[1], dtype=np.float64)
    logits = np.array([scale * float(np.dot(q, k[i])) for i in range(n)], dtype=np.float64)
    m = logits.max()
    w = np.exp(logits - m)
    acc = np.zeros(v.shape[1], dtype=np.float64)
    for i in range(n):
        acc += w[i] * v[i]
    return float(m), float(w.sum()), acc


def merge_partials(parts) -> np.ndarray:
    """Combine per-partition (m, l, acc) into the normalised output."""
    parts = [p for p in parts if p[1] > 0.0]
    if not parts:
        return None
    M = max(p[0] for p in parts)
    L = sum(p[1] * np.exp(p[0] - M) for p in parts)
    acc = sum(p[2] * np.exp(p[0] - M) for p in parts)
    return acc / L


def decode_split(q, key_cache, value_cache, block_tables, context_lens, b, h, scale, dtype,
                 num_kv_heads, partition_size):
    """Decode of (b, h) computed partition by partition and merged (fp64 [D])."""
    num_heads = q.shape[1]
    kv_head = h // (num_heads // num_kv_heads)
    bs = key_cache.shape[2]
    ctx = int(context_lens[b])
    kb = to_f64(gather_kv(key_cache, block_tables[b], ctx, kv_head, bs), dtype)
    vb = to_f64(gather_kv(value_cache, block_tables[b], ctx, kv_head, bs), dtype)
    qv = to_f64(q[b, h], dtype)
    parts = [partition_partial(qv, kb[s:s + partition_size], vb[s:s + partition_size], scale)
             for s in range(0, ctx, partition_size)]
    out = merge_partials(parts)
    return np.zeros(q.shape[2]) if out is None else out


# ---------------------------------------------------------------------------
# Cache write: each appended token's K/V goes into the slot the host chose
# ("LLM Inference Visualizer", lesson 06, "How paging grows": each token
# appends one KV entry inside the current logical block).
# ---------------------------------------------------------------------------


def reshape_and_cache(key: np.ndarray, value: np.ndarray, key_cache: np.ndarray,
                      value_cache: np.ndarray, slot_mapping: np.ndarray):
    """Return copies of the pools with token t's K/V written at slot_mapping[t].

    key/value [T, Hkv, D]; slot s >= 0 means block s // block_size, offset
    s % block_size; s < 0 is padding and writes nothing.  Byte-exact copy.
    """
    kc = key_cache.copy()
    vc = value_cache.copy()
    bs = kc.shape[2]
    nslots = kc.shape[0] * bs
    for t in range(key.shape[0]):
        s = int(slot_mapping[t])
        if s < 0:
            continue
        if s >= nslots:
            raise IndexError(f"slot {s} outside pool of {nslots} slots")
        blk, off = s // bs, s % bs
        for hk in range(kc.shape[1]):
            kc[blk, hk, off, :] = key[t, hk, :]
            vc[blk, hk, off, :] = value[t, hk, :]
    return kc, vc


# ---------------------------------------------------------------------------
# Copy-on-write clone: the engine copies the shared block into a fresh one and
# repoints the writer's table at the copy ("PagedAttention", section
# "Copy-on-write: when two requests share a prefix").
# ---------------------------------------------------------------------------


def copy_blocks(key_cache: np.ndarray, value_cache: np.ndarray, pairs: np.ndarray):
    """Return copies of the pools with block dst := block src for each (src, dst) pair.

    Sources are read from the pools as they were before any copy of the call.
    """
    kc = key_cache.copy()
    vc = value_cache.copy()
    nb = kc.shape[0]
    for src, dst in np.asarray(pairs).reshape(-1, 2):
        src, dst = int(src), int(dst)
        if not (0 <= src < nb and 0 <= dst < nb):
            raise IndexError(f"copy pair ({src}, {dst}) outside pool of {nb}")
        kc[dst] = key_cache[src]
        vc[dst] = value_cache[src]
    return kc, vc
