"""Seeded generators for the five workloads.

What is generated, and why it looks the way it does:

* Context lengths per sequence, drawn as each config states.  A context length
  counts the token that this decode step appends, so the step writes that
  token at position ``ctx - 1`` and then attends over ``[0, ctx)`` (the pages'
  "each token appends one KV entry inside the current logical block",
  LLM Inference Visualizer lesson 06, "How paging grows").
* Block tables: logical block ``j`` of sequence ``b`` lives at physical block
  ``block_tables[b, j]`` ("PagedAttention", section "PagedAttention in one
  picture": ``table[0] = 7``).  Entries past the last used logical block are
  ``-1`` so that a stray read is caught by bounds checks.
* Physical placement: a seeded permutation of the pool, an identity placement
  (contiguous, for the indirection-overhead measurement), a pool fragmented by
  allocate/free churn, or a shared-prefix layout with copy-on-write forks
  ("PagedAttention", section "Copy-on-write").
* The slot of each appended token: ``block_tables[b, (ctx-1) // 16] * 16 +
  (ctx-1) % 16``, and optional padding entries of ``-1`` (skipped by the write).
* Tensor values: N(0, 1) in the workload's storage dtype.

Nothing here computes attention, writes a cache or copies a block.
"""

from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

from .configs import WorkloadConfig

_NP_DTYPE = {"f32": np.float32, "f16": np.float16, "bf16": np.uint16}


@dataclass
class Workload:
    cfg: WorkloadConfig
    seed: int
    context_lens: np.ndarray        # int32 [B]
    block_tables: np.ndarray        # int32 [B, MB], -1 past the last used block
    slot_mapping: np.ndarray        # int64 [T]; -1 = padding (skip)
    copy_pairs: np.ndarray          # int64 [N, 2] (src, dst)
    num_blocks: int
    info: dict = field(default_factory=dict)

    @property
    def num_seqs(self) -> int:
        return int(self.context_lens.shape[0])

    @property
    def max_blocks_per_seq(self) -> int:
        return int(self.block_tables.shape[1])

    @property
    def max_context_len(self) -> int:
        return int(self.context_lens.max()) if self.context_lens.size else 0

    @property
    def num_tokens(self) -> int:
        return int(self.slot_mapping.shape[0])

    def kv_bytes(self) -> int:
        """Algorithmic K+V bytes one decode reads: sum_b ctx_b * Hkv * D * 2 * elt."""
        c = self.cfg
        return int(self.context_lens.astype(np.int64).sum()) * c.num_kv_heads * c.head_dim * 2 * c.elt_bytes


def _ceil_div(a, b):
    return -(-a // b)


def _draw_context_lens(cfg: WorkloadConfig, rng: np.random.Generator, num_seqs: int) -> np.ndarray:
    k, a = cfg.ctx_kind, cfg.ctx_args
    if k == "fixed":
        assert len(a) == num_seqs, (len(a), num_seqs)
        return np.asarray(a, dtype=np.int64)
    if k == "uniform":
        lo, hi = a
        return rng.integers(lo, hi + 1, size=num_seqs)
    if k == "lognormal":
        median, sigma, lo, hi = a
        return np.clip(np.round(median * np.exp(sigma * rng.standard_normal(num_seqs))), lo, hi).astype(np.int64)
    raise ValueError(k)


def _tables_from_lists(lists, num_blocks_per_seq_cap=None):
    mb = max(1, max((len(l) for l in lists), default=1))
    if num_blocks_per_seq_cap is not None:
        mb = max(mb, num_blocks_per_seq_cap)
    t = np.full((len(lists), mb), -1, dtype=np.int32)
    for b, l in enumerate(lists):
        t[b, :len(l)] = l
    return t


def _churn_free_list(rng: np.random.Generator, num_blocks: int, ops: int, max_run: int):
    """Pool fragmented by seeded allocate/free churn.

    Start from a free stack in random order, then run ``ops`` steps that either
    hand a run of 1..max_run blocks to a dummy owner or return a random dummy
    owner's blocks to the stack (probability 1/2 each).  Returns the free stack
    (top = end of list); the dummy owners keep their blocks.
    """
    free = list(rng.permutation(num_blocks))
    owners = []
    for _ in range(ops):
        if rng.random() < 0.5 or not owners:
            k = int(rng.integers(1, max_run + 1))
            if k <= len(free):
                owners.append([free.pop() for _ in range(k)])
        else:
            i = int(rng.integers(0, len(owners)))
            blocks = owners.pop(i)
            free.extend(blocks)
    return free


def build_workload(cfg: WorkloadConfig, seed: int = 0, *, num_seqs: int | None = None,
                   context_lens=None, pad_tokens: int = 0, placement: str | None = None) -> Workload:
    """Build the integer side of a workload (lengths, tables, slots, copy pairs).

    ``num_seqs`` / ``context_lens`` override the config (for reduced parity
    cases); ``pad_tokens`` inserts that many ``-1`` slots at seeded positions;
    ``placement`` overrides the physical placement scheme.
    """
    rng = np.random.default_rng(seed)
    bs = cfg.block_size
    placement = placement or cfg.placement
    info: dict = {}
    copy_pairs = np.zeros((0, 2), dtype=np.int64)

    if cfg.ctx_kind == "shared_prefix" and context_lens is None:
        prefix, lo, hi, nforks = cfg.ctx_args
        B = num_seqs or cfg.num_seqs
        nforks = min(nforks, B)
        nreg = B - nforks
        assert prefix % bs == 0
        npre = prefix // bs
        r = int(rng.integers(1, bs))              # tokens in the parent's partial shared block
        suffix = rng.integers(lo, hi + 1, size=nreg)
        free = list(rng.permutation(cfg.num_blocks))
        pre_blocks = [free.pop() for _ in range(npre)]
        parent_partial = free.pop()
        lists, ctx = [], []
        for s in suffix:
            own = [free.pop() for _ in range(_ceil_div(int(s), bs))]
            lists.append(pre_blocks + own)
            ctx.append(prefix + int(s))
        pairs = []
        for _ in range(nforks):
            clone = free.pop()
            pairs.append((parent_partial, clone))
            lists.append(pre_blocks + [clone])     # table already repointed at the clone
            ctx.append(prefix + r + 1)             # shared r tokens + the fork's own new token
        context = np.asarray(ctx, dtype=np.int64)
        tables = _tables_from_lists(lists)
        copy_pairs = np.asarray(pairs, dtype=np.int64).reshape(-1, 2)
        info.update(prefix_blocks=pre_blocks, parent_partial=parent_partial, shared_tokens_in_partial=r,
                    num_forks=nforks)
    else:
        if num_seqs:
            B = num_seqs
        elif context_lens is not None:
            B = len(context_lens)
        elif cfg.ctx_kind == "fixed":
            B = len(cfg.ctx_args)
        else:
            B = cfg.num_seqs
        if context_lens is not None:
            context = np.asarray(context_lens, dtype=np.int64)
        elif cfg.ctx_kind == "fixed" and num_seqs is not None and num_seqs != len(cfg.ctx_args):
            context = np.resize(np.asarray(cfg.ctx_args, dtype=np.int64), num_seqs)
        else:
            context = _draw_context_lens(cfg, rng, B)
        nblk = [_ceil_div(int(c), bs) for c in context]
        need = sum(nblk)
        if need > cfg.num_blocks:
            raise ValueError(f"workload needs {need} blocks, pool has {cfg.num_blocks}")
        if placement == "identity":
            order = list(range(cfg.num_blocks))[::-1]   # pop() yields 0, 1, 2, ...
            free = order
        elif placement == "churned":
            free = _churn_free_list(rng, cfg.num_blocks, ops=20000, max_run=64)
            if len(free) < need:
                raise ValueError("churn left too few free blocks")
        else:
            free = list(rng.permutation(cfg.num_blocks))
        lists = [[] for _ in range(B)]
        if placement == "churned":
            # sequences grow concurrently: logical block j of every sequence
            # is allocated before logical block j + 1 of any
            for j in range(max(nblk, default=0)):
                for b in range(B):
                    if nblk[b] > j:
                        lists[b].append(free.pop())
        else:
            for b in range(B):
                lists[b] = [free.pop() for _ in range(nblk[b])]
        tables = _tables_from_lists(lists)
        if placement == "churned":
            d = [abs(int(l[i + 1]) - int(l[i])) for l in lists for i in range(len(l) - 1)]
            info["mean_block_id_gap"] = float(np.mean(d)) if d else 0.0

    # the appended token of each sequence sits at position ctx - 1
    slots = []
    for b in range(len(context)):
        c = int(context[b])
        if c <= 0:
            continue
        pos = c - 1
        slots.append(int(tables[b, pos // bs]) * bs + pos % bs)
    slots = np.asarray(slots, dtype=np.int64)
    if pad_tokens:
        where = np.sort(rng.integers(0, len(slots) + 1, size=pad_tokens))
        slots = np.insert(slots, where, -1)
    return Workload(cfg=cfg, seed=seed, context_lens=context.astype(np.int32), block_tables=tables,
                    slot_mapping=slots, copy_pairs=copy_pairs, num_blocks=cfg.num_blocks, info=info)


def _f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bfloat16 (nearest, ties to even); returns the uint16 bit pattern."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    rounded = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return rounded.astype(np.uint16)


def _normal(rng: np.random.Generator, shape, dtype: str) -> np.ndarray:
    x = rng.standard_normal(size=shape, dtype=np.float32)
    if dtype == "f32":
        return x
    if dtype == "f16":
        return x.astype(np.float16)
    return _f32_to_bf16_bits(x)


def host_values(wl: Workload, seed: int | None = None) -> dict:
    """N(0,1) tensors on the host, in the storage dtype (bf16 as uint16 bits).

    Returns q [B,Hq,D], key/value (the appended tokens) [T,Hkv,D] and the
    pools key_cache/value_cache [NB,Hkv,16,D].  Padding rows of key/value
    (slot -1) get values too; the write must ignore them.
    """
    c = wl.cfg
    rng = np.random.default_rng(1_000_003 + (wl.seed if seed is None else seed))
    T = wl.num_tokens
    return {
        "q": _normal(rng, (wl.num_seqs, c.num_heads, c.head_dim), c.dtype),
        "key": _normal(rng, (T, c.num_kv_heads, c.head_dim), c.dtype),
        "value": _normal(rng, (T, c.num_kv_heads, c.head_dim), c.dtype),
        "key_cache": _normal(rng, (wl.num_blocks, c.num_kv_heads, c.block_size, c.head_dim), c.dtype),
        "value_cache": _normal(rng, (wl.num_blocks, c.num_kv_heads, c.block_size, c.head_dim), c.dtype),
    }


def device_values(wl: Workload, device, seed: int | None = None) -> dict:
    """The same kinds of tensors as :func:`host_values`, drawn on ``device`` with torch.

    Used for full-size workloads whose pools are too large to draw on the
    host; the stream differs from :func:`host_values` (a different RNG), so
    tests that need host copies read them back before any kernel runs.
    """
    import torch

    c = wl.cfg
    tdt = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}[c.dtype]
    g = torch.Generator(device=device)
    g.manual_seed(2_000_029 + (wl.seed if seed is None else seed))

    def normal(shape):
        out = torch.empty(shape, dtype=tdt, device=device)
        flat = out.view(-1)
        step = 1 << 26
        for i in range(0, flat.numel(), step):
            n = min(step, flat.numel() - i)
            flat[i:i + n].copy_(torch.randn(n, generator=g, device=device, dtype=torch.float32))
        return out

    T = wl.num_tokens
    return {
        "q": normal((wl.num_seqs, c.num_heads, c.head_dim)),
        "key": normal((T, c.num_kv_heads, c.head_dim)),
        "value": normal((T, c.num_kv_heads, c.head_dim)),
        "key_cache": normal((wl.num_blocks, c.num_kv_heads, c.block_size, c.head_dim)),
        "value_cache": normal((wl.num_blocks, c.num_kv_heads, c.block_size, c.head_dim)),
    }


# bit patterns of a quiet NaN in each storage dtype (bf16 held as uint16)
_NAN_BITS = {"f16": np.float16(np.nan), "bf16": np.uint16(0x7FC0), "f32": np.float32(np.nan)}


def unread_slots(wl: Workload):
    """Slots of the pool that no sequence of the workload reads: (blocks, offsets).

    A block in the middle of a table is read whole; a sequence's last block
    up to its context; a copy-pair source whole (its copy is read).  Every
    other slot -- the tail of last blocks, unreferenced blocks -- may hold
    anything in a real pool; tests fill them with NaN.
    """
    bs = wl.cfg.block_size
    extent = np.zeros(wl.num_blocks, dtype=np.int64)
    for b in range(wl.num_seqs):
        n = int(wl.context_lens[b])
        nb = _ceil_div(n, bs)
        if nb == 0:
            continue
        row = wl.block_tables[b, :nb].astype(np.int64)
        ok = (row >= 0) & (row < wl.num_blocks)
        mid = row[:-1][ok[:-1]]
        extent[mid] = bs
        if ok[-1]:
            extent[row[-1]] = max(extent[row[-1]], n - (nb - 1) * bs)
    for src, _ in np.asarray(wl.copy_pairs).reshape(-1, 2):
        extent[int(src)] = bs
    blk, off = np.nonzero(np.arange(bs)[None, :] >= extent[:, None])
    return blk, off


def poison_unread_slots(wl: Workload, vals: dict) -> int:
    """Write NaN into every unread slot of the host pools in ``vals`` (in place); returns the slot count."""
    blk, off = unread_slots(wl)
    nan = _NAN_BITS[wl.cfg.dtype]
    for k in ("key_cache", "value_cache"):
        vals[k][blk, :, off, :] = nan
    return int(blk.size)
