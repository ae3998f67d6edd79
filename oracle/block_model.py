"""Plain-Python model of the block bookkeeping around the paged KV cache (test infrastructure).

Only tests/ use it: it is the reference the C++ block manager
(include/pa_block_manager.h) is checked against, operation by operation.  It
shares no code with the library.

It follows the pages' description step by step:
  * the cache is a pool of fixed-size physical blocks; each request has a
    block table from its logical blocks to physical ones ("PagedAttention"
    digest, sections "This is just virtual memory" and "PagedAttention in one
    picture");
  * a request takes a new block only when its last one is full ("LLM
    Inference Visualizer", lesson 06, "How paging grows");
  * a fork shares the parent's blocks and counts references; a request that
    writes into a block others still reference first gets its own copy of it
    (digest, section "Copy-on-write: when two requests share a prefix");
  * a finished request gives its blocks back; a block is free again when no
    request references it;
  * under memory pressure a request is evicted to CPU memory, the OS's
    swapping; its shared blocks stay, because others still use them
    ("PagedAttention, Visualized", Part 3).

The pages say nothing about which free block is handed out next.  The reading
taken (and stated in the library's header): a stack, the most recently freed
block first, a fresh pool handing out 0, 1, 2, ...; a request that finishes
gives its blocks back last block first.
"""

from __future__ import annotations


class NoBlocks(Exception):
    """The pool has fewer free blocks than the operation needs (nothing was changed)."""


class BlockModel:
    def __init__(self, num_blocks: int, block_size: int, num_host_blocks: int = 0):
        self.num_blocks = num_blocks
        self.block_size = block_size
        self.refs = [0] * num_blocks
        self.free = list(range(num_blocks - 1, -1, -1))   # the end of the list is handed out next
        self.host_free = list(range(num_host_blocks - 1, -1, -1))
        self.tables: dict[int, list[int]] = {}
        self.lengths: dict[int, int] = {}
        self.on_host: dict[int, list[bool]] = {}            # swapped-out requests: which entries are host blocks

    # --- pool ---------------------------------------------------------------
    def _take(self) -> int:
        b = self.free.pop()
        self.refs[b] = 1
        return b

    def _release(self, b: int) -> None:
        self.refs[b] -= 1
        if self.refs[b] == 0:
            self.free.append(b)

    def slot(self, block: int, offset: int) -> int:
        return block * self.block_size + offset

    # --- operations -----------------------------------------------------------
    def add_sequence(self, sid: int, num_tokens: int) -> list[int]:
        """A new request with num_tokens tokens: enough fresh blocks, and the slot of every token."""
        assert sid not in self.tables
        nblocks = -(-num_tokens // self.block_size)
        if nblocks > len(self.free):
            raise NoBlocks()
        table = [self._take() for _ in range(nblocks)]
        self.tables[sid] = table
        self.lengths[sid] = num_tokens
        return [self.slot(table[t // self.block_size], t % self.block_size) for t in range(num_tokens)]

    def fork(self, parent: int, child: int) -> None:
        """The child shares all of the parent's blocks."""
        assert parent in self.tables and child not in self.tables
        self.tables[child] = list(self.tables[parent])
        self.lengths[child] = self.lengths[parent]
        for b in self.tables[child]:
            self.refs[b] += 1

    def append_tokens(self, sids: list[int]) -> tuple[list[int], list[tuple[int, int]]]:
        """One new token per listed request, in order: (slots, copy-on-write pairs (src, dst))."""
        # dry run on copies of the state, so that a failure changes nothing
        saved = (list(self.refs), list(self.free), {k: list(v) for k, v in self.tables.items()}, dict(self.lengths))
        slots, copies = [], []
        try:
            for sid in sids:
                table = self.tables[sid]
                n = self.lengths[sid]
                offset = n % self.block_size
                if offset == 0:
                    # the last block is full (or there is none): a fresh block
                    if not self.free:
                        raise NoBlocks()
                    table.append(self._take())
                elif self.refs[table[-1]] > 1:
                    # writing into a block others still reference: copy it first
                    if not self.free:
                        raise NoBlocks()
                    old = table[-1]
                    new = self._take()
                    copies.append((old, new))
                    self._release(old)
                    table[-1] = new
                slots.append(self.slot(table[-1], offset))
                self.lengths[sid] = n + 1
        except NoBlocks:
            self.refs, self.free, self.tables, self.lengths = saved
            raise
        return slots, copies

    def free_sequence(self, sid: int) -> None:
        table = self.tables.pop(sid)
        del self.lengths[sid]
        host = self.on_host.pop(sid, [False] * len(table))
        for b, h in zip(reversed(table), reversed(host)):
            if h:
                self.host_free.append(b)
            else:
                self._release(b)

    def swap_out(self, sid: int) -> list[tuple[int, int]]:
        """Evict a request: its private blocks move to host blocks, (device, host) pairs."""
        assert sid in self.tables and sid not in self.on_host
        table = self.tables[sid]
        private = [j for j, b in enumerate(table) if self.refs[b] == 1]
        if len(private) > len(self.host_free):
            raise NoBlocks()
        host = [False] * len(table)
        pairs = []
        for j in private:
            h = self.host_free.pop()
            pairs.append((table[j], h))
            self._release(table[j])
            table[j] = h
            host[j] = True
        self.on_host[sid] = host
        return pairs

    def swap_in(self, sid: int) -> list[tuple[int, int]]:
        """Bring an evicted request back: a fresh device block per host block, (host, device) pairs."""
        host = self.on_host[sid]
        table = self.tables[sid]
        if sum(host) > len(self.free):
            raise NoBlocks()
        pairs = []
        for j, h in enumerate(host):
            if h:
                d = self._take()
                pairs.append((table[j], d))
                self.host_free.append(table[j])
                table[j] = d
        del self.on_host[sid]
        return pairs

    def block_tables(self, sids: list[int], max_blocks: int) -> tuple[list[list[int]], list[int]]:
        rows = []
        for sid in sids:
            t = self.tables[sid]
            assert len(t) <= max_blocks
            rows.append(t + [-1] * (max_blocks - len(t)))
        return rows, [self.lengths[s] for s in sids]
