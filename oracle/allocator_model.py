"""The block pool and per-request block tables, as a plain Python model.

Test infrastructure only: the authority for bit-exact allocator state. It
follows the pages' account of on-demand allocation:

* fixed-size KV blocks of block_size tokens (16 by default) -- "vLLM KV Cache and
  PagedAttention Explained", 5단계 and Step 5 "PagedAttention in vLLM";
* a request of n tokens holds ceil(n / block_size) blocks (Step 6 "Prefill":
  ceil(6 / 16) = 1), and a new block is appended to its table when the length
  crosses a block boundary (5단계: the 17th token gets a new block; Step 6 "Decode";
  "PagedAttention" card, "OS paging과 같은 발상");
* the table maps logical block j to any free physical block (Step 5 "PagedAttention
  in vLLM": blocks 7, 23, 61);
* on completion the request's blocks go back to the pool, immediately reusable
  (Step 7, item 7; Step 8 "Continuous Batching in vLLM").

* prefix sharing ("vLLM KV Cache and PagedAttention Explained", Step 9 "Safe
  Sharing with Copy-on-Write"): a block may be named by several requests' tables
  and keeps a reference count; it returns to the pool when the count drops to
  zero; a request that is about to write into a block others also name first
  gets its own copy of that block (the copy is queued for the device) and its
  table entry is repointed, the others keep the original.

Readings where the pages are silent (listed in the design notes): the free list
is a LIFO stack; ``initial_order`` lists the ids in the order they are first
handed out (identity when omitted); growth pops ids one at a time and appends
them in pop order; a freed request pushes its ids back in logical order; a grow
that does not fit changes nothing (OOM); a slot is block * block_size + offset.
"""

INVALID, OOM, OUT_OF_RANGE = 1, 2, 3


class PoolError(Exception):
    def __init__(self, code, msg):
        super().__init__(msg)
        self.code = code


class BlockPoolModel:
    def __init__(self, num_blocks, block_size, initial_order=None):
        if num_blocks < 0 or block_size <= 0:
            raise PoolError(INVALID, "bad pool size")
        order = list(range(num_blocks)) if initial_order is None else [int(x) for x in initial_order]
        if sorted(order) != list(range(num_blocks)):
            raise PoolError(INVALID, "initial_order is not a permutation of the pool")
        self.num_blocks = num_blocks
        self.block_size = block_size
        self.free = order[::-1]  # top of the stack = end of the list = next id handed out
        self.tables = {}
        self.lens = {}
        self.refs = [0] * num_blocks   # how many tables name each block
        self.copies = []               # pending (src, dst) block copies from copy-on-write

    def blocks_needed(self, n_tokens):
        return -(-n_tokens // self.block_size)

    def _cow_needed(self, seq_id, new_len):
        """Growing past the current length writes into the last block if it is
        partly filled; if other tables also name it, it must be copied first."""
        table = self.tables.get(seq_id, [])
        cur = self.lens.get(seq_id, 0)
        return (new_len > cur and cur % self.block_size != 0 and table
                and self.refs[table[-1]] > 1)

    def grow(self, seq_id, new_len):
        if new_len < 0:
            raise PoolError(INVALID, "negative length")
        table = self.tables.get(seq_id, [])
        cur = self.lens.get(seq_id, 0)
        if new_len < cur:
            raise PoolError(INVALID, "a sequence cannot shrink")
        cow = self._cow_needed(seq_id, new_len)
        need = self.blocks_needed(new_len) - len(table) + (1 if cow else 0)
        if need > len(self.free):
            raise PoolError(OOM, "pool exhausted")
        table = list(table)
        if cow:
            src = table[-1]
            dst = self.free.pop()
            self.refs[src] -= 1
            self.refs[dst] = 1
            table[-1] = dst
            self.copies.append((src, dst))
        for _ in range(self.blocks_needed(new_len) - len(table)):
            b = self.free.pop()
            self.refs[b] = 1
            table.append(b)
        self.tables[seq_id] = table
        self.lens[seq_id] = new_len

    def fork(self, parent, child):
        """child starts as a copy of parent's table and length; every block is shared."""
        if parent not in self.tables or child in self.tables:
            raise PoolError(INVALID, "unknown parent or existing child")
        self.tables[child] = list(self.tables[parent])
        self.lens[child] = self.lens[parent]
        for b in self.tables[child]:
            self.refs[b] += 1

    def take_copies(self):
        out, self.copies = self.copies, []
        return out

    def release(self, seq_id):
        if seq_id not in self.tables:
            raise PoolError(INVALID, "unknown sequence")
        for b in self.tables.pop(seq_id):
            self.refs[b] -= 1
            if self.refs[b] == 0:
                self.free.append(b)
        del self.lens[seq_id]

    def block_table(self, seq_id):
        if seq_id not in self.tables:
            raise PoolError(INVALID, "unknown sequence")
        return list(self.tables[seq_id])

    def slot_mapping(self, seq_ids, start_pos, n_tok):
        out = []
        for sid, p0, n in zip(seq_ids, start_pos, n_tok):
            if sid not in self.tables:
                raise PoolError(INVALID, "unknown sequence")
            if p0 < 0 or n < 0 or p0 + n > self.lens[sid]:
                raise PoolError(OUT_OF_RANGE, "token position not allocated")
            table = self.tables[sid]
            for pos in range(p0, p0 + n):
                out.append(table[pos // self.block_size] * self.block_size + pos % self.block_size)
        return out

    def block_tables(self, seq_ids, max_blocks):
        rows = []
        for sid in seq_ids:
            if sid not in self.tables:
                raise PoolError(INVALID, "unknown sequence")
            t = self.tables[sid]
            if len(t) > max_blocks:
                raise PoolError(OUT_OF_RANGE, "table wider than max_blocks")
            rows.append(t + [-1] * (max_blocks - len(t)))
        return rows

    def stats(self):
        used = sum(self.lens.values())
        held = sum(len(t) for t in self.tables.values()) * self.block_size
        return len(self.free), used, held - used

    def dump(self):
        return list(self.free)
