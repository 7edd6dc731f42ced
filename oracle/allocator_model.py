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

    def blocks_needed(self, n_tokens):
        return -(-n_tokens // self.block_size)

    def grow(self, seq_id, new_len):
        if new_len < 0:
            raise PoolError(INVALID, "negative length")
        table = self.tables.get(seq_id, [])
        cur = self.lens.get(seq_id, 0)
        if new_len < cur:
            raise PoolError(INVALID, "a sequence cannot shrink")
        need = self.blocks_needed(new_len) - len(table)
        if need > len(self.free):
            raise PoolError(OOM, "pool exhausted")
        table = list(table)
        for _ in range(need):
            table.append(self.free.pop())
        self.tables[seq_id] = table
        self.lens[seq_id] = new_len

    def release(self, seq_id):
        if seq_id not in self.tables:
            raise PoolError(INVALID, "unknown sequence")
        self.free.extend(self.tables.pop(seq_id))
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
