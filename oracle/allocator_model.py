"""Plain-Python model of the paged KV block manager -- TEST INFRASTRUCTURE ONLY.

It restates, one step at a time, what the pages say a block manager does:

* the KV cache is cut into fixed-size physical blocks; a sequence's
  tokens are logically contiguous and its block table maps logical block
  i to a physical block (page "大语言模型推理内存管理算法 paged attention",
  sections 2 and 3; page "08. PagedAttention：把 KV Cache 分页管理", section
  "借用操作系统的办法：分页");
* blocks are taken from a free list on demand -- a new block only when
  the current last block is full -- and every block of a finished
  sequence goes back to the free list for reuse (first page, sections 7
  and 8; third page, same section);
* a token's slot is block_table[logical block] * block_size + offset
  (third page, section "为什么叫 PagedAttention");
* sharing: several tables may point at one physical block, whose
  reference count says how many sequences use it; a fork copies the
  parent's table and adds one reference to each block (third page,
  section "分页还顺带解决了什么"; page "PagedAttention 核心思想解析",
  sections 2.3 and 5.1);
* copy-on-write: when a sequence must write into a block whose reference
  count is above one, a new block is allocated, the old block's contents
  are copied into it, the table entry is pointed at the new block and the
  old block's count drops by one (second page, section 2.3). A sole owner
  writes in place.

Which physical id the free list hands out is not fixed by the pages; this
model pops the most recently freed block (a LIFO stack). Tests compare the
product allocator with this model only up to a relabelling of ids.
"""
from __future__ import annotations


class OutOfBlocks(RuntimeError):
    pass


class BadState(RuntimeError):
    pass


class BlockManagerModel:
    def __init__(self, num_blocks: int, block_size: int):
        if num_blocks <= 0 or block_size <= 0:
            raise ValueError("num_blocks and block_size must be positive")
        self.num_blocks = num_blocks
        self.block_size = block_size
        self.free = list(range(num_blocks - 1, -1, -1))  # top of the stack is the end
        self.ref = [0] * num_blocks
        self.tables: dict[int, list[int]] = {}
        self.lens: dict[int, int] = {}

    # -- allocation ---------------------------------------------------------------------------
    def _blocks_for(self, num_tokens: int) -> int:
        # whole blocks needed to hold num_tokens tokens
        return -(-num_tokens // self.block_size)

    def _pop(self) -> int:
        if not self.free:
            raise OutOfBlocks("free list is empty")
        blk = self.free.pop()
        self.ref[blk] = 1
        return blk

    def add_seq(self, seq: int, num_tokens: int) -> list[int]:
        """A new request: take the blocks its prompt needs, all or none."""
        if seq in self.tables:
            raise BadState(f"sequence {seq} exists")
        if num_tokens < 0:
            raise ValueError("negative length")
        need = self._blocks_for(num_tokens)
        if need > len(self.free):
            raise OutOfBlocks(f"need {need} blocks, {len(self.free)} free")
        self.tables[seq] = [self._pop() for _ in range(need)]
        self.lens[seq] = num_tokens
        return list(self.tables[seq])

    def fork(self, parent: int, child: int):
        """The child shares every block of the parent; each gains a reference."""
        if parent not in self.tables or child in self.tables:
            raise BadState("bad fork")
        self.tables[child] = list(self.tables[parent])
        self.lens[child] = self.lens[parent]
        for blk in self.tables[child]:
            self.ref[blk] += 1

    def append_slot(self, seq: int):
        """Reserve the slot of the sequence's next token.

        Returns (slot, cow_src, cow_dst); cow_* are -1 unless the write had
        to copy a shared block first. Nothing changes if no block is free."""
        if seq not in self.tables:
            raise BadState(f"no sequence {seq}")
        table = self.tables[seq]
        pos = self.lens[seq]
        logical = pos // self.block_size
        offset = pos % self.block_size
        cow_src = cow_dst = -1
        if logical == len(table):
            table.append(self._pop())            # the last block is full: take a new one
        else:
            blk = table[logical]
            if self.ref[blk] > 1:                 # shared: copy on write
                new = self._pop()
                self.ref[blk] -= 1
                table[logical] = new
                cow_src, cow_dst = blk, new
        self.lens[seq] = pos + 1
        return table[logical] * self.block_size + offset, cow_src, cow_dst

    def free_seq(self, seq: int):
        """A finished request: drop one reference per block; blocks nobody uses
        go back on the free list."""
        if seq not in self.tables:
            raise BadState(f"no sequence {seq}")
        for blk in reversed(self.tables.pop(seq)):
            if self.ref[blk] <= 0:
                raise BadState("reference count underflow")
            self.ref[blk] -= 1
            if self.ref[blk] == 0:
                self.free.append(blk)
        del self.lens[seq]

    # -- queries ------------------------------------------------------------------------------
    def slot(self, seq: int, pos: int) -> int:
        table = self.tables[seq]
        return table[pos // self.block_size] * self.block_size + pos % self.block_size

    def seq_slots(self, seq: int, start: int, count: int) -> list[int]:
        return [self.slot(seq, p) for p in range(start, start + count)]

    def block_table(self, seq: int) -> list[int]:
        return list(self.tables[seq])

    def num_free(self) -> int:
        return len(self.free)

    def stats(self):
        """(free blocks, token slots holding a valid token, slots allocated but empty).

        A block's filled count is the largest number of positions any
        sequence referencing it has stored in it."""
        filled: dict[int, int] = {}
        for seq, table in self.tables.items():
            n = self.lens[seq]
            for i, blk in enumerate(table):
                f = min(self.block_size, n - i * self.block_size)
                filled[blk] = max(filled.get(blk, 0), max(f, 0))
        used_blocks = self.num_blocks - len(self.free)
        used_tokens = sum(filled.values())
        return len(self.free), used_tokens, used_blocks * self.block_size - used_tokens
