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
  writes in place;
* sliding window: blocks that fall wholly out of the attention window are
  given back (second page, section 5.2). Here a block is out of the window
  of length W when all its positions precede len - W; the sequence drops its
  reference and its table entry becomes -1;
* swapping: a preempted request's blocks move to CPU memory and come back
  later (third page, section "分页还顺带解决了什么"; second page, section 3.1,
  swap_out of a victim). Here a group of sequences moves together: each
  distinct block the group uses is copied once into a free host block (its
  host count = the group's references), the device block loses those
  references, and the tables then name host blocks; swapping in is the
  mirror image. A block also used outside the group stays where it is for
  the others, so the group gets its own copy;
* prefix caching: requests whose prompts begin with the same tokens point
  their first blocks at the same physical blocks, and only completely
  filled blocks are shared (third page, section "分页还顺带解决了什么"); the
  KV of a common prompt prefix is kept as a cache (first page, section 9).
  Here a cached block stands for the whole token prefix up to its end. A
  new prompt shares, from its start, every full block whose prefix is
  cached, except that the block holding the prompt's last token is never
  looked up (that token's attention must be computed); then each full block
  of the prompt whose prefix is not cached yet is recorded. A cached block
  nobody uses any more stays cached and counts as free; it is reused only
  when no plain free block is left, the one released longest ago first, and
  only its own prefix is then forgotten.

Which physical id the free list hands out is not fixed by the pages; this
model pops the most recently freed block (a LIFO stack). Tests compare the
product allocator with this model only up to a relabelling of ids.
"""
from __future__ import annotations

from collections import OrderedDict


RELEASED = -1  # table entry of a block given back by the sliding window


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
        self.swapped: set[int] = set()
        self.host_free: list[int] = []
        self.host_ref: list[int] = []
        # prefix cache: token prefix (whole blocks) -> the block holding its last block
        self.cached: dict[tuple, int] = {}
        self.prefix_of: dict[int, tuple] = {}
        self.idle: OrderedDict[int, None] = OrderedDict()  # unused cached blocks, oldest first

    # -- allocation ---------------------------------------------------------------------------
    def _blocks_for(self, num_tokens: int) -> int:
        # whole blocks needed to hold num_tokens tokens
        return -(-num_tokens // self.block_size)

    def _pop(self) -> int:
        if self.free:
            blk = self.free.pop()
        elif self.idle:
            blk = next(iter(self.idle))  # the unused cached block released longest ago
            del self.idle[blk]
            del self.cached[self.prefix_of.pop(blk)]
        else:
            raise OutOfBlocks("free list is empty")
        self.ref[blk] = 1
        return blk

    def _release(self, blk: int):
        """blk's last reference is gone."""
        if blk in self.prefix_of:
            self.idle[blk] = None
        else:
            self.free.append(blk)

    def add_seq(self, seq: int, num_tokens: int) -> list[int]:
        """A new request: take the blocks its prompt needs, all or none."""
        if seq in self.tables:
            raise BadState(f"sequence {seq} exists")
        if num_tokens < 0:
            raise ValueError("negative length")
        need = self._blocks_for(num_tokens)
        if need > self.num_free():
            raise OutOfBlocks(f"need {need} blocks, {self.num_free()} free")
        self.tables[seq] = [self._pop() for _ in range(need)]
        self.lens[seq] = num_tokens
        return list(self.tables[seq])

    def add_seq_cached(self, seq: int, tokens) -> int:
        """A new request with prompt ``tokens``: share its cached leading full
        blocks, take the rest from the free list (all or none), record its full
        blocks. Returns the number of positions already held (shared blocks x
        block size)."""
        if seq in self.tables:
            raise BadState(f"sequence {seq} exists")
        tokens = [int(t) for t in tokens]
        n, bs = len(tokens), self.block_size
        shared = []
        for i in range(max(n - 1, 0) // bs):  # full blocks before the last token
            blk = self.cached.get(tuple(tokens[:(i + 1) * bs]))
            if blk is None:
                break
            shared.append(blk)
        need = self._blocks_for(n) - len(shared)
        unused = sum(1 for b in shared if self.ref[b] == 0)  # counted as free until shared
        if need > self.num_free() - unused:
            raise OutOfBlocks(f"need {need} blocks, {self.num_free() - unused} free")
        for b in shared:
            self.idle.pop(b, None)
            self.ref[b] += 1
        table = shared + [self._pop() for _ in range(need)]
        for i in range(len(shared), n // bs):
            key = tuple(tokens[:(i + 1) * bs])
            if key not in self.cached:
                self.cached[key] = table[i]
                self.prefix_of[table[i]] = key
        self.tables[seq] = table
        self.lens[seq] = n
        return len(shared) * bs

    def cached_blocks(self):
        """(blocks holding a cached prefix, of which unused)."""
        return len(self.cached), len(self.idle)

    def reset_prefix_cache(self):
        self.free.extend(self.idle)
        self.idle.clear()
        self.cached.clear()
        self.prefix_of.clear()

    def fork(self, parent: int, child: int):
        """The child shares every block of the parent; each gains a reference."""
        if parent not in self.tables or child in self.tables or parent in self.swapped:
            raise BadState("bad fork")
        self.tables[child] = list(self.tables[parent])
        self.lens[child] = self.lens[parent]
        for blk in self.tables[child]:
            if blk != RELEASED:
                self.ref[blk] += 1

    def append_slot(self, seq: int):
        """Reserve the slot of the sequence's next token.

        Returns (slot, cow_src, cow_dst); cow_* are -1 unless the write had
        to copy a shared block first. Nothing changes if no block is free."""
        if seq not in self.tables or seq in self.swapped:
            raise BadState(f"no resident sequence {seq}")
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
        host = seq in self.swapped
        ref = self.host_ref if host else self.ref
        for blk in reversed(self.tables.pop(seq)):
            if blk == RELEASED:
                continue
            if ref[blk] <= 0:
                raise BadState("reference count underflow")
            ref[blk] -= 1
            if ref[blk] == 0:
                if host:
                    self.host_free.append(blk)
                else:
                    self._release(blk)
        del self.lens[seq]
        self.swapped.discard(seq)

    def slide_window(self, seq: int, window: int) -> int:
        """Give back every block whose positions all precede len - window.
        Returns how many blocks went back on the free list."""
        if seq not in self.tables or seq in self.swapped:
            raise BadState(f"no resident sequence {seq}")
        if window <= 0:
            raise ValueError("window must be positive")
        start = max(0, self.lens[seq] - window)      # first position inside the window
        table = self.tables[seq]
        freed = 0
        for i in range(start // self.block_size):     # blocks ending at or before start
            blk = table[i]
            if blk == RELEASED:
                continue
            table[i] = RELEASED
            self.ref[blk] -= 1
            if self.ref[blk] == 0:
                self._release(blk)
                freed += 1
        return freed

    # -- swapping -----------------------------------------------------------------------------
    def set_host_blocks(self, num_host_blocks: int):
        if self.host_ref:
            raise BadState("swap space already set")
        self.host_ref = [0] * num_host_blocks
        self.host_free = list(range(num_host_blocks - 1, -1, -1))

    def _swap(self, seqs, out: bool):
        if not self.host_ref:
            raise BadState("no swap space")
        if len(set(seqs)) != len(seqs):
            raise ValueError("sequence listed twice")
        for s in seqs:
            if s not in self.tables or (s in self.swapped) == out:
                raise BadState(f"sequence {s} is not on the side it leaves")
        order, refs = [], {}
        for s in seqs:
            for blk in self.tables[s]:
                if blk == RELEASED:
                    continue
                if blk not in refs:
                    refs[blk] = 0
                    order.append(blk)
                refs[blk] += 1
        src_ref = self.ref if out else self.host_ref
        dst_ref = self.host_ref if out else self.ref
        room = len(self.host_free) if out else self.num_free()
        if len(order) > room:
            raise OutOfBlocks(f"need {len(order)} blocks on the other side, {room} free")
        moved, pairs = {}, []
        for blk in order:
            new = self.host_free.pop() if out else self._pop()
            dst_ref[new] = refs[blk]
            src_ref[blk] -= refs[blk]
            if src_ref[blk] == 0:
                if out:
                    self._release(blk)
                else:
                    self.host_free.append(blk)
            moved[blk] = new
            pairs.append((blk, new))
        for s in seqs:
            self.tables[s] = [moved[b] if b != RELEASED else RELEASED for b in self.tables[s]]
            if out:
                self.swapped.add(s)
            else:
                self.swapped.discard(s)
        return pairs

    def swap_out(self, seqs):
        """Move a group to the host swap space; returns (device block, host block) pairs."""
        return self._swap(list(seqs), True)

    def swap_in(self, seqs):
        """Bring a swapped group back; returns (host block, device block) pairs."""
        return self._swap(list(seqs), False)

    # -- queries ------------------------------------------------------------------------------
    def slot(self, seq: int, pos: int) -> int:
        table = self.tables[seq]
        blk = table[pos // self.block_size]
        if blk == RELEASED:
            raise BadState("position released by the sliding window")
        return blk * self.block_size + pos % self.block_size

    def seq_slots(self, seq: int, start: int, count: int) -> list[int]:
        return [self.slot(seq, p) for p in range(start, start + count)]

    def block_table(self, seq: int) -> list[int]:
        return list(self.tables[seq])

    def num_free(self) -> int:
        return len(self.free) + len(self.idle)

    def stats(self):
        """(free blocks, token slots holding a valid token, slots allocated but empty).

        A block's filled count is the largest number of positions any
        sequence referencing it has stored in it."""
        filled: dict[int, int] = {}
        for seq, table in self.tables.items():
            if seq in self.swapped:
                continue
            n = self.lens[seq]
            for i, blk in enumerate(table):
                if blk == RELEASED:
                    continue
                f = min(self.block_size, n - i * self.block_size)
                filled[blk] = max(filled.get(blk, 0), max(f, 0))
        used_blocks = self.num_blocks - self.num_free()
        used_tokens = sum(filled.values())
        return self.num_free(), used_tokens, used_blocks * self.block_size - used_tokens
