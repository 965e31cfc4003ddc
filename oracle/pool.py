"""Plain-Python block pool: the oracle for the host-side KV block manager.

TEST INFRASTRUCTURE ONLY -- never imported by the product package.

Pages followed:
  [源码解析]  "vLLM 源码解析：PagedAttention 如何让大模型推理提速 10 倍", §三 (BlockAllocator:
              allocate / free / get_num_free_blocks; the page table), §五
              (CopyOnWriteBlockAllocator.allocate_or_get_cow), §六 (a new page only when
              the last one is full: token 5 -> 1 page, token 17 -> 2 pages at 16 tokens/page).
  [深度解析]  "vLLM 核心源码深度解析 …", «内存分配与回收流程» (free_list, O(1) pop / push,
              all blocks returned when a request finishes), «Copy-on-Write 与 Prefix Caching»
              (shared prompt blocks, reference count; on a write: copy, write the new value,
              reference count minus one), «核心方法 allocate» (free_list.pop()).
  [论文专题]  "论文专题讲解：vLLM / PagedAttention：为什么 KV cache 需要分页管理",
              «Block table：为什么它能减少碎片» (Figure 6 text: block size 4, a 7-token prompt
              takes 2 logical blocks filled 4 + 3 with 1 free slot; the next decode writes into
              that slot, and a new physical block is requested only when the last is full),
              «共享前缀和 copy-on-write» (copy before the write when a block's reference
              count is above 1).

Readings where the pages are silent:
  * The free list pops from its END (Python list.pop()), freed blocks are appended at
    the end.  The initial order is supplied by the caller.
  * A block whose reference count reaches 0 returns to the free list.
  * Copy-on-write is decided per write: reference count > 1 -> take a fresh block,
    record (src, dst), decrement src.  The last remaining owner writes in place.
"""

from __future__ import annotations


class PoolExhausted(RuntimeError):
    """Raised when allocate() asks for more blocks than are free (can_allocate false)."""


class OraclePool:
    def __init__(self, num_blocks: int, block_size: int, free_order=None):
        if free_order is None:
            free_order = list(range(num_blocks))
        free_order = [int(b) for b in free_order]
        if sorted(free_order) != list(range(num_blocks)):
            raise ValueError("free_order must be a permutation of range(num_blocks)")
        self.num_blocks = num_blocks
        self.block_size = block_size
        self.free_list = list(free_order)
        self.refcount = [0] * num_blocks

    # -- BlockAllocator ([源码解析 §三]) --------------------------------------
    def get_num_free_blocks(self) -> int:
        return len(self.free_list)

    def allocate(self, num_blocks: int) -> list[int]:
        if num_blocks > len(self.free_list):
            raise PoolExhausted(f"need {num_blocks}, {len(self.free_list)} free")
        out = []
        for _ in range(num_blocks):
            b = self.free_list.pop()
            self.refcount[b] = 1
            out.append(b)
        return out

    def free(self, block_id: int) -> None:
        if self.refcount[block_id] <= 0:
            raise ValueError(f"block {block_id} is not allocated")
        self.refcount[block_id] -= 1
        if self.refcount[block_id] == 0:
            self.free_list.append(block_id)

    # -- sharing and copy-on-write ([源码解析 §五], [论文专题 共享前缀和 copy-on-write]) --
    def fork(self, table: list[int]) -> list[int]:
        """A second owner of every block in `table` (parallel sampling / beam search)."""
        for b in table:
            if self.refcount[b] <= 0:
                raise ValueError(f"block {b} is not allocated")
            self.refcount[b] += 1
        return list(table)

    def allocate_or_get_cow(self, block_id: int):
        """Return (block to write, (src, dst) pair or None)."""
        if self.refcount[block_id] > 1:
            new_id = self.allocate(1)[0]
            self.refcount[block_id] -= 1
            return new_id, (block_id, new_id)
        return block_id, None

    # -- one sequence's growth by one token ([源码解析 §六], [论文专题 Figure 6]) --------
    def append_token(self, table: list[int], pos: int):
        """Make room for the token at logical position `pos` (= tokens already cached).

        Returns (slot, pair, allocated) where pair is the copy-on-write (src, dst) or
        None and allocated says whether a fresh block was taken for a new page.
        The table is updated in place.
        """
        bs = self.block_size
        logical = pos // bs
        offset = pos % bs
        allocated = False
        pair = None
        if logical == len(table):
            if offset != 0:
                raise ValueError("position skips a block")
            table.append(self.allocate(1)[0])
            allocated = True
        elif logical < len(table):
            new_id, pair = self.allocate_or_get_cow(table[logical])
            table[logical] = new_id
        else:
            raise ValueError("position beyond the table")
        slot = table[logical] * bs + offset
        return slot, pair, allocated

    def allocate_prompt(self, num_tokens: int) -> list[int]:
        """Blocks for a prompt of num_tokens: ceil(num_tokens / block_size) of them."""
        need = -(-num_tokens // self.block_size)
        return self.allocate(need)

    def free_sequence(self, table: list[int]) -> None:
        for b in table:
            self.free(b)
        table.clear()

    def utilisation(self, tables, seq_lens) -> float:
        """Live tokens / slots of the distinct blocks in use."""
        used = {b for t in tables for b in t}
        live = sum(int(x) for x in seq_lens)
        return live / (len(used) * self.block_size) if used else 0.0


def slot_of(table, pos: int, block_size: int) -> int:
    """Address translation of [深度解析 «Block Table 数据结构»]: pos -> physical slot."""
    return table[pos // block_size] * block_size + pos % block_size
