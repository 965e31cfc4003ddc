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
  * Prefix caching ([深度解析 «Copy-on-Write 与 Prefix Caching»]: hash =
    hash(token_ids[0:block_size]); an existing block with the same prefix is
    referenced, O(1)).  The hash is 64-bit FNV-1a, chained: a block's hash covers
    the previous block's hash (8 little-endian bytes; 0 for the first block) and
    its token ids (4 little-endian bytes each).  Only the leading run of cached
    full blocks of a prompt is reused; later full blocks are registered; a
    partly filled block never is; a block leaves the cache when it is freed.
"""

from __future__ import annotations

FNV_OFFSET = 14695981039346656037
FNV_PRIME = 1099511628211
MASK64 = (1 << 64) - 1


def fnv1a_64(data: bytes, h: int = FNV_OFFSET) -> int:
    """64-bit FNV-1a: for each byte, h = (h XOR byte) * prime mod 2^64."""
    for byte in data:
        h = ((h ^ byte) * FNV_PRIME) & MASK64
    return h


def block_hash(parent_hash: int, token_ids) -> int:
    data = (parent_hash & MASK64).to_bytes(8, "little")
    data += b"".join((int(t) & 0xFFFFFFFF).to_bytes(4, "little") for t in token_ids)
    return fnv1a_64(data)


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
        self.cache = {}          # chained block hash -> block id
        self.hash_of = {}        # block id -> the hash it is registered under

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
            h = self.hash_of.pop(block_id, None)
            if h is not None and self.cache.get(h) == block_id:
                del self.cache[h]
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

    # -- prefix caching ([深度解析 «Copy-on-Write 与 Prefix Caching»]) ----------------
    def allocate_prompt_cached(self, token_ids):
        """(table, num_cached_tokens) for a prompt, reusing the leading cached blocks."""
        bs = self.block_size
        toks = [int(t) for t in token_ids]
        n_full = len(toks) // bs
        n_all = -(-len(toks) // bs)
        hashes, parent = [], 0
        for j in range(n_full):
            parent = block_hash(parent, toks[j * bs:(j + 1) * bs])
            hashes.append(parent)
        hits = 0
        while hits < n_full and hashes[hits] in self.cache and self.refcount[self.cache[hashes[hits]]] > 0:
            hits += 1
        if n_all - hits > len(self.free_list):
            raise PoolExhausted(f"need {n_all - hits}, {len(self.free_list)} free")
        table = []
        for j in range(hits):
            b = self.cache[hashes[j]]
            self.refcount[b] += 1
            table.append(b)
        for j in range(hits, n_all):
            b = self.free_list.pop()
            self.refcount[b] = 1
            table.append(b)
            if j < n_full:
                old = self.cache.get(hashes[j])
                if old is not None:
                    self.hash_of.pop(old, None)
                self.cache[hashes[j]] = b
                self.hash_of[b] = hashes[j]
        return table, hits * bs


def swap_plan(src: OraclePool, dst: OraclePool, table):
    """Move a table's blocks from pool `src` to pool `dst` (the swap of the GPU/CPU
    two-level allocator, [深度解析 «BlockAllocator 源码核心»]).

    Every distinct block gets one dst block, in order of first appearance; its
    dst reference count is its number of entries in the table; every entry gives
    up its reference on the src block.  Returns (new_table, [(src, dst), ...])."""
    distinct = list(dict.fromkeys(int(b) for b in table))
    for b in distinct:
        if src.refcount[b] <= 0:
            raise ValueError(f"block {b} is not allocated")
    if len(distinct) > len(dst.free_list):
        raise PoolExhausted(f"need {len(distinct)}, {len(dst.free_list)} free")
    moved, pairs = {}, []
    for b in distinct:
        d = dst.free_list.pop()
        dst.refcount[d] = 0
        moved[b] = d
        pairs.append((b, d))
    new_table = []
    for b in table:
        d = moved[int(b)]
        dst.refcount[d] += 1
        new_table.append(d)
        src.free(int(b))
    return new_table, pairs


def slot_of(table, pos: int, block_size: int) -> int:
    """Address translation of [深度解析 «Block Table 数据结构»]: pos -> physical slot."""
    return table[pos // block_size] * block_size + pos % block_size
