"""Host-side block manager: the bookkeeping that produces the decode path's inputs.

It owns no device memory. It decides which physical block of the global pool
holds each token, and it emits the three things the kernels consume:
per-sequence block tables, the slot of every new token (``slot_mapping``), and
the (src, dst) pairs of copy-on-write block copies.

Behaviour, cited by page and section:
  * "别再让GPU内存拖后腿了：vLLM的PagedAttention如何像操作系统一样管理KV Cache",
    section 2.1: a pool of fixed-size pages, a free list that hands out pages by
    popping its end, and an out-of-memory error once it is empty; section 2.2:
    pages are shared across sequences under a per-page reference count.
  * "vLLM架构深度解析：PagedAttention如何实现高吞吐LLM推理", sections 按需分配 and
    KV Cache内存共享: a block is allocated only when a token needs it; a block
    whose reference count is above one is copied (new block, copy, table
    update) before a sequence appends into it; the last holder writes in place.
  * slot = block_table[pos // block_size] * block_size + pos % block_size.
  * "vLLM架构深度解析：PagedAttention如何实现高吞吐LLM推理", section 抢占与恢复:
    a preempted sequence's blocks can be swapped out to CPU memory and back;
    ``swap_out`` / ``swap_in`` plan those copies against a host block pool.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np


class OutOfBlocks(MemoryError):
    """The free list is empty."""


@dataclass
class AppendResult:
    slot: int
    cow: tuple[int, int] | None = None  # (src, dst) block copy needed before the write


@dataclass
class BlockManager:
    num_blocks: int
    block_size: int
    free_order: list[int] | None = None
    free: list[int] = field(init=False)
    ref: list[int] = field(init=False)
    tables: dict[int, list[int]] = field(init=False, default_factory=dict)
    lens: dict[int, int] = field(init=False, default_factory=dict)

    def __post_init__(self):
        order = list(range(self.num_blocks)) if self.free_order is None else list(self.free_order)
        if sorted(order) != list(range(self.num_blocks)):
            raise ValueError("free_order must be a permutation of range(num_blocks)")
        self.free = order
        self.ref = [0] * self.num_blocks

    # -- allocation -----------------------------------------------------------
    def _pop(self) -> int:
        if not self.free:
            raise OutOfBlocks("no free blocks in the pool")
        b = self.free.pop()
        assert self.ref[b] == 0
        self.ref[b] = 1
        return b

    def _release(self, b: int) -> None:
        assert self.ref[b] > 0
        self.ref[b] -= 1
        if self.ref[b] == 0:
            self.free.append(b)

    def allocate(self, seq: int, num_tokens: int) -> list[int]:
        """New sequence holding num_tokens tokens (blocks for all of them)."""
        if seq in self.tables:
            raise KeyError(f"sequence {seq} exists")
        need = -(-num_tokens // self.block_size)
        if need > len(self.free):
            raise OutOfBlocks("no free blocks in the pool")
        self.tables[seq] = [self._pop() for _ in range(need)]
        self.lens[seq] = num_tokens
        return list(self.tables[seq])

    def fork(self, parent: int, child: int) -> None:
        """child shares every block of parent (reference counts go up)."""
        if child in self.tables:
            raise KeyError(f"sequence {child} exists")
        self.tables[child] = list(self.tables[parent])
        self.lens[child] = self.lens[parent]
        for b in self.tables[child]:
            self.ref[b] += 1

    def free_seq(self, seq: int) -> None:
        for b in self.tables.pop(seq):
            self._release(b)
        del self.lens[seq]

    def append_slot(self, seq: int) -> AppendResult:
        """Reserve the slot of the sequence's next token (copy-on-write if shared)."""
        pos = self.lens[seq]
        table = self.tables[seq]
        cow = None
        if pos % self.block_size == 0:
            table.append(self._pop())
        else:
            tail = table[-1]
            if self.ref[tail] > 1:
                new = self._pop()
                self.ref[tail] -= 1
                table[-1] = new
                cow = (tail, new)
        slot = table[pos // self.block_size] * self.block_size + pos % self.block_size
        self.lens[seq] = pos + 1
        return AppendResult(slot, cow)

    # -- views ------------------------------------------------------------------
    def block_table_array(self, seqs, width: int, pad: int = -1) -> np.ndarray:
        out = np.full((len(seqs), width), pad, dtype=np.int32)
        for i, s in enumerate(seqs):
            t = self.tables[s]
            if len(t) > width:
                raise ValueError(f"sequence {s} needs {len(t)} blocks > width {width}")
            out[i, :len(t)] = t
        return out

    def context_lens(self, seqs) -> np.ndarray:
        return np.array([self.lens[s] for s in seqs], dtype=np.int32)

    def used_blocks(self) -> int:
        return self.num_blocks - len(self.free)

    def shared_blocks(self) -> int:
        return sum(1 for r in self.ref if r > 1)

    def check(self) -> None:
        """Internal consistency: reference counts equal table occurrences."""
        count = [0] * self.num_blocks
        for t in self.tables.values():
            for b in t:
                count[b] += 1
        assert count == self.ref, "reference counts disagree with the tables"
        assert sorted(self.free) == [b for b in range(self.num_blocks) if count[b] == 0]


@dataclass
class HostPool:
    """Free list of a page-locked host pool holding swapped-out blocks."""
    num_blocks: int
    free: list[int] = field(init=False)
    tables: dict[int, list[int]] = field(init=False, default_factory=dict)
    lens: dict[int, int] = field(init=False, default_factory=dict)

    def __post_init__(self):
        self.free = list(range(self.num_blocks))


def swap_out(bm: BlockManager, host: HostPool, seq: int) -> list[tuple[int, int]]:
    """Move sequence `seq` to the host pool: returns (gpu block, host block) copy
    pairs and releases the GPU blocks (a shared block stays with its other holders)."""
    table = bm.tables[seq]
    if len(table) > len(host.free):
        raise OutOfBlocks("no free blocks in the host pool")
    pairs = [(g, host.free.pop()) for g in table]
    host.tables[seq] = [c for _, c in pairs]
    host.lens[seq] = bm.lens[seq]
    bm.free_seq(seq)
    return pairs


def swap_in(bm: BlockManager, host: HostPool, seq: int) -> list[tuple[int, int]]:
    """Bring sequence `seq` back into fresh GPU blocks: returns (host block, gpu
    block) copy pairs and releases the host blocks."""
    cpu = host.tables[seq]
    if len(cpu) > len(bm.free):
        raise OutOfBlocks("no free blocks in the pool")
    if seq in bm.tables:
        raise KeyError(f"sequence {seq} is resident")
    del host.tables[seq]
    gpu = [bm._pop() for _ in cpu]
    bm.tables[seq] = gpu
    bm.lens[seq] = host.lens.pop(seq)
    host.free.extend(reversed(cpu))
    return list(zip(cpu, gpu))
