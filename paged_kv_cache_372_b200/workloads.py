"""The five synthetic decode workloads, built on the host from seeded draws.

A workload is an initial K/V pool plus a list of decode steps. One step is the
hot path once, in order:

  1. ``pa_copy_blocks``       copy-on-write copies planned by the block manager,
  2. ``pa_reshape_and_cache`` write each new token's K/V into its slot,
  3. ``pa_decode``            every sequence's query attends over its blocks.

Context lengths are post-append: a step's new token is the last one attended.
All values are N(0,1) cast to the element type; pools are filled everywhere,
including blocks no table references. Block placement comes from a
``BlockManager`` whose free list is a seeded shuffle of the pool.

Workloads (sizes as named):
  tiny       4 seqs, ctx {1,7,16,33}, H=Hkv=2, D=64, bs=16, fp16, 32 blocks;
             4 appended tokens and 2 block copies.
  llama7b    64 seqs, H=Hkv=32, D=128, bs=16, fp16, ctx uniform in [128, 2048],
             pool 1.25x the blocks needed.
  llama3_8b  256 seqs, H=32, Hkv=8, D=128, bs=16, bf16, ctx lognormal
             (median 512, sigma 1) clipped to [16, 8192], pool 1.25x needed.
  beam       8 groups x 8 seqs sharing a 1024-token prefix per group, suffixes
             uniform in [16, 512]; H=32, Hkv=8, D=128, bs=16, bf16; each step
             keeps 2 parents per group and forks each into 4 beams, so appends
             into a shared partly-filled tail block copy it first.
  beam256    the other reading of beam: all 8 sequences of a group fork 4 ways
             (256 sequences per step; 8 of a group's 32 beams are kept later).
  long32k    8 seqs at ctx 32768, H=32, Hkv=8, D=128, bs=64, bf16, 512-token
             split-context partitions; the same step also writes 4096 prefill
             tokens into distinct random free slots.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np
import torch

from . import inputs
from .block_manager import BlockManager

NAMES = ("tiny", "llama7b", "llama3_8b", "beam", "beam256", "long32k")


@dataclass
class Step:
    q: torch.Tensor               # [B][H][D]
    block_tables: np.ndarray      # int32 [B][W]
    context_lens: np.ndarray      # int32 [B]
    k_new: torch.Tensor           # [T][Hkv][D]
    v_new: torch.Tensor           # [T][Hkv][D]
    slot_mapping: np.ndarray      # int64 [T]
    copy_pairs: np.ndarray        # int64 [P][2]


@dataclass
class Workload:
    name: str
    dtype: str
    num_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    num_blocks: int
    partition_size: int
    k_pool: torch.Tensor          # [NB][Hkv][bs][D]
    v_pool: torch.Tensor
    steps: list[Step] = field(default_factory=list)

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.head_dim)

    @property
    def num_seqs(self) -> int:
        return int(self.steps[0].q.shape[0])

    @property
    def block_bytes(self) -> int:
        """Bytes of one physical block of one pool (all KV heads)."""
        return self.num_kv_heads * self.block_size * self.head_dim * 2

    def kv_bytes(self, step: int = 0) -> int:
        """Algorithmic K+V bytes one decode reads: valid tokens only, counted
        once per sequence (logical bytes; shared blocks count every time)."""
        return int(self.steps[step].context_lens.astype(np.int64).sum()) * \
            self.num_kv_heads * self.head_dim * 2 * 2

    def kv_bytes_unique(self, step: int = 0) -> int:
        """K+V bytes of the distinct physical block slots one decode reads:
        a block shared by several sequences counts once (its longest use)."""
        st = self.steps[step]
        used = {}
        for s, n in enumerate(st.context_lens):
            n = int(n)
            for j in range(-(-n // self.block_size)):
                b = int(st.block_tables[s, j])
                used[b] = max(used.get(b, 0), min(self.block_size, n - j * self.block_size))
        return sum(used.values()) * self.num_kv_heads * self.head_dim * 2 * 2


def _pool(num_blocks, hkv, bs, d, dtype, gen):
    return inputs.normal((num_blocks, hkv, bs, d), dtype, gen)


def _decode_batch(name, ctx, *, heads, kv_heads, head_dim, block_size, dtype, seed,
                  partition_size=0, pool_factor=1.25, extra_blocks=0, prefill_tokens=0):
    """Sequences laid out by a shuffled free list; each appends its last token."""
    gen = inputs.generator(seed)
    need = sum(-(-c // block_size) for c in ctx)
    nb = int(math.ceil(pool_factor * (need + extra_blocks)))
    bm = BlockManager(nb, block_size, inputs.permutation(nb, gen))
    seqs = list(range(len(ctx)))
    slots = []
    for s, c in zip(seqs, ctx):
        bm.allocate(s, c - 1)
        slots.append(bm.append_slot(s).slot)
    width = max(len(t) for t in bm.tables.values())
    T = len(ctx)
    if prefill_tokens:
        used = set(b for t in bm.tables.values() for b in t)
        free_blocks = [b for b in range(nb) if b not in used]
        cand = inputs.choice(len(free_blocks) * block_size, prefill_tokens, gen)
        slots += [free_blocks[c // block_size] * block_size + c % block_size for c in cand]
        T += prefill_tokens
    step = Step(
        q=inputs.normal((len(ctx), heads, head_dim), dtype, gen),
        block_tables=bm.block_table_array(seqs, width),
        context_lens=bm.context_lens(seqs),
        k_new=inputs.normal((T, kv_heads, head_dim), dtype, gen),
        v_new=inputs.normal((T, kv_heads, head_dim), dtype, gen),
        slot_mapping=np.array(slots, dtype=np.int64),
        copy_pairs=np.zeros((0, 2), dtype=np.int64),
    )
    wl = Workload(name, dtype, heads, kv_heads, head_dim, block_size, nb, partition_size,
                  _pool(nb, kv_heads, block_size, head_dim, dtype, gen),
                  _pool(nb, kv_heads, block_size, head_dim, dtype, gen), [step])
    return wl, bm


def tiny(seed: int = 0) -> Workload:
    gen = inputs.generator(seed + 1000)
    ctx = [1, 7, 16, 33]
    nb, bs, hkv, d = 32, 16, 2, 64
    wl = Workload("tiny", "f16", 2, hkv, d, bs, nb, 0,
                  _pool(nb, hkv, bs, d, "f16", gen), _pool(nb, hkv, bs, d, "f16", gen))
    bm = BlockManager(nb, bs, inputs.permutation(nb, gen))
    slots = []
    for s, c in enumerate(ctx):
        bm.allocate(s, c - 1)
        slots.append(bm.append_slot(s).slot)
    used = sorted(set(b for t in bm.tables.values() for b in t))
    src = [used[i] for i in inputs.choice(len(used), 2, gen)]
    bm.allocate(99, 2 * bs)                 # two fresh blocks receive the copies
    dst = bm.tables[99]
    seqs = list(range(len(ctx)))
    wl.steps.append(Step(
        q=inputs.normal((4, 2, d), "f16", gen),
        block_tables=bm.block_table_array(seqs, 4),
        context_lens=bm.context_lens(seqs),
        k_new=inputs.normal((4, hkv, d), "f16", gen),
        v_new=inputs.normal((4, hkv, d), "f16", gen),
        slot_mapping=np.array(slots, dtype=np.int64),
        copy_pairs=np.array(list(zip(src, dst)), dtype=np.int64),
    ))
    return wl


def _shape_name(base: str, block_size: int, head_dim: int, kv_heads: int | None = None) -> str:
    """Name of a workload run at a block size / head size (/ KV head count)
    other than its own."""
    name = base if (block_size, head_dim) == (16, 128) else f"{base}_bs{block_size}_d{head_dim}"
    return name if kv_heads is None else f"{name}_kv{kv_heads}"


def llama7b(seed: int = 0, num_seqs: int = 64, block_size: int = 16, head_dim: int = 128) -> Workload:
    gen = inputs.generator(seed + 2000)
    ctx = inputs.uniform_int(128, 2048, num_seqs, gen)
    wl, _ = _decode_batch(_shape_name("llama7b", block_size, head_dim), ctx, heads=32, kv_heads=32,
                          head_dim=head_dim, block_size=block_size, dtype="f16", seed=seed + 2001)
    return wl


def llama3_8b(seed: int = 0, num_seqs: int = 256, block_size: int = 16, head_dim: int = 128,
              kv_heads: int = 8) -> Workload:
    gen = inputs.generator(seed + 3000)
    ctx = inputs.lognormal_int(512.0, 1.0, 16, 8192, num_seqs, gen)
    wl, _ = _decode_batch(_shape_name("llama3_8b", block_size, head_dim, None if kv_heads == 8 else kv_heads), ctx,
                          heads=32, kv_heads=kv_heads, head_dim=head_dim, block_size=block_size, dtype="bf16",
                          seed=seed + 3001)
    return wl


def long32k(seed: int = 0, num_seqs: int = 8, ctx_len: int = 32768,
            prefill_tokens: int = 4096) -> Workload:
    ctx = [ctx_len] * num_seqs
    wl, _ = _decode_batch("long32k", ctx, heads=32, kv_heads=8, head_dim=128, block_size=64,
                          dtype="bf16", seed=seed + 5001, partition_size=512,
                          extra_blocks=-(-prefill_tokens // 64), prefill_tokens=prefill_tokens)
    return wl


def beam(seed: int = 0, groups: int = 8, width: int = 8, prefix: int = 1024,
         steps: int = 8, parents: int = 2, initial: int | None = None, name: str = "beam") -> Workload:
    """Shared prefix + beam fork. A group starts with `initial` sequences (default
    `width`) sharing the prefix, each with its own suffix. Per step and group:
    keep `parents` beams, fork each into width // parents children, free the
    rest, and append one token per child."""
    gen = inputs.generator(seed + 4000)
    bs, hkv, heads, d, dtype = 16, 8, 32, 128, "bf16"
    start = width if initial is None else initial
    suffix = inputs.uniform_int(16, 512, groups * start, gen)
    need = groups * (prefix // bs) + sum(-(-x // bs) + 1 for x in suffix)
    nb = int(math.ceil(1.25 * need)) + steps * groups * width * 2
    bm = BlockManager(nb, bs, inputs.permutation(nb, gen))
    live = []
    for g in range(groups):
        root = g * start
        bm.allocate(root, prefix)
        for j in range(1, start):
            bm.fork(root, root + j)
        for j in range(start):
            for _ in range(suffix[root + j]):
                bm.append_slot(root + j)
        live.append([root + j for j in range(start)])
    next_id = groups * start
    plans = []
    for _ in range(steps):
        pairs, slots, order = [], [], []
        for g in range(groups):
            keep = [live[g][i] for i in inputs.choice(len(live[g]), parents, gen)]
            children = []
            for p in keep:
                for _ in range(width // parents):
                    bm.fork(p, next_id)
                    children.append(next_id)
                    next_id += 1
            for s in live[g]:
                bm.free_seq(s)
            for c in children:
                r = bm.append_slot(c)
                if r.cow is not None:
                    pairs.append(r.cow)
                slots.append(r.slot)
            live[g] = children
            order += children
        bm.check()
        plans.append((order, pairs, slots, {s: list(bm.tables[s]) for s in order},
                      bm.context_lens(order)))
    width_blocks = max(len(t) for _, _, _, tabs, _ in plans for t in tabs.values())
    wl = Workload(name, dtype, heads, hkv, d, bs, nb, 0,
                  _pool(nb, hkv, bs, d, dtype, gen), _pool(nb, hkv, bs, d, dtype, gen))
    for order, pairs, slots, tabs, lens in plans:
        bt = np.full((len(order), width_blocks), -1, dtype=np.int32)
        for i, s in enumerate(order):
            bt[i, :len(tabs[s])] = tabs[s]
        T = len(order)
        wl.steps.append(Step(
            q=inputs.normal((T, heads, d), dtype, gen),
            block_tables=bt, context_lens=lens,
            k_new=inputs.normal((T, hkv, d), dtype, gen),
            v_new=inputs.normal((T, hkv, d), dtype, gen),
            slot_mapping=np.array(slots, dtype=np.int64),
            copy_pairs=np.array(pairs, dtype=np.int64).reshape(-1, 2),
        ))
    return wl


def beam256(seed: int = 0, steps: int = 8, groups: int = 8) -> Workload:
    """The other reading of the beam workload: every one of a group's 8
    sequences forks 4 ways (32 per group, 256 in all); later steps keep 8 of a
    group's 32 beams and fork each 4 ways again."""
    return beam(seed, groups=groups, width=32, prefix=1024, steps=steps, parents=8, initial=8, name="beam256")


def build(name: str, seed: int = 0, **kw) -> Workload:
    return {"tiny": tiny, "llama7b": llama7b, "llama3_8b": llama3_8b, "beam": beam, "beam256": beam256,
            "long32k": long32k}[name](seed, **kw)
