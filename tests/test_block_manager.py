"""Host block manager and workload builders (CPU only)."""
import json
import os

import numpy as np
import pytest

import oracle
from paged_kv_cache_372_b200 import workloads
from paged_kv_cache_372_b200.block_manager import BlockManager, HostPool, OutOfBlocks, swap_in, swap_out

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def test_lifo_free_list_matches_pages():
    g = golden("allocator_lifo.json")
    bs = 16
    bm = BlockManager(g["max_pages"], bs)
    for (seq, pages), want in zip(g["requests"], g["expected"]):
        if want == "error":
            with pytest.raises(OutOfBlocks):
                bm.allocate(seq, pages * bs)
        else:
            assert bm.allocate(seq, pages * bs) == want


def test_kv_bytes_per_token_matches_pages():
    g = golden("kv_bytes_per_token.json")
    wl = workloads.llama7b(0, num_seqs=2)
    per_layer = wl.num_kv_heads * wl.head_dim * 2 * 2          # K and V, fp16
    assert wl.num_kv_heads * wl.head_dim == g["hidden"]
    assert per_layer * g["layers"] == g["bytes_per_token"]
    toks = int(wl.steps[0].context_lens.sum())
    assert wl.kv_bytes() == toks * per_layer


def test_page_is_4kb():
    g = golden("page_bytes.json")
    wl = workloads.llama7b(0, num_seqs=2)
    assert (wl.block_size, wl.head_dim) == (g["block_size"], g["head_dim"])
    chunk = wl.k_pool[0, 0].numel() * wl.k_pool.element_size()
    assert chunk == g["page_bytes"]


def test_cow_fork_matches_pages():
    g = golden("cow_fork.json")
    bs = 16
    bm = BlockManager(16, bs)
    bm.allocate(0, 20)                       # tail block holds 4 of 16 tokens
    tail = bm.tables[0][-1]
    for c in range(1, g["beams"] + 1):
        bm.fork(0, c)
    bm.free_seq(0)
    copies, in_place = 0, 0
    for c in range(1, g["beams"] + 1):
        r = bm.append_slot(c)
        if r.cow:
            assert r.cow[0] == tail
            copies += 1
            assert r.slot == r.cow[1] * bs + 4
        else:
            assert r.slot == tail * bs + 4
            in_place += 1
    assert (copies, in_place) == (g["expected_copies"], g["expected_in_place"])
    bm.check()


def test_full_tail_gets_fresh_block_without_copy():
    bm = BlockManager(8, 16)
    bm.allocate(0, 32)
    bm.fork(0, 1)
    r0, r1 = bm.append_slot(0), bm.append_slot(1)
    assert r0.cow is None and r1.cow is None and r0.slot != r1.slot
    assert r0.slot % 16 == 0 and r1.slot % 16 == 0
    bm.check()


def test_slots_agree_with_oracle_rule():
    rng = np.random.default_rng(0)
    bm = BlockManager(64, 16, list(rng.permutation(64)))
    seqs, pos, slots = [], [], []
    for s, n in enumerate([1, 15, 16, 17, 40]):
        bm.allocate(s, 0)
        for p in range(n):
            seqs.append(s)
            pos.append(p)
            slots.append(bm.append_slot(s).slot)
    tables = bm.block_table_array(range(5), 4, pad=0)
    want = oracle.slot_mapping(tables, seqs, pos, 16)
    assert np.array_equal(np.array(slots), want)


def test_free_returns_blocks_and_refcounts_hold():
    bm = BlockManager(10, 16)
    bm.allocate(0, 40)
    bm.fork(0, 1)
    bm.append_slot(1)
    bm.free_seq(0)
    bm.check()
    bm.free_seq(1)
    bm.check()
    assert len(bm.free) == 10


def test_tiny_workload_shape():
    wl = workloads.tiny(0)
    st = wl.steps[0]
    assert list(st.context_lens) == [1, 7, 16, 33]
    assert wl.k_pool.shape == (32, 2, 16, 64) and wl.dtype == "f16"
    assert st.copy_pairs.shape == (2, 2) and st.slot_mapping.shape == (4,)
    used = set(st.block_tables[st.block_tables >= 0].tolist())
    assert set(st.copy_pairs[:, 0].tolist()) <= used
    assert not (set(st.copy_pairs[:, 1].tolist()) & used)
    for s, n in enumerate(st.context_lens):
        last = st.block_tables[s, (n - 1) // 16] * 16 + (n - 1) % 16
        assert st.slot_mapping[s] == last


def test_beam_workload_steps_are_consistent():
    wl = workloads.beam(0, groups=2, steps=3)
    for st in wl.steps:
        B = st.q.shape[0]
        assert B == 16 and st.slot_mapping.shape == (B,)
        dst = st.copy_pairs[:, 1]
        assert len(set(dst.tolist())) == len(dst)
        assert not (set(dst.tolist()) & set(st.copy_pairs[:, 0].tolist()))
        for s in range(B):
            n = int(st.context_lens[s])
            assert st.slot_mapping[s] == st.block_tables[s, (n - 1) // 16] * 16 + (n - 1) % 16
    assert sum(len(st.copy_pairs) for st in wl.steps) > 0


def test_long_context_prefill_slots_are_free_and_distinct():
    wl = workloads.long32k(0, num_seqs=2, ctx_len=1024, prefill_tokens=256)
    st = wl.steps[0]
    pre = st.slot_mapping[2:]
    assert len(set(pre.tolist())) == 256
    used = set(st.block_tables[st.block_tables >= 0].tolist())
    assert not (set((pre // 64).tolist()) & used)


def test_swap_out_and_in_round_trip_keeps_tokens_and_refcounts():
    bm = BlockManager(12, 16, list(range(12))[::-1])
    host = HostPool(8)
    bm.allocate(0, 40)                     # 3 blocks
    bm.fork(0, 1)                          # shares them
    before = list(bm.tables[0])
    out_pairs = swap_out(bm, host, 0)
    assert [g for g, _ in out_pairs] == before and len(set(c for _, c in out_pairs)) == 3
    assert 0 not in bm.tables and all(bm.ref[b] == 1 for b in before)   # still held by seq 1
    bm.check()
    in_pairs = swap_in(bm, host, 0)
    assert [c for c, _ in in_pairs] == [c for _, c in out_pairs]
    assert bm.lens[0] == 40 and len(bm.tables[0]) == 3
    assert not set(bm.tables[0]) & set(before)                          # fresh private blocks
    assert sorted(host.free) == list(range(8))
    bm.check()


def test_swap_out_fails_cleanly_when_host_pool_is_full():
    bm = BlockManager(8, 16)
    host = HostPool(1)
    bm.allocate(0, 40)
    with pytest.raises(OutOfBlocks):
        swap_out(bm, host, 0)
    assert len(bm.tables[0]) == 3
    bm.check()


def test_beam256_workload_forks_every_beam():
    wl = workloads.beam256(0, steps=2, groups=2)
    for st in wl.steps:
        assert st.q.shape[0] == 64                        # 2 groups x 32 beams
        dst = st.copy_pairs[:, 1]
        assert len(set(dst.tolist())) == len(dst)
        assert not (set(dst.tolist()) & set(st.copy_pairs[:, 0].tolist()))
    # first step: 8 parents per group, each forked 4 ways -> 3 copies per parent with a partial tail
    assert 0 < len(wl.steps[0].copy_pairs) <= 2 * 8 * 3


def _check_decode_batch(wl, B, H, Hkv, D, bs, dtype, lo, hi):
    st = wl.steps[0]
    assert (wl.num_heads, wl.num_kv_heads, wl.head_dim, wl.block_size, wl.dtype) == (H, Hkv, D, bs, dtype)
    assert st.q.shape == (B, H, D) and st.k_new.shape[1:] == (Hkv, D)
    ctx = st.context_lens
    assert ctx.shape == (B,) and ctx.min() >= lo and ctx.max() <= hi
    need = sum(-(-int(c) // bs) for c in ctx)
    assert wl.num_blocks >= 1.25 * need - 1          # pool 1.25x what the tables hold
    used = st.block_tables[st.block_tables >= 0]
    assert len(set(used.tolist())) == len(used)      # no block is shared in a decode batch
    for s in range(B):
        n = int(ctx[s])
        assert (st.block_tables[s, :-(-n // bs)] >= 0).all()
        assert st.slot_mapping[s] == st.block_tables[s, (n - 1) // bs] * bs + (n - 1) % bs
    return ctx


def test_decode_batches_follow_the_recipe():
    ctx = _check_decode_batch(workloads.llama7b(0), 64, 32, 32, 128, 16, "f16", 128, 2048)
    assert 700 < ctx.mean() < 1400                   # uniform on [128, 2048]
    ctx = _check_decode_batch(workloads.llama3_8b(0), 256, 32, 8, 128, 16, "bf16", 16, 8192)
    assert 350 < np.median(ctx) < 750                # lognormal, median 512
    # the same batches at another block size or head size (same contexts)
    wl = workloads.llama7b(0, block_size=32, head_dim=64)
    assert wl.name == "llama7b_bs32_d64"
    _check_decode_batch(wl, 64, 32, 32, 64, 32, "f16", 128, 2048)
    assert np.array_equal(wl.steps[0].context_lens, workloads.llama7b(0).steps[0].context_lens)


def test_beam_groups_share_their_prefix():
    """Every step of the beam workload: the sequences of a group hold the same
    64 leading blocks (the 1024-token prefix), which is what shared-prefix
    decode finds and streams once per group."""
    wl = workloads.beam(0, groups=4, steps=2)
    for st in wl.steps:
        first = st.block_tables[:, 0]
        groups = {}
        for s, b in enumerate(first.tolist()):
            groups.setdefault(b, []).append(s)
        assert len(groups) == 4 and all(len(m) == 8 for m in groups.values())
        for members in groups.values():
            lead = st.block_tables[members[0]]
            for s in members[1:]:
                row = st.block_tables[s]
                lcp = 0
                while row[lcp] == lead[lcp]:
                    lcp += 1
                assert lcp >= 64
                # the block holding the sequence's newest token is its own
                n = int(st.context_lens[s])
                others = st.block_tables[[m for m in range(len(first)) if m != s]]
                assert row[(n - 1) // 16] not in set(others[others >= 0].tolist())
