"""GPU invariants the pages fix, checked bit-exactly on the CUDA path, plus the
error paths of the C ABI (status codes and device error bits, no faults)."""
import numpy as np
import pytest
import torch

import paged_kv_cache_372_b200 as pa
from paged_kv_cache_372_b200 import workloads

pytestmark = pytest.mark.gpu


def decode(wl, kp, vp, tables, ctx, q=None, partition=0):
    st = wl.steps[0]
    q = (st.q if q is None else q).cuda()
    out = torch.full_like(q, float("nan"))  # every row must be written
    pa.pa_decode(out, q, kp, vp, torch.as_tensor(tables).cuda(), torch.as_tensor(ctx).cuda(),
                 wl.scale, int(np.max(ctx)), partition)
    torch.cuda.synchronize()
    return out


@pytest.mark.parametrize("partition", [0, 256, 16])
def test_block_permutation_bit_identical(partition):
    """Physical placement of blocks does not change the result: with one merge
    level (auto: at most 8 partitions a sequence here), two (256-token
    partitions: up to 16, in chunks of 8) and the merge in a launch of its own
    (16-token partitions: up to 248)."""
    wl = workloads.llama3_8b(4, num_seqs=16)
    st = wl.steps[0]
    kp, vp = wl.k_pool.cuda(), wl.v_pool.cuda()
    a = decode(wl, kp, vp, st.block_tables, st.context_lens, partition=partition)
    pi = torch.randperm(wl.num_blocks, generator=torch.Generator().manual_seed(0))
    kp2 = torch.empty_like(kp)
    vp2 = torch.empty_like(vp)
    kp2[pi.cuda()] = kp
    vp2[pi.cuda()] = vp
    tab = st.block_tables.copy()
    tab[tab >= 0] = pi.numpy()[tab[tab >= 0]]
    b = decode(wl, kp2, vp2, tab, st.context_lens, partition=partition)
    assert torch.equal(a, b)


def test_shared_equals_duplicated_bit_identical():
    """A copy-on-write-shared block gives the same result as a duplicated one."""
    wl = workloads.llama7b(5, num_seqs=4)
    st = wl.steps[0]
    kp, vp = wl.k_pool.cuda(), wl.v_pool.cuda()
    used = set(st.block_tables[st.block_tables >= 0].tolist())
    free_all = [b for b in range(wl.num_blocks) if b not in used]
    ctx = st.context_lens.copy()
    ctx[0] = min(int(ctx[0]), wl.block_size * len(free_all) - 3)   # ragged tail
    ctx[1] = ctx[0]
    q = st.q.clone()
    q[1] = q[0]
    shared = st.block_tables.copy()
    nblk = -(-int(ctx[0]) // wl.block_size)
    shared[1, :nblk] = shared[0, :nblk]
    # duplicated: sequence 1 gets byte copies of sequence 0's blocks in fresh blocks
    free = free_all[:nblk]
    assert len(free) == nblk
    dup = st.block_tables.copy()
    dup[1, :] = -1
    dup[1, :nblk] = free
    pairs = torch.tensor([[shared[0, j], free[j]] for j in range(nblk)], dtype=torch.int64).cuda()
    pa.pa_copy_blocks([kp, vp], pairs)
    a = decode(wl, kp, vp, shared, ctx, q)
    b = decode(wl, kp, vp, dup, ctx, q)
    assert torch.equal(a, b)
    assert torch.equal(a[0], a[1])


@pytest.mark.parametrize("name", ["tiny", "llama3_8b"])
def test_single_token_returns_value_row(name):
    wl = workloads.build(name, 6, **({} if name == "tiny" else {"num_seqs": 8}))
    st = wl.steps[0]
    ctx = np.ones_like(st.context_lens)
    kp, vp = wl.k_pool.cuda(), wl.v_pool.cuda()
    out = decode(wl, kp, vp, st.block_tables, ctx)
    G = wl.num_heads // wl.num_kv_heads
    for s in range(len(ctx)):
        rows = wl.v_pool[int(st.block_tables[s, 0])][:, 0, :]         # [Hkv][D]
        assert torch.equal(out[s].cpu(), rows.repeat_interleave(G, dim=0))


def test_nan_tail_slots_do_not_leak():
    wl = workloads.llama3_8b(7, num_seqs=12)
    st = wl.steps[0]
    kp, vp = wl.k_pool.cuda(), wl.v_pool.cuda()
    a = decode(wl, kp, vp, st.block_tables, st.context_lens)
    bs = wl.block_size
    for s, n in enumerate(st.context_lens):
        n = int(n)
        if n % bs:
            b = int(st.block_tables[s, n // bs])
            kp[b, :, n % bs:, :] = float("nan")
            vp[b, :, n % bs:, :] = float("nan")
    b = decode(wl, kp, vp, st.block_tables, st.context_lens)
    assert torch.isfinite(b.float()).all()
    assert torch.equal(a, b)


def test_split_matches_unsplit_within_tolerance():
    wl = workloads.llama3_8b(8, num_seqs=16)
    st = wl.steps[0]
    kp, vp = wl.k_pool.cuda(), wl.v_pool.cuda()
    a = decode(wl, kp, vp, st.block_tables, st.context_lens, partition=16).float()
    b = decode(wl, kp, vp, st.block_tables, st.context_lens, partition=512).float()
    assert (a - b).abs().max().item() <= 1e-2


def test_empty_context_gives_zero_rows():
    wl = workloads.tiny(0)
    st = wl.steps[0]
    kp, vp = wl.k_pool.cuda(), wl.v_pool.cuda()
    ctx = st.context_lens.copy()
    ctx[2] = 0
    out = decode(wl, kp, vp, st.block_tables, ctx)
    assert torch.count_nonzero(out[2]).item() == 0
    assert torch.count_nonzero(out[3]).item() > 0


def test_bad_block_id_is_flagged_not_faulted():
    wl = workloads.tiny(0)
    st = wl.steps[0]
    kp, vp = wl.k_pool.cuda(), wl.v_pool.cuda()
    pa.pa_device_errors(clear=True)
    tab = st.block_tables.copy()
    tab[3, 1] = wl.num_blocks + 5
    decode(wl, kp, vp, tab, st.context_lens)
    assert pa.pa_device_errors(clear=True) & pa.DEVERR_BLOCK_ID
    assert pa.pa_device_errors(clear=True) == 0


def test_context_above_limit_is_clamped_and_flagged():
    wl = workloads.tiny(0)
    st = wl.steps[0]
    kp, vp = wl.k_pool.cuda(), wl.v_pool.cuda()
    q = st.q.cuda()
    out = torch.full_like(q, float("nan"))  # every row must be written
    pa.pa_device_errors(clear=True)
    ctx = torch.as_tensor(st.context_lens).cuda()
    pa.pa_decode(out, q, kp, vp, torch.as_tensor(st.block_tables).cuda(), ctx, wl.scale, 20)
    assert pa.pa_device_errors(clear=True) & pa.DEVERR_CONTEXT


def test_bad_slot_and_pair_are_flagged():
    wl = workloads.tiny(0)
    kp, vp = wl.k_pool.cuda(), wl.v_pool.cuda()
    before = kp.clone()
    pa.pa_device_errors(clear=True)
    k = torch.zeros((1, 2, 64), dtype=torch.float16, device="cuda")
    pa.pa_reshape_and_cache(k, k, kp, vp, torch.tensor([32 * 16], dtype=torch.int64, device="cuda"))
    assert pa.pa_device_errors(clear=True) & pa.DEVERR_SLOT
    pa.pa_copy_blocks([kp, vp], torch.tensor([[0, 32]], dtype=torch.int64, device="cuda"))
    assert pa.pa_device_errors(clear=True) & pa.DEVERR_PAIR
    assert torch.equal(kp, before)


def test_invalid_arguments_return_status():
    wl = workloads.tiny(0)
    st = wl.steps[0]
    kp, vp = wl.k_pool.cuda(), wl.v_pool.cuda()
    q = st.q.cuda()
    out = torch.full_like(q, float("nan"))  # every row must be written
    tab = torch.as_tensor(st.block_tables).cuda()
    ctx = torch.as_tensor(st.context_lens).cuda()
    L = pa.lib()
    ws = pa.alloc_workspace(4, 2, 2, 64, 16, 33)
    args = [out.data_ptr(), q.data_ptr(), kp.data_ptr(), vp.data_ptr(), tab.data_ptr(), ctx.data_ptr(),
            4, 2, 2, 64, 16, tab.shape[1], 32, 33, 0.125, pa.PA_F16, 0, ws.data_ptr(), ws.numel(), None]
    assert L.pa_decode(*args) == pa.PA_OK
    bad = list(args); bad[9] = 96                        # head_dim
    assert L.pa_decode(*bad) == pa.PA_ERR_UNSUPPORTED
    bad = list(args); bad[7] = 3                         # heads not a multiple of kv heads
    assert L.pa_decode(*bad) == pa.PA_ERR_UNSUPPORTED
    bad = list(args); bad[0] = out.data_ptr() + 2        # misaligned
    assert L.pa_decode(*bad) == pa.PA_ERR_INVALID
    bad = list(args); bad[18] = 16                       # workspace too small
    assert L.pa_decode(*bad) == pa.PA_ERR_INVALID
    bad = list(args); bad[16] = 24                       # partition not a multiple of 16
    assert L.pa_decode(*bad) == pa.PA_ERR_INVALID
    bad = list(args); bad[2] = None                      # null pool
    assert L.pa_decode(*bad) == pa.PA_ERR_INVALID
    assert L.pa_reshape_and_cache(None, None, None, None, None, 1, 2, 64, 16, 32, 0, None) == pa.PA_ERR_INVALID
    assert L.pa_copy_blocks(None, 1, None, 1, 100, 32, None) == pa.PA_ERR_INVALID
    torch.cuda.synchronize()
    assert pa.pa_device_errors() == 0


def test_cpu_tensors_are_rejected():
    wl = workloads.tiny(0)
    st = wl.steps[0]
    with pytest.raises(ValueError):
        pa.pa_decode(torch.empty_like(st.q), st.q, wl.k_pool, wl.v_pool,
                     torch.as_tensor(st.block_tables), torch.as_tensor(st.context_lens), wl.scale, 33)


def test_bounded_wait_runs_out_reports_and_leaves_the_context_usable():
    """A device-side wait that nothing completes ends at its limit with
    DEVERR_TIMEOUT instead of hanging; decoding works afterwards."""
    import time
    pa.pa_device_errors(clear=True)
    t0 = time.perf_counter()
    pa.pa_selftest_bounded_wait(20_000_000)          # 20 ms
    flags = pa.pa_device_errors(clear=True)
    elapsed = time.perf_counter() - t0
    assert flags & pa.DEVERR_TIMEOUT
    assert 0.015 < elapsed < 5.0
    wl = workloads.tiny(0)
    st = wl.steps[0]
    out = decode(wl, wl.k_pool.cuda(), wl.v_pool.cuda(), st.block_tables, st.context_lens)
    assert torch.isfinite(out.float()).all() and pa.pa_device_errors() == 0


def test_swap_blocks_round_trip_through_pinned_host_memory():
    """Swap a batch out to a page-locked host pool and back into fresh GPU
    blocks: pools bit-exact against the oracle's copies, and the decode after
    swap-in equals the decode before swap-out bit for bit."""
    import oracle
    from paged_kv_cache_372_b200.block_manager import BlockManager, HostPool, swap_in, swap_out
    from tests.bruteforce import bits_of
    wl = workloads.llama3_8b(9, num_seqs=12)
    st = wl.steps[0]
    nb, bs = wl.num_blocks, wl.block_size
    bm = BlockManager(nb, bs, list(range(nb)))
    used = set(st.block_tables[st.block_tables >= 0].tolist())
    bm.free = [b for b in range(nb) if b not in used][::-1]
    for s_, n in enumerate(st.context_lens):
        k = -(-int(n) // bs)
        bm.tables[s_] = [int(b) for b in st.block_tables[s_, :k]]
        bm.lens[s_] = int(n)
        for b in bm.tables[s_]:
            bm.ref[b] += 1
    bm.check()
    kp, vp = wl.k_pool.cuda(), wl.v_pool.cuda()
    before = decode(wl, kp, vp, st.block_tables, st.context_lens)
    host = HostPool(len(used) + 8)
    hk = torch.empty((host.num_blocks,) + tuple(wl.k_pool.shape[1:]), dtype=wl.k_pool.dtype).pin_memory()
    hv = torch.empty_like(hk).pin_memory()
    okp, ovp = bits_of(wl.k_pool).copy(), bits_of(wl.v_pool).copy()
    ohk, ohv = np.zeros_like(bits_of(hk)), np.zeros_like(bits_of(hv))
    hk.zero_(); hv.zero_()
    seqs = list(range(len(st.context_lens)))
    out_pairs = [pr for s_ in seqs for pr in swap_out(bm, host, s_)]
    pairs = torch.tensor(out_pairs, dtype=torch.int64).cuda()
    pa.pa_swap_blocks([hk, hv], [kp, vp], pairs)
    torch.cuda.synchronize()
    oracle.swap_blocks([ohk, ohv], [okp, ovp], np.array(out_pairs), wl.block_bytes)
    assert np.array_equal(bits_of(hk), ohk) and np.array_equal(bits_of(hv), ohv)
    kp.fill_(float("nan")); vp.fill_(float("nan"))          # the GPU copies are gone
    torch.cuda.synchronize()
    start_k, start_v = bits_of(kp.cpu()).copy(), bits_of(vp.cpu()).copy()
    in_pairs = [pr for s_ in seqs for pr in swap_in(bm, host, s_)]
    pairs_in = torch.tensor(in_pairs, dtype=torch.int64).pin_memory()   # pairs from host memory
    pa.pa_swap_blocks([kp, vp], [hk, hv], pairs_in)
    torch.cuda.synchronize()
    assert pa.pa_device_errors() == 0
    oracle.swap_blocks([start_k, start_v], [ohk, ohv], np.array(in_pairs), wl.block_bytes)
    assert np.array_equal(bits_of(kp.cpu()), start_k) and np.array_equal(bits_of(vp.cpu()), start_v)
    width = max(len(t) for t in bm.tables.values())
    tables = bm.block_table_array(seqs, width)
    after = decode(wl, kp, vp, tables, st.context_lens)
    assert torch.equal(before, after)


def test_swap_blocks_rejects_pageable_host_memory():
    wl = workloads.tiny(0)
    kp = wl.k_pool.cuda()
    pageable = torch.zeros_like(wl.k_pool)                 # not page-locked
    with pytest.raises(ValueError):
        pa.pa_swap_blocks([pageable], [kp], torch.tensor([[0, 1]], dtype=torch.int64).cuda())
    L = pa.lib()
    import ctypes
    dst = (ctypes.c_void_p * 1)(pageable.data_ptr())
    src = (ctypes.c_void_p * 1)(kp.data_ptr())
    pairs = torch.tensor([[0, 1]], dtype=torch.int64).cuda()
    st = L.pa_swap_blocks(dst, src, 1, pairs.data_ptr(), 1, kp[0].numel() * 2, 32, 32, None)
    assert st == pa.PA_ERR_INVALID and b"pageable" in L.pa_last_error()
    torch.cuda.synchronize()
    assert pa.pa_device_errors() == 0
