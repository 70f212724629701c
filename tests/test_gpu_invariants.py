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
    out = torch.empty_like(q)
    pa.pa_decode(out, q, kp, vp, torch.as_tensor(tables).cuda(), torch.as_tensor(ctx).cuda(),
                 wl.scale, int(np.max(ctx)), partition)
    torch.cuda.synchronize()
    return out


def test_block_permutation_bit_identical():
    """Physical placement of blocks does not change the result."""
    wl = workloads.llama3_8b(4, num_seqs=16)
    st = wl.steps[0]
    kp, vp = wl.k_pool.cuda(), wl.v_pool.cuda()
    a = decode(wl, kp, vp, st.block_tables, st.context_lens)
    pi = torch.randperm(wl.num_blocks, generator=torch.Generator().manual_seed(0))
    kp2 = torch.empty_like(kp)
    vp2 = torch.empty_like(vp)
    kp2[pi.cuda()] = kp
    vp2[pi.cuda()] = vp
    tab = st.block_tables.copy()
    tab[tab >= 0] = pi.numpy()[tab[tab >= 0]]
    b = decode(wl, kp2, vp2, tab, st.context_lens)
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
    out = torch.empty_like(q)
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
    out = torch.empty_like(q)
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
