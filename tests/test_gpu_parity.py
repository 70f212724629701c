"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle.

Cache writes and block copies must be bit-exact (the whole pool is compared,
which also catches stray writes); attention must be within max-abs 2e-3
(fp16) / 1e-2 (bf16) of the oracle.
"""
import numpy as np
import pytest
import torch

import paged_kv_cache_372_b200 as pa
from paged_kv_cache_372_b200 import workloads
from tests import gpu_harness as H
from tests import margins

pytestmark = pytest.mark.gpu


def run_and_compare(wl, partition_size=None, steps=None, label=None):
    kp, vp = H.to_gpu(wl)
    okp, ovp = H.oracle_state(wl)
    errs = []
    for i in range(len(wl.steps) if steps is None else steps):
        out = H.gpu_step(wl, i, kp, vp, partition_size)
        ref = H.oracle_step(wl, i, okp, ovp)
        torch.cuda.synchronize()
        assert pa.pa_device_errors() == 0
        assert H.pools_equal(kp, vp, okp, ovp), f"pools differ after step {i}"
        err = H.max_err(out, ref)
        errs.append(err)
        assert err <= H.TOL[wl.dtype], (wl.name, i, err)
    P = wl.partition_size if partition_size is None else partition_size
    margins.record(label or f"{wl.name} {wl.dtype} B={wl.num_seqs} P={P or 'auto'}", max(errs), H.TOL[wl.dtype])
    return errs


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_tiny(seed):
    run_and_compare(workloads.tiny(seed))


@pytest.mark.parametrize("seed", [1, 2])
def test_llama7b_small(seed):
    run_and_compare(workloads.llama7b(seed, num_seqs=6))


@pytest.mark.parametrize("seed", [1, 2])
def test_llama3_8b_small(seed):
    run_and_compare(workloads.llama3_8b(seed, num_seqs=12))


def test_llama7b_full():
    run_and_compare(workloads.llama7b(0))


def test_llama3_8b_full():
    run_and_compare(workloads.llama3_8b(0))


def test_beam_all_steps():
    run_and_compare(workloads.beam(0))


def test_beam256_steps():
    run_and_compare(workloads.beam256(0, steps=3))


def test_long32k_full():
    run_and_compare(workloads.long32k(0))


@pytest.mark.parametrize("num_seqs", [512, 513, 700])
def test_batch_sizes_around_the_early_start_limit(num_seqs):
    """Up to 512 sequences the attention kernel starts before the plan kernel
    has finished (each warp derives its first unit from the contexts); above
    it, it waits for the plan first. Both agree with the oracle."""
    from paged_kv_cache_372_b200 import inputs
    gen = inputs.generator(9000 + num_seqs)
    ctx = inputs.uniform_int(1, 700, num_seqs, gen)
    wl, _ = workloads._decode_batch("batch", ctx, heads=16, kv_heads=4, head_dim=128, block_size=16,
                                    dtype="bf16", seed=9100 + num_seqs)
    run_and_compare(wl, partition_size=128, label=f"batch B={num_seqs} bf16 P=128")


@pytest.mark.parametrize("partition", [16, 32, 128, 256])
def test_split_partitions(partition):
    wl = workloads.llama3_8b(3, num_seqs=10)
    run_and_compare(wl, partition_size=partition)


@pytest.mark.parametrize("shape", [(64, 1), (64, 2), (64, 4), (64, 8), (128, 1), (128, 2), (128, 4), (128, 8)])
@pytest.mark.parametrize("block_size", [16, 32, 64])
def test_shapes(shape, block_size):
    """Every supported (head_dim, group, block_size), ragged contexts, both dtypes."""
    D, G = shape
    from paged_kv_cache_372_b200 import inputs
    from paged_kv_cache_372_b200.block_manager import BlockManager
    import math
    for dtype in ("f16", "bf16"):
        gen = inputs.generator(D * 100 + G * 10 + block_size)
        ctx = [1, 15, 16, 17, 100, 333, 700]
        hkv = 2
        need = sum(-(-c // block_size) for c in ctx)
        nb = need + 5
        bm = BlockManager(nb, block_size, inputs.permutation(nb, gen))
        for s, c in enumerate(ctx):
            bm.allocate(s, c)
        width = max(len(t) for t in bm.tables.values())
        st = workloads.Step(
            q=inputs.normal((len(ctx), hkv * G, D), dtype, gen),
            block_tables=bm.block_table_array(range(len(ctx)), width),
            context_lens=bm.context_lens(range(len(ctx))),
            k_new=inputs.normal((0, hkv, D), dtype, gen), v_new=inputs.normal((0, hkv, D), dtype, gen),
            slot_mapping=np.zeros(0, np.int64), copy_pairs=np.zeros((0, 2), np.int64))
        wl = workloads.Workload("shape", dtype, hkv * G, hkv, D, block_size, nb, 0,
                                inputs.normal((nb, hkv, block_size, D), dtype, gen),
                                inputs.normal((nb, hkv, block_size, D), dtype, gen), [st])
        for P in (0, block_size * max(1, 64 // block_size)):
            run_and_compare(wl, partition_size=P, label=f"shapes D={D} G={G} bs={block_size} {dtype} P={P or 'auto'}")


@pytest.mark.parametrize("name,kw", [("tiny", {}), ("llama7b", {"num_seqs": 8}), ("llama3_8b", {"num_seqs": 16}),
                                     ("beam", {"groups": 2, "steps": 4}),
                                     ("long32k", {"num_seqs": 2, "ctx_len": 3000, "prefill_tokens": 64})])
def test_fused_append_matches_oracle_and_unfused_path(name, kw):
    """pa_decode_append = cache write of the last positions + pa_decode: same
    pools bit for bit, same outputs bit for bit, oracle within tolerance."""
    wl = workloads.build(name, 21, **kw)
    kf, vf = H.to_gpu(wl)                 # fused path state
    ku, vu = H.to_gpu(wl)                 # unfused path state
    okp, ovp = H.oracle_state(wl)
    for i in range(len(wl.steps)):
        fused = H.gpu_step_fused(wl, i, kf, vf)
        unfused = H.gpu_step(wl, i, ku, vu)
        ref = H.oracle_step(wl, i, okp, ovp)
        torch.cuda.synchronize()
        assert pa.pa_device_errors() == 0
        assert torch.equal(kf, ku) and torch.equal(vf, vu), f"pools differ at step {i}"
        assert H.pools_equal(kf, vf, okp, ovp)
        assert torch.equal(fused, unfused), f"outputs differ at step {i}"
        err = H.max_err(fused, ref)
        assert err <= H.TOL[wl.dtype]
        margins.record(f"fused append {name} {wl.dtype}", err, H.TOL[wl.dtype])


@pytest.mark.parametrize("partition,launches", [(512, 2), (128, 3)])
def test_launch_count(partition, launches):
    """A decode call is the plan and the attention launch; with more than 16
    partitions a sequence's merge runs in a third launch. The library's
    counter (the bench's gpu_launches) sees exactly these."""
    wl = workloads.long32k(3, num_seqs=2, ctx_len=4096, prefill_tokens=0)
    st = wl.steps[0]
    dev = torch.device("cuda")
    q = st.q.to(dev)
    out = torch.full_like(q, float("nan"))  # every row must be written
    kp, vp = wl.k_pool.to(dev), wl.v_pool.to(dev)
    tab, ctx = torch.from_numpy(st.block_tables).to(dev), torch.from_numpy(st.context_lens).to(dev)
    ws = pa.alloc_workspace(wl.num_seqs, wl.num_heads, wl.num_kv_heads, wl.head_dim, wl.block_size, 4096,
                            partition, dev)
    n0 = pa.pa_launch_count()
    pa.pa_decode(out, q, kp, vp, tab, ctx, wl.scale, 4096, partition, ws)
    assert pa.pa_launch_count() - n0 == launches
    torch.cuda.synchronize()
    assert pa.pa_device_errors() == 0


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_merge_launch_beside_in_kernel_merges(dtype):
    """One sequence with more than 16 partitions (merged in the merge launch)
    next to sequences of 1, 2, 8, 9 and 16 partitions (written directly, merged
    in one level and in two levels inside the attention kernel) in one call."""
    P = 64
    ctx = [40 * P + 5, 1, P, 2 * P - 3, 8 * P, 9 * P - 1, 16 * P, 17 * P, 3]
    wl, _ = workloads._decode_batch("mixed_merges", ctx, heads=8, kv_heads=2, head_dim=128, block_size=16,
                                    dtype=dtype, seed=77)
    n0 = pa.pa_launch_count()
    run_and_compare(wl, partition_size=P)
    assert pa.pa_launch_count() - n0 == 4  # cache write, plan, attention, merge launch
