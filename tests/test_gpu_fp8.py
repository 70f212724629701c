"""E4M3 (fp8) KV cache on the GPU against the oracle: the quantising cache
write bit for bit, decode within the attention tolerance, and the invariants.

Decode inputs are cast to E4M3 with torch's own float8_e4m3fn conversion
(neither the library's quantiser nor the oracle's), so the decode parity does
not lean on the write path."""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_372_b200 as pa
from paged_kv_cache_372_b200 import workloads
from tests import margins
from tests.bruteforce import bits_of

pytestmark = pytest.mark.gpu

TOL = {"f16": 2e-3, "bf16": 1e-2}
K_SCALE, V_SCALE = 0.0375, 0.05


def codes(x: torch.Tensor, scale: float) -> torch.Tensor:
    """E4M3 codes of x / scale through torch's cast (values stay well inside +-448)."""
    return (x.float() / scale).to(torch.float8_e4m3fn).view(torch.uint8)


def fp8_pools(wl):
    return codes(wl.k_pool, K_SCALE), codes(wl.v_pool, V_SCALE)


def run_decode(wl, k8, v8, partition=None, tables=None):
    st = wl.steps[0]
    q = st.q.cuda()
    out = torch.full_like(q, float("nan"))  # every row must be written
    tab = st.block_tables if tables is None else tables
    pa.pa_decode_fp8(out, q, k8.cuda(), v8.cuda(), torch.as_tensor(tab).cuda(),
                     torch.from_numpy(st.context_lens).cuda(), wl.scale, int(st.context_lens.max()),
                     K_SCALE, V_SCALE, wl.partition_size if partition is None else partition)
    torch.cuda.synchronize()
    assert pa.pa_device_errors() == 0
    return out


def oracle_decode(wl, k8, v8, tables=None):
    st = wl.steps[0]
    return oracle.paged_attention_fp8(bits_of(st.q), k8.numpy(), v8.numpy(),
                                      st.block_tables if tables is None else tables, st.context_lens, wl.scale,
                                      wl.dtype, K_SCALE, V_SCALE)


@pytest.mark.parametrize("name,kw", [("llama7b", {"num_seqs": 8}), ("llama3_8b", {"num_seqs": 24}),
                                     ("llama3_8b", {}), ("long32k", {"num_seqs": 2, "ctx_len": 5000,
                                                                     "prefill_tokens": 0})])
def test_fp8_decode_matches_oracle(name, kw):
    wl = workloads.build(name, 31, **kw)
    k8, v8 = fp8_pools(wl)
    out = run_decode(wl, k8, v8)
    ref = oracle_decode(wl, k8, v8)
    err = float(np.abs(out.float().cpu().double().numpy() - ref).max())
    assert err <= TOL[wl.dtype], err
    margins.record(f"fp8 {name} {wl.dtype} B={wl.num_seqs}", err, TOL[wl.dtype])


@pytest.mark.parametrize("partition", [16, 64, 256])
def test_fp8_split_partitions(partition):
    wl = workloads.llama3_8b(32, num_seqs=10)
    k8, v8 = fp8_pools(wl)
    out = run_decode(wl, k8, v8, partition)
    ref = oracle_decode(wl, k8, v8)
    assert float(np.abs(out.float().cpu().double().numpy() - ref).max()) <= TOL[wl.dtype]


def test_fp8_block_permutation_bit_identical():
    wl = workloads.llama3_8b(33, num_seqs=16)
    k8, v8 = fp8_pools(wl)
    a = run_decode(wl, k8, v8)
    pi = torch.randperm(wl.num_blocks, generator=torch.Generator().manual_seed(1))
    k2, v2 = torch.empty_like(k8), torch.empty_like(v8)
    k2[pi] = k8
    v2[pi] = v8
    tab = wl.steps[0].block_tables.copy()
    tab[tab >= 0] = pi.numpy()[tab[tab >= 0]]
    b = run_decode(wl, k2, v2, tables=tab)
    assert torch.equal(a, b)


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_fp8_cache_write_bit_exact(dtype):
    """pa_reshape_and_cache_fp8 vs the oracle's quantiser, including values past
    the saturation point and exact ties."""
    from paged_kv_cache_372_b200 import inputs
    gen = inputs.generator(34)
    NB, Hkv, bs, D, T = 40, 4, 16, 128, 300
    k = inputs.normal((T, Hkv, D), dtype, gen) * 3
    v = inputs.normal((T, Hkv, D), dtype, gen) * 40        # many values saturate at 448 * v_scale
    kp = torch.randint(0, 256, (NB, Hkv, bs, D), dtype=torch.uint8, generator=gen)
    vp = torch.randint(0, 256, (NB, Hkv, bs, D), dtype=torch.uint8, generator=gen)
    slots = torch.randperm(NB * bs, generator=gen)[:T].to(torch.int64)
    slots[7] = -1
    okp, ovp = kp.numpy().copy(), vp.numpy().copy()
    gk, gv = kp.cuda(), vp.cuda()
    pa.pa_reshape_and_cache_fp8(k.cuda(), v.cuda(), gk, gv, slots.cuda(), K_SCALE, V_SCALE)
    oracle.reshape_and_cache_fp8(bits_of(k), bits_of(v), okp, ovp, slots.numpy(), dtype, K_SCALE, V_SCALE)
    torch.cuda.synchronize()
    assert pa.pa_device_errors() == 0
    assert np.array_equal(gk.cpu().numpy(), okp) and np.array_equal(gv.cpu().numpy(), ovp)


def test_fp8_write_then_decode_end_to_end():
    """Quantise a whole workload's cache with the library's write, decode it, and
    compare with the oracle over the same codes."""
    wl = workloads.llama3_8b(35, num_seqs=12)
    st = wl.steps[0]
    NB, Hkv, bs, D = wl.k_pool.shape
    k8 = torch.zeros((NB, Hkv, bs, D), dtype=torch.uint8, device="cuda")
    v8 = torch.zeros_like(k8)
    rows = wl.k_pool.permute(0, 2, 1, 3).reshape(NB * bs, Hkv, D)      # token rows in slot order
    vrows = wl.v_pool.permute(0, 2, 1, 3).reshape(NB * bs, Hkv, D)
    slots = torch.arange(NB * bs, dtype=torch.int64)
    pa.pa_reshape_and_cache_fp8(rows.contiguous().cuda(), vrows.contiguous().cuda(), k8, v8, slots.cuda(),
                                K_SCALE, V_SCALE)
    out = run_decode(wl, k8, v8)
    ref = oracle_decode(wl, k8.cpu(), v8.cpu())
    assert float(np.abs(out.float().cpu().double().numpy() - ref).max()) <= TOL[wl.dtype]


@pytest.mark.parametrize("name,kw", [("tiny", {}), ("llama7b", {"num_seqs": 8, "head_dim": 64}),
                                     ("llama3_8b", {"num_seqs": 24, "head_dim": 64})])
def test_fp8_head_dim_64(name, kw):
    """head_dim 64: 64-byte tile rows (one 64-byte TMA box with the 64-byte
    swizzle) against the oracle, one partition and split."""
    wl = workloads.build(name, 37, **kw)
    k8, v8 = fp8_pools(wl)
    ref = oracle_decode(wl, k8, v8)
    for partition in (None, 64):
        out = run_decode(wl, k8, v8, partition)
        err = float(np.abs(out.float().cpu().double().numpy() - ref).max())
        assert err <= TOL[wl.dtype], (partition, err)
        margins.record(f"fp8 D=64 {name} {wl.dtype} P={partition or 'auto'}", err, TOL[wl.dtype])


def test_fp8_flags_bf16_queries_outside_f16_range():
    """The fp8 kernel multiplies in f16: a bf16 query element above 65504 in
    magnitude has no f16 value, so the kernel flags it (DEVERR_QRANGE) instead
    of returning NaN silently. In-range queries raise nothing."""
    wl = workloads.llama3_8b(36, num_seqs=4)
    k8, v8 = fp8_pools(wl)
    st = wl.steps[0]
    q = st.q.clone()
    q[2, 5, 17] = 1.0e5                           # representable in bf16, not in f16
    out = torch.full_like(q, float("nan")).cuda()
    pa.pa_decode_fp8(out, q.cuda(), k8.cuda(), v8.cuda(), torch.from_numpy(st.block_tables).cuda(),
                     torch.from_numpy(st.context_lens).cuda(), wl.scale, int(st.context_lens.max()),
                     K_SCALE, V_SCALE)
    assert pa.pa_device_errors(clear=True) == pa.DEVERR_QRANGE
    run_decode(wl, k8, v8)                         # the unmodified queries flag nothing
