"""8-bit KV cache with one scale per KV head (E4M3 and INT8 codes) on the GPU
against the oracle: the quantising write bit for bit, decode within the
attention tolerance, and the invariants.

Decode inputs are quantised independently of both the library and the oracle
(E4M3 through torch's float8_e4m3fn cast, INT8 through torch's round-half-even
and clamp), with per-KV-head scales spanning 100x, so that a wrong head index
or a dropped scale shows."""
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
FORMATS = ("e4m3", "int8")


def head_scales(n: int, base: float) -> torch.Tensor:
    """Per-KV-head scales from base / 10 to base * 10 (100x), interleaved so that
    neighbouring heads differ."""
    s = base * 10.0 ** np.linspace(-1.0, 1.0, n)
    order = np.argsort(np.arange(n) % 2 * n + np.arange(n))
    return torch.tensor(s[order], dtype=torch.float32)


def quantise(x: torch.Tensor, scales: torch.Tensor, fmt: str) -> torch.Tensor:
    """Codes of x [..., Hkv, bs, D] (pools) with one scale per KV head (dim 1)."""
    y = x.float() / scales.view(1, -1, 1, 1)
    if fmt == "e4m3":
        return y.clamp(-448, 448).to(torch.float8_e4m3fn).view(torch.uint8)
    return (torch.round(y).clamp(-127, 127).to(torch.int16) + 128).to(torch.uint8)


def quant_pools(wl, fmt):
    ks, vs = head_scales(wl.num_kv_heads, 0.0375), head_scales(wl.num_kv_heads, 0.05).flip(0)
    return quantise(wl.k_pool, ks, fmt), quantise(wl.v_pool, vs, fmt), ks, vs


def run_decode(wl, fmt, k8, v8, ks, vs, partition=None, tables=None):
    st = wl.steps[0]
    q = st.q.cuda()
    out = torch.full_like(q, float("nan"))  # every row must be written
    tab = st.block_tables if tables is None else tables
    pa.pa_decode_quant(out, q, k8.cuda(), v8.cuda(), torch.as_tensor(tab).cuda(),
                       torch.from_numpy(st.context_lens).cuda(), wl.scale, int(st.context_lens.max()), fmt,
                       ks.cuda(), vs.cuda(), wl.partition_size if partition is None else partition)
    torch.cuda.synchronize()
    assert pa.pa_device_errors() == 0
    return out


def oracle_decode(wl, fmt, k8, v8, ks, vs):
    st = wl.steps[0]
    return oracle.paged_attention_kv8(bits_of(st.q), k8.numpy(), v8.numpy(), st.block_tables, st.context_lens,
                                      wl.scale, wl.dtype, fmt, ks.double().numpy(), vs.double().numpy())


@pytest.mark.parametrize("fmt", FORMATS)
@pytest.mark.parametrize("name,kw", [("llama7b", {}), ("llama3_8b", {}), ("llama3_8b", {"num_seqs": 24}),
                                     ("long32k", {"num_seqs": 2, "ctx_len": 5000, "prefill_tokens": 0})])
def test_quant_decode_matches_oracle(fmt, name, kw):
    wl = workloads.build(name, 41, **kw)
    k8, v8, ks, vs = quant_pools(wl, fmt)
    out = run_decode(wl, fmt, k8, v8, ks, vs)
    ref = oracle_decode(wl, fmt, k8, v8, ks, vs)
    err = float(np.abs(out.float().cpu().double().numpy() - ref).max())
    assert err <= TOL[wl.dtype], err
    margins.record(f"{fmt} per-head {name} {wl.dtype} B={wl.num_seqs}", err, TOL[wl.dtype])


@pytest.mark.parametrize("fmt", FORMATS)
@pytest.mark.parametrize("partition", [16, 64, 256])
def test_quant_split_partitions(fmt, partition):
    wl = workloads.llama3_8b(42, num_seqs=10)
    k8, v8, ks, vs = quant_pools(wl, fmt)
    out = run_decode(wl, fmt, k8, v8, ks, vs, partition)
    ref = oracle_decode(wl, fmt, k8, v8, ks, vs)
    assert float(np.abs(out.float().cpu().double().numpy() - ref).max()) <= TOL[wl.dtype]


@pytest.mark.parametrize("fmt", FORMATS)
def test_quant_longest_partitions(fmt):
    """2048-token partitions (32 blocks of 64): the value sums of a whole
    partition stay within the tolerance (INT8 values enter the product as
    exact signed codes, not offset by a constant that the sums would carry)."""
    wl = workloads.long32k(48, num_seqs=2, ctx_len=5000, prefill_tokens=0)
    k8, v8, ks, vs = quant_pools(wl, fmt)
    out = run_decode(wl, fmt, k8, v8, ks, vs, 2048)
    ref = oracle_decode(wl, fmt, k8, v8, ks, vs)
    err = float(np.abs(out.float().cpu().double().numpy() - ref).max())
    assert err <= TOL[wl.dtype], err
    margins.record(f"{fmt} per-head long32k {wl.dtype} P=2048", err, TOL[wl.dtype])


def test_quant_e4m3_with_equal_scales_is_the_fp8_path():
    """Per-head scales all equal to s give pa_decode_fp8's result with k_scale =
    v_scale = s, bit for bit (the same kernel, the scales only moved)."""
    wl = workloads.llama3_8b(43, num_seqs=16)
    s = 0.0375
    k8 = quantise(wl.k_pool, torch.full((wl.num_kv_heads,), s), "e4m3")
    v8 = quantise(wl.v_pool, torch.full((wl.num_kv_heads,), s), "e4m3")
    one = torch.full((wl.num_kv_heads,), s, dtype=torch.float32)
    a = run_decode(wl, "e4m3", k8, v8, one, one)
    st = wl.steps[0]
    b = torch.full_like(a, float("nan"))
    pa.pa_decode_fp8(b, st.q.cuda(), k8.cuda(), v8.cuda(), torch.from_numpy(st.block_tables).cuda(),
                     torch.from_numpy(st.context_lens).cuda(), wl.scale, int(st.context_lens.max()), s, s)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


@pytest.mark.parametrize("fmt", FORMATS)
def test_quant_block_permutation_bit_identical(fmt):
    wl = workloads.llama3_8b(44, num_seqs=16)
    k8, v8, ks, vs = quant_pools(wl, fmt)
    a = run_decode(wl, fmt, k8, v8, ks, vs)
    pi = torch.randperm(wl.num_blocks, generator=torch.Generator().manual_seed(2))
    k2, v2 = torch.empty_like(k8), torch.empty_like(v8)
    k2[pi] = k8
    v2[pi] = v8
    tab = wl.steps[0].block_tables.copy()
    tab[tab >= 0] = pi.numpy()[tab[tab >= 0]]
    assert torch.equal(a, run_decode(wl, fmt, k2, v2, ks, vs, tables=tab))


@pytest.mark.parametrize("fmt", FORMATS)
@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_quant_cache_write_bit_exact(fmt, dtype):
    """pa_reshape_and_cache_quant vs the oracle's quantiser, per-head scales,
    values past the clamp / saturation point, exact ties and a skipped token."""
    from paged_kv_cache_372_b200 import inputs
    gen = inputs.generator(45)
    NB, Hkv, bs, D, T = 40, 4, 16, 128, 300
    k = inputs.normal((T, Hkv, D), dtype, gen) * 3
    v = inputs.normal((T, Hkv, D), dtype, gen) * 40
    ks = head_scales(Hkv, 0.02)
    vs = head_scales(Hkv, 0.25)
    k[5, 1, :8] = (torch.arange(8, dtype=torch.float32) + 0.5) * ks[1]   # ties when exact in fp32
    kp = torch.randint(0, 256, (NB, Hkv, bs, D), dtype=torch.uint8, generator=gen)
    vp = torch.randint(0, 256, (NB, Hkv, bs, D), dtype=torch.uint8, generator=gen)
    slots = torch.randperm(NB * bs, generator=gen)[:T].to(torch.int64)
    slots[7] = -1
    okp, ovp = kp.numpy().copy(), vp.numpy().copy()
    gk, gv = kp.cuda(), vp.cuda()
    pa.pa_reshape_and_cache_quant(k.cuda(), v.cuda(), gk, gv, slots.cuda(), fmt, ks.cuda(), vs.cuda())
    oracle.reshape_and_cache_kv8(bits_of(k), bits_of(v), okp, ovp, slots.numpy(), dtype, fmt, ks.numpy(),
                                 vs.numpy())
    torch.cuda.synchronize()
    assert pa.pa_device_errors() == 0
    assert np.array_equal(gk.cpu().numpy(), okp) and np.array_equal(gv.cpu().numpy(), ovp)


@pytest.mark.parametrize("fmt", FORMATS)
def test_quant_write_then_decode_end_to_end(fmt):
    """Quantise a whole workload's cache with the library's write, decode it, and
    compare with the oracle over the same codes and scales."""
    wl = workloads.llama3_8b(46, num_seqs=12)
    NB, Hkv, bs, D = wl.k_pool.shape
    ks, vs = head_scales(Hkv, 0.0375), head_scales(Hkv, 0.05)
    k8 = torch.zeros((NB, Hkv, bs, D), dtype=torch.uint8, device="cuda")
    v8 = torch.zeros_like(k8)
    rows = wl.k_pool.permute(0, 2, 1, 3).reshape(NB * bs, Hkv, D)
    vrows = wl.v_pool.permute(0, 2, 1, 3).reshape(NB * bs, Hkv, D)
    slots = torch.arange(NB * bs, dtype=torch.int64)
    pa.pa_reshape_and_cache_quant(rows.contiguous().cuda(), vrows.contiguous().cuda(), k8, v8, slots.cuda(), fmt,
                                  ks.cuda(), vs.cuda())
    out = run_decode(wl, fmt, k8, v8, ks, vs)
    ref = oracle_decode(wl, fmt, k8.cpu(), v8.cpu(), ks, vs)
    assert float(np.abs(out.float().cpu().double().numpy() - ref).max()) <= TOL[wl.dtype]


def test_quant_rejects_bad_arguments():
    wl = workloads.llama3_8b(47, num_seqs=2)
    st = wl.steps[0]
    k8 = torch.zeros(tuple(wl.k_pool.shape), dtype=torch.uint8, device="cuda")
    ks = torch.ones(wl.num_kv_heads, dtype=torch.float32, device="cuda")
    args = (torch.empty_like(st.q).cuda(), st.q.cuda(), k8, k8, torch.from_numpy(st.block_tables).cuda(),
            torch.from_numpy(st.context_lens).cuda(), wl.scale, int(st.context_lens.max()))
    with pytest.raises(ValueError):
        pa.pa_decode_quant(*args, "int8", ks[:3], ks)            # wrong number of scales
    L = pa.lib()
    assert L.pa_decode_quant(*([None] * 6), 1, 32, 8, 128, 16, 4, 8, 16, 0.1, 0, 7, None, None, 0, None, 0,
                             None) == pa.PA_ERR_INVALID          # unknown format
    assert L.pa_decode_quant(*([None] * 6), 1, 32, 8, 128, 16, 4, 8, 16, 0.1, 0, 1, None, None, 0, None, 0,
                             None) == pa.PA_ERR_INVALID          # null scale arrays


@pytest.mark.parametrize("fmt", FORMATS)
@pytest.mark.parametrize("group", [1, 2, 4, 8])
@pytest.mark.parametrize("dtype", ["f16", "bf16"])
@pytest.mark.parametrize("head_dim", [128, 64])
def test_quant_every_head_group(fmt, group, dtype, head_dim):
    """Every query-head group size over both 8-bit formats and both head sizes,
    ragged contexts (1 token to several partitions, partial last tiles), both
    query types."""
    ctx = [1, 15, 16, 17, 100, 333, 700, 1500]
    wl, _ = workloads._decode_batch("groups", ctx, heads=2 * group, kv_heads=2, head_dim=head_dim, block_size=16,
                                    dtype=dtype, seed=4900 + group + head_dim)
    k8, v8, ks, vs = quant_pools(wl, fmt)
    for partition in (0, 64):
        out = run_decode(wl, fmt, k8, v8, ks, vs, partition)
        ref = oracle_decode(wl, fmt, k8, v8, ks, vs)
        err = float(np.abs(out.float().cpu().double().numpy() - ref).max())
        assert err <= TOL[dtype], (partition, err)
        margins.record(f"{fmt} per-head G={group} D={head_dim} {dtype} P={partition or 'auto'}", err, TOL[dtype])


@pytest.mark.parametrize("fmt", FORMATS)
def test_quant_merge_launch_beside_in_kernel_merges(fmt):
    """8-bit cache: one sequence past 16 partitions (merge launch) next to
    sequences merged in the attention kernel or written directly."""
    P = 64
    ctx = [40 * P + 5, 1, P, 2 * P - 3, 8 * P, 9 * P - 1, 16 * P, 17 * P, 3]
    wl, _ = workloads._decode_batch("mixed_merges", ctx, heads=8, kv_heads=2, head_dim=128, block_size=16,
                                    dtype="bf16", seed=78)
    k8, v8, ks, vs = quant_pools(wl, fmt)
    out = run_decode(wl, fmt, k8, v8, ks, vs, P)
    ref = oracle_decode(wl, fmt, k8, v8, ks, vs)
    assert not torch.isnan(out).any()
    err = float(np.abs(out.float().cpu().double().numpy() - ref).max())
    assert err <= TOL[wl.dtype], err
