"""8-bit KV cache with one scale per (physical block, KV head) on the GPU:
pa_reshape_and_cache_quant_blocks bit for bit against the oracle's quantiser,
pa_decode_quant_blocks within the attention tolerance of the oracle's
attention over the cache dequantised block by block.

Decode inputs are quantised independently of both the library and the oracle
(E4M3 through torch's float8_e4m3fn cast, INT8 through torch's round-half-even
and clamp), with scales spanning 100x across blocks and heads, so that a wrong
block index, a head's scale in place of the block's, or a dropped scale shows."""
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


def block_scales(nb: int, hkv: int, base: float, seed: int) -> torch.Tensor:
    """[nb][hkv] scales from base / 10 to base * 10 (100x), drawn per block and head."""
    g = torch.Generator().manual_seed(seed)
    return (base * 10.0 ** (2.0 * torch.rand((nb, hkv), generator=g, dtype=torch.float64) - 1.0)).float()


def quantise_blocks(x: torch.Tensor, scales: torch.Tensor, fmt: str) -> torch.Tensor:
    """Codes of pools x [NB][Hkv][bs][D] with one scale per (block, KV head)."""
    y = x.float() / scales[:, :, None, None]
    if fmt == "e4m3":
        return y.clamp(-448, 448).to(torch.float8_e4m3fn).view(torch.uint8)
    return (torch.round(y).clamp(-127, 127).to(torch.int16) + 128).to(torch.uint8)


def quant_pools(wl, fmt, seed=0):
    NB, Hkv = wl.k_pool.shape[0], wl.num_kv_heads
    base = 0.01 if fmt == "int8" else 0.0375
    ks, vs = block_scales(NB, Hkv, base, seed), block_scales(NB, Hkv, base, seed + 1)
    return quantise_blocks(wl.k_pool, ks, fmt), quantise_blocks(wl.v_pool, vs, fmt), ks, vs


def run_decode(wl, fmt, k8, v8, ks, vs, partition=None):
    st = wl.steps[0]
    q = st.q.cuda()
    out = torch.full_like(q, float("nan"))
    pa.pa_decode_quant_blocks(out, q, k8.cuda(), v8.cuda(), torch.from_numpy(st.block_tables).cuda(),
                              torch.from_numpy(st.context_lens).cuda(), wl.scale, int(st.context_lens.max()), fmt,
                              ks.cuda(), vs.cuda(), wl.partition_size if partition is None else partition)
    torch.cuda.synchronize()
    assert pa.pa_device_errors() == 0
    assert not torch.isnan(out).any()
    return out


def oracle_decode(wl, fmt, k8, v8, ks, vs):
    st = wl.steps[0]
    return oracle.paged_attention_kv8(bits_of(st.q), k8.numpy(), v8.numpy(), st.block_tables, st.context_lens,
                                      wl.scale, wl.dtype, fmt, ks.double().numpy(), vs.double().numpy())


def max_err(out, ref):
    return float(np.abs(out.float().cpu().double().numpy() - ref).max())


@pytest.mark.parametrize("fmt", FORMATS)
@pytest.mark.parametrize("name,kw", [("llama7b", {"num_seqs": 16}), ("llama3_8b", {"num_seqs": 48}),
                                     ("long32k", {"num_seqs": 2, "ctx_len": 5000, "prefill_tokens": 0})])
def test_block_scaled_decode_matches_oracle(fmt, name, kw):
    wl = workloads.build(name, 51, **kw)
    k8, v8, ks, vs = quant_pools(wl, fmt, 3)
    out = run_decode(wl, fmt, k8, v8, ks, vs)
    err = max_err(out, oracle_decode(wl, fmt, k8, v8, ks, vs))
    assert err <= TOL[wl.dtype], err
    margins.record(f"{fmt} per-block {name} {wl.dtype} B={wl.num_seqs}", err, TOL[wl.dtype])


@pytest.mark.parametrize("fmt", FORMATS)
@pytest.mark.parametrize("partition", [16, 64, 256])
def test_block_scaled_split_partitions(fmt, partition):
    wl = workloads.llama3_8b(52, num_seqs=10)
    k8, v8, ks, vs = quant_pools(wl, fmt, 5)
    out = run_decode(wl, fmt, k8, v8, ks, vs, partition)
    assert max_err(out, oracle_decode(wl, fmt, k8, v8, ks, vs)) <= TOL[wl.dtype]


@pytest.mark.parametrize("fmt", FORMATS)
@pytest.mark.parametrize("group", [1, 2, 4, 8])
@pytest.mark.parametrize("head_dim", [128, 64])
@pytest.mark.parametrize("block_size", [16, 64])
def test_block_scaled_every_head_group(fmt, group, head_dim, block_size):
    """Every group size, both head sizes, two block sizes (a 32-token item
    spans two blocks at 16, lies in one at 64), ragged contexts."""
    ctx = [1, 15, 16, 17, 100, 333, 700, 1500]
    wl, _ = workloads._decode_batch("groups", ctx, heads=2 * group, kv_heads=2, head_dim=head_dim,
                                    block_size=block_size, dtype="bf16", seed=5100 + group + head_dim + block_size)
    k8, v8, ks, vs = quant_pools(wl, fmt, 7)
    for partition in (0, 4 * block_size):
        out = run_decode(wl, fmt, k8, v8, ks, vs, partition)
        err = max_err(out, oracle_decode(wl, fmt, k8, v8, ks, vs))
        assert err <= TOL["bf16"], (partition, err)
        margins.record(f"{fmt} per-block G={group} D={head_dim} bs={block_size} P={partition or 'auto'}", err,
                       TOL["bf16"])


@pytest.mark.parametrize("fmt", FORMATS)
def test_block_scales_equal_per_head_match_the_per_head_path(fmt):
    """Every block of a head carrying the head's scale: the same attention as
    pa_decode_quant with per-head scales (up to the order of the fp32 sums)."""
    wl = workloads.llama3_8b(53, num_seqs=16)
    NB, Hkv = wl.k_pool.shape[0], wl.num_kv_heads
    kh = torch.linspace(0.01, 0.1, Hkv)
    vh = torch.linspace(0.2, 0.02, Hkv)
    kb, vb = kh[None, :].expand(NB, Hkv).contiguous(), vh[None, :].expand(NB, Hkv).contiguous()
    k8, v8 = quantise_blocks(wl.k_pool, kb, fmt), quantise_blocks(wl.v_pool, vb, fmt)
    a = run_decode(wl, fmt, k8, v8, kb, vb)
    st = wl.steps[0]
    b = torch.full_like(a, float("nan"))
    pa.pa_decode_quant(b, st.q.cuda(), k8.cuda(), v8.cuda(), torch.from_numpy(st.block_tables).cuda(),
                       torch.from_numpy(st.context_lens).cuda(), wl.scale, int(st.context_lens.max()), fmt,
                       kh.cuda(), vh.cuda())
    torch.cuda.synchronize()
    assert float((a.float() - b.float()).abs().max()) <= TOL[wl.dtype]


@pytest.mark.parametrize("fmt", FORMATS)
@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_block_scaled_cache_write_bit_exact(fmt, dtype):
    """pa_reshape_and_cache_quant_blocks against the oracle's quantiser, scales
    per (block, head), values past the clamp, a skipped token."""
    from paged_kv_cache_372_b200 import inputs
    gen = inputs.generator(54)
    NB, Hkv, bs, D, T = 40, 4, 16, 128, 300
    k = inputs.normal((T, Hkv, D), dtype, gen) * 3
    v = inputs.normal((T, Hkv, D), dtype, gen) * 40
    ks, vs = block_scales(NB, Hkv, 0.02, 11), block_scales(NB, Hkv, 0.25, 12)
    kp = torch.randint(0, 256, (NB, Hkv, bs, D), dtype=torch.uint8, generator=gen)
    vp = torch.randint(0, 256, (NB, Hkv, bs, D), dtype=torch.uint8, generator=gen)
    slots = torch.randperm(NB * bs, generator=gen)[:T].to(torch.int64)
    slots[9] = -1
    okp, ovp = kp.numpy().copy(), vp.numpy().copy()
    gk, gv = kp.cuda(), vp.cuda()
    pa.pa_reshape_and_cache_quant_blocks(k.cuda(), v.cuda(), gk, gv, slots.cuda(), fmt, ks.cuda(), vs.cuda())
    oracle.reshape_and_cache_kv8(bits_of(k), bits_of(v), okp, ovp, slots.numpy(), dtype, fmt, ks.numpy(),
                                 vs.numpy())
    torch.cuda.synchronize()
    assert pa.pa_device_errors() == 0
    assert np.array_equal(gk.cpu().numpy(), okp) and np.array_equal(gv.cpu().numpy(), ovp)


@pytest.mark.parametrize("fmt", FORMATS)
def test_block_scaled_write_then_decode_end_to_end(fmt):
    """The library's block-scaled write of a whole workload's cache, then its
    decode, against the oracle over the same codes and scales."""
    wl = workloads.llama3_8b(55, num_seqs=12)
    NB, Hkv, bs, D = wl.k_pool.shape
    ks, vs = block_scales(NB, Hkv, 0.0375, 13), block_scales(NB, Hkv, 0.05, 14)
    k8 = torch.zeros((NB, Hkv, bs, D), dtype=torch.uint8, device="cuda")
    v8 = torch.zeros_like(k8)
    rows = wl.k_pool.permute(0, 2, 1, 3).reshape(NB * bs, Hkv, D)
    vrows = wl.v_pool.permute(0, 2, 1, 3).reshape(NB * bs, Hkv, D)
    slots = torch.arange(NB * bs, dtype=torch.int64)
    pa.pa_reshape_and_cache_quant_blocks(rows.contiguous().cuda(), vrows.contiguous().cuda(), k8, v8, slots.cuda(),
                                         fmt, ks.cuda(), vs.cuda())
    out = run_decode(wl, fmt, k8, v8, ks, vs)
    ref = oracle_decode(wl, fmt, k8.cpu(), v8.cpu(), ks, vs)
    assert max_err(out, ref) <= TOL[wl.dtype]


def test_block_scaled_rejects():
    wl = workloads.llama3_8b(56, num_seqs=2)
    st = wl.steps[0]
    NB, Hkv = wl.k_pool.shape[0], wl.num_kv_heads
    k8 = torch.zeros(tuple(wl.k_pool.shape), dtype=torch.uint8, device="cuda")
    s = torch.ones((NB, Hkv), dtype=torch.float32, device="cuda")
    args = (torch.empty_like(st.q).cuda(), st.q.cuda(), k8, k8, torch.from_numpy(st.block_tables).cuda(),
            torch.from_numpy(st.context_lens).cuda(), wl.scale, int(st.context_lens.max()))
    with pytest.raises(ValueError):
        pa.pa_decode_quant_blocks(*args, "int8", s[:, 0].contiguous(), s)  # per-head shape
    L = pa.lib()
    assert L.pa_decode_quant_blocks(*([None] * 6), 1, 32, 8, 128, 16, 4, 8, 16, 0.1, 0, 1, None, None, 0, None, 0,
                                    None) == pa.PA_ERR_INVALID   # null scale arrays
