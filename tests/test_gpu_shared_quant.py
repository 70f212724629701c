"""pa_decode_shared_quant: shared-prefix decode over an 8-bit cache (E4M3 or
INT8 codes, one scale per KV head) on the GPU.

The result must be the oracle's attention over the dequantised cache (fp64)
within the dtype's tolerance, agree within tolerance with pa_decode_quant on
the same inputs, group the sequences as pa_decode_shared does (the unit count
of the work list is checked against a direct count from the block tables),
ignore whatever the slots no sequence covers hold, and be deterministic.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_372_b200 as pa
from paged_kv_cache_372_b200 import workloads
from tests import gpu_harness as H
from tests import margins
from tests.bruteforce import bits_of
from tests.test_gpu_quant import head_scales, quantise
from tests.test_gpu_shared import expected_entries, sharing_case, whole_unit_case

pytestmark = pytest.mark.gpu

FORMATS = ("e4m3", "int8")


def quant_case(case, fmt, seed):
    """Codes of the case's pools with per-KV-head scales spanning 100x; the
    slots no sequence covers get E4M3 NaN codes (0x7f) or random bytes."""
    kp, vp = case["kp"], case["vp"]
    bad = torch.isnan(kp)
    Hkv = kp.shape[1]
    ks, vs = head_scales(Hkv, 0.0375), head_scales(Hkv, 0.05).flip(0)
    k8 = quantise(torch.nan_to_num(kp), ks, fmt)
    v8 = quantise(torch.nan_to_num(vp), vs, fmt)
    if fmt == "e4m3":
        k8[bad] = 0x7F
        v8[bad] = 0x7F
    else:
        g = torch.Generator().manual_seed(seed)
        k8[bad] = torch.randint(0, 256, (int(bad.sum()),), generator=g, dtype=torch.uint8)
        v8[bad] = torch.randint(0, 256, (int(bad.sum()),), generator=g, dtype=torch.uint8)
    return k8, v8, ks, vs


def run_shared_quant(case, fmt, k8, v8, ks, vs, P):
    dev = torch.device("cuda")
    q = case["q"].to(dev)
    out = torch.full_like(q, float("nan"))  # every row must be written
    B, H_, D = q.shape
    mx = int(case["ctx"].max())
    ws = pa.alloc_workspace(B, H_, case["kv_heads"], D, case["bs"], mx, P, dev, shared=True)
    pa.pa_decode_shared_quant(out, q, k8.to(dev), v8.to(dev), torch.from_numpy(case["tables"]).to(dev),
                              torch.from_numpy(case["ctx"]).to(dev), case["scale"], mx, fmt, ks.to(dev),
                              vs.to(dev), P, ws)
    torch.cuda.synchronize()
    assert pa.pa_device_errors() == 0
    return out, ws


def run_plain_quant(case, fmt, k8, v8, ks, vs, P):
    dev = torch.device("cuda")
    q = case["q"].to(dev)
    out = torch.full_like(q, float("nan"))  # every row must be written
    mx = int(case["ctx"].max())
    pa.pa_decode_quant(out, q, k8.to(dev), v8.to(dev), torch.from_numpy(case["tables"]).to(dev),
                       torch.from_numpy(case["ctx"]).to(dev), case["scale"], mx, fmt, ks.to(dev), vs.to(dev), P)
    torch.cuda.synchronize()
    assert pa.pa_device_errors() == 0
    return out


def oracle_quant(case, fmt, k8, v8, ks, vs):
    return oracle.paged_attention_kv8(bits_of(case["q"]), k8.numpy(), v8.numpy(), case["tables"], case["ctx"],
                                      case["scale"], case["dtype"], fmt, ks.double().numpy(), vs.double().numpy())


SHAPES = [  # (heads, kv_heads, head_dim, block_size, dtype): every head group, both head sizes
    (8, 8, 128, 16, "f16"),
    (8, 4, 64, 32, "bf16"),
    (16, 4, 128, 16, "bf16"),
    (16, 2, 128, 64, "f16"),
    (4, 4, 64, 64, "bf16"),
    (8, 2, 64, 16, "f16"),
    (16, 2, 64, 16, "bf16"),
]


@pytest.mark.parametrize("fmt", FORMATS)
@pytest.mark.parametrize("shape", SHAPES)
def test_shared_quant_matches_oracle(shape, fmt):
    heads, kv_heads, D, bs, dtype = shape
    case = sharing_case(11 + bs + D, heads, kv_heads, D, bs, dtype, False)
    k8, v8, ks, vs = quant_case(case, fmt, 5)
    ref = oracle_quant(case, fmt, k8, v8, ks, vs)
    for P in (0, 2 * bs):
        out, ws = run_shared_quant(case, fmt, k8, v8, ks, vs, P)
        err = H.max_err(out, ref)
        assert err <= H.TOL[dtype], (shape, fmt, P, err)
        margins.record(f"shared {fmt} {heads}/{kv_heads} D={D} bs={bs} {dtype} P={P or 'auto'}", err, H.TOL[dtype])
        Pr = pa.pa_decode_shared_partition_size(len(case["ctx"]), heads, kv_heads, D, bs, int(case["ctx"].max()), P)
        n_expect, n_shared = expected_entries(case, Pr, False)
        assert int(ws[4:8].view(torch.int32).item()) == n_expect
        assert n_shared >= 10
        plain = run_plain_quant(case, fmt, k8, v8, ks, vs, P)
        assert float((plain.float() - out.float()).abs().max()) <= H.TOL[dtype]


@pytest.mark.parametrize("fmt", FORMATS)
@pytest.mark.parametrize("group", [1, 2, 4, 8])
def test_shared_quant_whole_context_in_one_shared_unit(group, fmt):
    case = whole_unit_case(group)
    k8, v8, ks, vs = quant_case(case, fmt, 7)
    ref = oracle_quant(case, fmt, k8, v8, ks, vs)
    for P in (256, 32):
        out = run_shared_quant(case, fmt, k8, v8, ks, vs, P)[0]
        assert not torch.isnan(out).any()
        err = H.max_err(out, ref)
        assert err <= H.TOL["f16"], (P, err)


@pytest.mark.parametrize("fmt", FORMATS)
def test_shared_quant_deterministic(fmt):
    case = sharing_case(3, 16, 4, 128, 16, "bf16", False)
    k8, v8, ks, vs = quant_case(case, fmt, 6)
    a = run_shared_quant(case, fmt, k8, v8, ks, vs, 32)[0]
    b = run_shared_quant(case, fmt, k8, v8, ks, vs, 32)[0]
    assert torch.equal(a, b)


@pytest.mark.parametrize("fmt", FORMATS)
@pytest.mark.parametrize("name", ["beam", "beam256"])
def test_shared_quant_beam_workloads(name, fmt):
    """The beam workloads' first step over the quantised pools."""
    wl = workloads.build(name, 0, steps=1)
    st = wl.steps[0]
    ks, vs = head_scales(wl.num_kv_heads, 0.0375), head_scales(wl.num_kv_heads, 0.05).flip(0)
    k8, v8 = quantise(wl.k_pool, ks, fmt), quantise(wl.v_pool, vs, fmt)
    case = dict(q=st.q, tables=st.block_tables, ctx=st.context_lens, scale=wl.scale, dtype=wl.dtype,
                kv_heads=wl.num_kv_heads, bs=wl.block_size)
    out, _ = run_shared_quant(case, fmt, k8, v8, ks, vs, 0)
    ref = oracle_quant(case, fmt, k8, v8, ks, vs)
    err = H.max_err(out, ref)
    assert err <= H.TOL[wl.dtype]
    margins.record(f"shared {fmt} {name} {wl.dtype}", err, H.TOL[wl.dtype])


def test_shared_quant_rejects():
    dev = torch.device("cuda")
    q = torch.zeros((2, 8, 128), dtype=torch.float16, device=dev)
    k8 = torch.zeros((4, 8, 16, 128), dtype=torch.uint8, device=dev)
    tab = torch.zeros((2, 1), dtype=torch.int32, device=dev)
    ctx = torch.ones((2,), dtype=torch.int32, device=dev)
    s = torch.ones((8,), dtype=torch.float32, device=dev)
    with pytest.raises(KeyError):
        pa.pa_decode_shared_quant(torch.empty_like(q), q, k8, k8.clone(), tab, ctx, 0.1, 1, "nf4", s, s)
    with pytest.raises(ValueError):
        pa.pa_decode_shared_quant(torch.empty_like(q), q, k8.half(), k8.half(), tab, ctx, 0.1, 1, "e4m3", s, s)
    with pytest.raises(ValueError):
        pa.pa_decode_shared_quant(torch.empty_like(q), q, k8, k8.clone(), tab, ctx, 0.1, 1, "int8", s[:4], s)


def quant_case_blocks(case, fmt, seed):
    """As quant_case with one scale per (block, KV head), spanning 100x."""
    from tests.test_gpu_quant_blocks import block_scales, quantise_blocks
    kp, vp = case["kp"], case["vp"]
    bad = torch.isnan(kp)
    NB, Hkv = kp.shape[0], kp.shape[1]
    base = 0.01 if fmt == "int8" else 0.0375
    ks, vs = block_scales(NB, Hkv, base, seed), block_scales(NB, Hkv, base, seed + 1)
    k8 = quantise_blocks(torch.nan_to_num(kp), ks, fmt)
    v8 = quantise_blocks(torch.nan_to_num(vp), vs, fmt)
    if fmt == "e4m3":
        k8[bad] = 0x7F
        v8[bad] = 0x7F
    return k8, v8, ks, vs


def run_shared_quant_blocks(case, fmt, k8, v8, ks, vs, P):
    dev = torch.device("cuda")
    q = case["q"].to(dev)
    out = torch.full_like(q, float("nan"))
    mx = int(case["ctx"].max())
    pa.pa_decode_shared_quant_blocks(out, q, k8.to(dev), v8.to(dev), torch.from_numpy(case["tables"]).to(dev),
                                     torch.from_numpy(case["ctx"]).to(dev), case["scale"], mx, fmt, ks.to(dev),
                                     vs.to(dev), P)
    torch.cuda.synchronize()
    assert pa.pa_device_errors() == 0
    return out


@pytest.mark.parametrize("fmt", FORMATS)
@pytest.mark.parametrize("shape", SHAPES)
def test_shared_quant_block_scales_match_oracle(shape, fmt):
    """Shared units over an 8-bit cache with one scale per (block, KV head):
    the group's shared blocks carry their own scales, for every member."""
    heads, kv_heads, D, bs, dtype = shape
    case = sharing_case(31 + bs + D, heads, kv_heads, D, bs, dtype, False)
    k8, v8, ks, vs = quant_case_blocks(case, fmt, 8)
    ref = oracle_quant(case, fmt, k8, v8, ks, vs)
    for P in (0, 2 * bs):
        out = run_shared_quant_blocks(case, fmt, k8, v8, ks, vs, P)
        assert not torch.isnan(out).any()
        err = H.max_err(out, ref)
        assert err <= H.TOL[dtype], (shape, fmt, P, err)
        margins.record(f"shared {fmt} per-block {heads}/{kv_heads} D={D} bs={bs} {dtype} P={P or 'auto'}", err,
                       H.TOL[dtype])


@pytest.mark.parametrize("fmt", FORMATS)
def test_shared_quant_block_scales_beam(fmt):
    from tests.test_gpu_quant_blocks import block_scales, quantise_blocks
    wl = workloads.build("beam", 0, steps=1)
    st = wl.steps[0]
    NB = wl.k_pool.shape[0]
    ks, vs = block_scales(NB, wl.num_kv_heads, 0.0375, 21), block_scales(NB, wl.num_kv_heads, 0.05, 22)
    k8, v8 = quantise_blocks(wl.k_pool, ks, fmt), quantise_blocks(wl.v_pool, vs, fmt)
    case = dict(q=st.q, tables=st.block_tables, ctx=st.context_lens, scale=wl.scale, dtype=wl.dtype,
                kv_heads=wl.num_kv_heads, bs=wl.block_size)
    out = run_shared_quant_blocks(case, fmt, k8, v8, ks, vs, 0)
    ref = oracle_quant(case, fmt, k8, v8, ks, vs)
    err = H.max_err(out, ref)
    assert err <= H.TOL[wl.dtype]
    margins.record(f"shared {fmt} per-block beam {wl.dtype}", err, H.TOL[wl.dtype])
