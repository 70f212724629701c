"""Seeded random shapes through every decode entry point, against the oracle.

Each case draws the batch size, query heads per KV head, KV heads, head size,
block size, dtype, context lengths (empty, one token, block edges, several
partitions), the partition size and the entry point: pa_decode,
pa_decode_append, pa_decode_shared (with and without the fused append),
pa_decode_fp8, pa_decode_quant in both formats, pa_decode_shared_quant, and
the per-(block, KV head) scale entry points pa_decode_quant_blocks and
pa_decode_shared_quant_blocks.
Sequences of the shared-prefix cases come in groups whose tables begin with
the same blocks. Every output row starts as NaN, so a row no kernel writes
fails; cache writes are compared bit for bit.
"""
from __future__ import annotations

import math

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_372_b200 as pa
from paged_kv_cache_372_b200 import inputs
from tests import gpu_harness as H
from tests.bruteforce import bits_of
from tests.test_gpu_quant import head_scales, quantise
from tests.test_gpu_quant_blocks import block_scales, quantise_blocks

pytestmark = pytest.mark.gpu

PATHS = ("plain", "append", "shared", "shared_append", "fp8", "quant_int8", "quant_e4m3", "shared_quant_int8",
         "shared_quant_e4m3", "blocks_int8", "blocks_e4m3", "shared_blocks_int8")
CASES = 8 * len(PATHS)


def draw(seed: int) -> dict:
    rng = np.random.default_rng(9000 + seed)
    path = PATHS[seed % len(PATHS)]
    G = int(rng.choice([1, 2, 4, 8]))
    Hkv = int(rng.choice([1, 2, 4]))
    D = int(rng.choice([64, 128]))
    bs = int(rng.choice([16, 32, 64]))
    dtype = str(rng.choice(["f16", "bf16"]))
    B = int(rng.integers(1, 41))
    edges = [1, bs - 1, bs, bs + 1, 2 * bs, 16, 17]
    ctx = []
    for _ in range(B):
        r = rng.random()
        if r < 0.06 and "append" not in path:
            ctx.append(0)
        elif r < 0.3:
            ctx.append(int(rng.choice(edges)))
        else:
            ctx.append(int(rng.integers(1, 1500)))
    cap = 32 * bs
    P = 0 if rng.random() < 0.4 else int(rng.choice([m for m in (16, 32, 64, 128, 256, 512, 1024, 2048)
                                                      if m % bs == 0 and m <= cap]))
    return dict(seed=seed, path=path, G=G, Hkv=Hkv, H=G * Hkv, D=D, bs=bs, dtype=dtype, B=B, ctx=ctx, P=P)


def tables_for(c: dict, gen: torch.Generator, rng: np.random.Generator):
    """Block tables from a shuffled free list; for shared-prefix paths the
    sequences come in groups of 2-6 whose tables start with the same blocks."""
    bs, ctx = c["bs"], c["ctx"]
    need = [max(1, -(-n // bs)) for n in ctx]
    NB = int(sum(need) * 1.25) + 8
    free = list(inputs.permutation(NB, gen))
    W = max(need)
    tables = np.full((len(ctx), W), -1, dtype=np.int32)
    i = 0
    while i < len(ctx):
        n = int(rng.integers(2, 7)) if c["path"].startswith("shared") else 1
        group = list(range(i, min(i + n, len(ctx))))
        common = min(need[g] for g in group)
        k = int(rng.integers(0, common + 1)) if len(group) > 1 else 0
        prefix = [free.pop() for _ in range(k)]
        for g in group:
            tables[g, :k] = prefix
            for j in range(k, need[g]):
                tables[g, j] = free.pop()
        i += n
    return tables, NB


@pytest.mark.parametrize("seed", range(CASES))
def test_random_shape(seed):
    c = draw(seed)
    gen = inputs.generator(9100 + seed)
    rng = np.random.default_rng(9200 + seed)
    B, Hh, Hkv, D, bs, dtype, path = c["B"], c["H"], c["Hkv"], c["D"], c["bs"], c["dtype"], c["path"]
    tables, NB = tables_for(c, gen, rng)
    ctx = np.array(c["ctx"], dtype=np.int32)
    # A fused append writes each sequence's last position: keep that block private.
    if "append" in path:
        for s in range(B):
            last = (int(ctx[s]) - 1) // bs
            shared = [t for t in range(B) if t != s and tables[t, last] == tables[s, last]]
            if shared:
                tables[s, last] = NB
                NB += 1
    kp = inputs.normal((NB, Hkv, bs, D), dtype, gen)
    vp = inputs.normal((NB, Hkv, bs, D), dtype, gen)
    q = inputs.normal((B, Hh, D), dtype, gen)
    scale = 1.0 / math.sqrt(D)
    mx = max(1, int(ctx.max()))
    dev = torch.device("cuda")
    tab, ctx_d = torch.from_numpy(tables).to(dev), torch.from_numpy(ctx).to(dev)
    out = torch.full_like(q, float("nan")).to(dev)
    qd = q.to(dev)
    label = f"{c}"

    if path in ("plain", "append", "shared", "shared_append"):
        okp, ovp = bits_of(kp).copy(), bits_of(vp).copy()
        kpd, vpd = kp.to(dev), vp.to(dev)
        kw = {}
        if "append" in path:
            k_new = inputs.normal((B, Hkv, D), dtype, gen)
            v_new = inputs.normal((B, Hkv, D), dtype, gen)
            slots = np.array([tables[s, (int(ctx[s]) - 1) // bs] * bs + (int(ctx[s]) - 1) % bs for s in range(B)],
                             dtype=np.int64)
            oracle.reshape_and_cache(bits_of(k_new), bits_of(v_new), okp, ovp, slots)
            kw = dict(k_new=k_new.to(dev), v_new=v_new.to(dev))
        if path == "plain":
            pa.pa_decode(out, qd, kpd, vpd, tab, ctx_d, scale, mx, c["P"])
        elif path == "append":
            pa.pa_decode_append(out, qd, kw["k_new"], kw["v_new"], kpd, vpd, tab, ctx_d, scale, mx, c["P"])
        else:
            pa.pa_decode_shared(out, qd, kpd, vpd, tab, ctx_d, scale, mx, c["P"], **kw)
        torch.cuda.synchronize()
        assert pa.pa_device_errors() == 0, label
        ref = oracle.paged_attention(bits_of(q), okp, ovp, tables, ctx, scale, dtype)
        if "append" in path:
            assert H.pools_equal(kpd, vpd, okp, ovp), label
    else:
        fmt = "int8" if path.endswith("int8") else "e4m3"
        blocks = "blocks" in path
        base = 0.01 if fmt == "int8" else 0.0375
        if path == "fp8":
            ks = vs = torch.full((Hkv,), 0.0375, dtype=torch.float32)
        elif blocks:
            ks, vs = block_scales(NB, Hkv, base, 9300 + seed), block_scales(NB, Hkv, base, 9400 + seed)
        else:
            ks, vs = head_scales(Hkv, base), head_scales(Hkv, base).flip(0).contiguous()
        if blocks:
            k8, v8 = quantise_blocks(kp, ks, fmt), quantise_blocks(vp, vs, fmt)
        else:
            k8, v8 = quantise(kp, ks, fmt), quantise(vp, vs, fmt)
        k8d, v8d = k8.to(dev), v8.to(dev)
        if path == "fp8":
            pa.pa_decode_fp8(out, qd, k8d, v8d, tab, ctx_d, scale, mx, 0.0375, 0.0375, c["P"])
        elif path == "shared_blocks_int8":
            pa.pa_decode_shared_quant_blocks(out, qd, k8d, v8d, tab, ctx_d, scale, mx, fmt, ks.to(dev), vs.to(dev),
                                             c["P"])
        elif blocks:
            pa.pa_decode_quant_blocks(out, qd, k8d, v8d, tab, ctx_d, scale, mx, fmt, ks.to(dev), vs.to(dev), c["P"])
        elif path.startswith("shared"):
            pa.pa_decode_shared_quant(out, qd, k8d, v8d, tab, ctx_d, scale, mx, fmt, ks.to(dev), vs.to(dev), c["P"])
        else:
            pa.pa_decode_quant(out, qd, k8d, v8d, tab, ctx_d, scale, mx, fmt, ks.to(dev), vs.to(dev), c["P"])
        torch.cuda.synchronize()
        assert pa.pa_device_errors() == 0, label
        ref = oracle.paged_attention_kv8(bits_of(q), k8.numpy(), v8.numpy(), tables, ctx, scale, dtype, fmt,
                                         ks.double().numpy(), vs.double().numpy())
    assert not torch.isnan(out).any(), label
    err = H.max_err(out, ref)
    assert err <= H.TOL[dtype], (label, err)
