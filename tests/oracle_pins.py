"""Pins for the oracle: checks against things other than the oracle itself.

Each ``pin_*`` takes an ``oracle.Oracle`` handle and raises AssertionError on a
mismatch. ``test_oracle_pins.py`` runs them on the real oracle (all must pass);
``test_oracle_mutants.py`` runs them on copies of the oracle with one planted
mistake each (at least one pin must fail for every copy).

What pins what:
  * element decoding      all 65536 patterns vs numpy float16 / float32 types
  * paged attention       numpy contiguous-cache brute force; torch SDPA (fp64),
                          on fixed shapes and on seeded random tiny shapes;
                          closed forms (1 token -> its V row; equal keys or
                          scale 0 -> mean of V; a 2-token case with weights
                          1/(1+e) and e/(1+e)); invariants (physical block
                          permutation, shared == duplicated blocks, NaN in
                          unwritten tail slots, GQA head mapping)
  * cache write / copies  numpy fancy-index scatter and slice copies
  * slot mapping          enumeration of the contiguous token order
  * E4M3 (fp8) codes      all 256 codes vs torch's float8_e4m3fn; encoding vs
                          torch's cast (in range, exact midpoints), saturation
                          closed forms, round trip of every finite code
  * fp8 attention / write brute force over the numpy-dequantised cache; numpy
                          float32 division + torch's cast
  * INT8 codes            every byte decodes to byte - 128; encoding vs numpy's
                          round-half-to-even clipped to [-127, 127]
  * 8-bit cache with      E4M3 and INT8, per-KV-head scales spanning up to
    per-head scales       100x: brute force over the numpy-dequantised cache;
                          the write vs numpy / torch per head
"""
from __future__ import annotations

import math

import numpy as np
import torch

from tests.bruteforce import bits_of, contiguous_attention, decode, sdpa_attention

ATOL = 1e-12


def _rand_bits(rng, shape, dtype):
    x = torch.from_numpy(rng.standard_normal(shape).astype(np.float32))
    return bits_of(x.to(torch.float16 if dtype == "f16" else torch.bfloat16))


def _case(rng, B, H, Hkv, D, bs, ctx, dtype, extra_blocks=3):
    """Random pools and a random (scattered) block placement."""
    need = sum(-(-c // bs) for c in ctx)
    NB = need + extra_blocks
    perm = rng.permutation(NB)
    width = max(1, max(-(-c // bs) for c in ctx))
    tables = np.full((B, width), -1, dtype=np.int32)
    k = 0
    for s, c in enumerate(ctx):
        for j in range(-(-c // bs)):
            tables[s, j] = perm[k]
            k += 1
    q = _rand_bits(rng, (B, H, D), dtype)
    kp = _rand_bits(rng, (NB, Hkv, bs, D), dtype)
    vp = _rand_bits(rng, (NB, Hkv, bs, D), dtype)
    return q, kp, vp, tables, np.array(ctx, dtype=np.int32)


SHAPES = [  # B, H, Hkv, D, bs, ctx, dtype
    (3, 2, 2, 64, 16, [1, 17, 40], "f16"),
    (2, 8, 2, 64, 16, [33, 5], "bf16"),
    (2, 4, 1, 128, 32, [64, 95], "bf16"),
    (2, 8, 1, 64, 64, [130, 64], "f16"),
    (4, 6, 3, 16, 16, [16, 31, 2, 48], "f16"),
]


def pin_decode_f16(orc):
    bits = np.arange(65536, dtype=np.uint16)
    got = orc.to_double(bits, "f16")
    ref = decode(bits, "f16")
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    m = ~np.isnan(ref)
    assert np.array_equal(got[m], ref[m])
    assert np.array_equal(np.signbit(got[m]), np.signbit(ref[m]))


def pin_decode_bf16(orc):
    bits = np.arange(65536, dtype=np.uint16)
    got = orc.to_double(bits, "bf16")
    ref = decode(bits, "bf16")
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    m = ~np.isnan(ref)
    assert np.array_equal(got[m], ref[m])
    assert np.array_equal(np.signbit(got[m]), np.signbit(ref[m]))
    # torch's own bfloat16 -> float64 conversion agrees as well
    t = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(got[m], t[m])


def pin_bruteforce(orc, seed=0):
    rng = np.random.default_rng(seed)
    for B, H, Hkv, D, bs, ctx, dt in SHAPES:
        q, kp, vp, tab, cl = _case(rng, B, H, Hkv, D, bs, ctx, dt)
        scale = 1.0 / math.sqrt(D)
        got = orc.paged_attention(q, kp, vp, tab, cl, scale, dt)
        ref = contiguous_attention(decode(q, dt), decode(kp, dt), decode(vp, dt), tab, cl, scale)
        assert np.abs(got - ref).max() <= ATOL, (B, H, Hkv, D, bs, ctx, dt)


def pin_sdpa(orc, seed=1):
    rng = np.random.default_rng(seed)
    for B, H, Hkv, D, bs, ctx, dt in SHAPES:
        q, kp, vp, tab, cl = _case(rng, B, H, Hkv, D, bs, ctx, dt)
        scale = 0.5 / math.sqrt(D)
        got = orc.paged_attention(q, kp, vp, tab, cl, scale, dt)
        ref = sdpa_attention(decode(q, dt), decode(kp, dt), decode(vp, dt), tab, cl, scale)
        assert np.abs(got - ref).max() <= ATOL


def random_shapes(rng, n):
    """n seeded random tiny shapes: 1-4 sequences with contexts in [0, 80)
    (empty ones included), 1-3 KV heads with groups of 1-4 query heads, head
    sizes 8-64, block sizes 1-32, fp16 or bf16."""
    shapes = []
    for _ in range(n):
        B = int(rng.integers(1, 5))
        Hkv = int(rng.integers(1, 4))
        G = int(rng.choice([1, 2, 3, 4]))
        D = int(rng.choice([8, 16, 24, 64]))
        bs = int(rng.choice([1, 2, 4, 8, 16, 32]))
        ctx = [int(c) for c in rng.integers(0, 80, B)]
        shapes.append((B, G * Hkv, Hkv, D, bs, ctx, str(rng.choice(["f16", "bf16"]))))
    return shapes


def pin_random_shapes(orc, seed=15, n=24):
    """The oracle against the numpy brute force and torch SDPA on seeded random
    tiny shapes, each with its own random scale."""
    rng = np.random.default_rng(seed)
    for B, H, Hkv, D, bs, ctx, dt in random_shapes(rng, n):
        q, kp, vp, tab, cl = _case(rng, B, H, Hkv, D, bs, ctx, dt)
        scale = float(rng.uniform(0.1, 2.0)) / math.sqrt(D)
        got = orc.paged_attention(q, kp, vp, tab, cl, scale, dt)
        args = (decode(q, dt), decode(kp, dt), decode(vp, dt), tab, cl, scale)
        for ref in (contiguous_attention(*args), sdpa_attention(*args)):
            assert np.abs(got - ref).max() <= ATOL, (B, H, Hkv, D, bs, ctx, dt)


def pin_single_token(orc, seed=2):
    """context_len 1: the softmax of one score is 1, so out is that token's V row."""
    rng = np.random.default_rng(seed)
    q, kp, vp, tab, cl = _case(rng, 3, 4, 2, 64, 16, [1, 1, 1], "bf16")
    got = orc.paged_attention(q, kp, vp, tab, cl, 0.125, "bf16")
    V = decode(vp, "bf16")
    for s in range(3):
        for h in range(4):
            assert np.array_equal(got[s, h], V[tab[s, 0], h // 2, 0])


def pin_equal_keys(orc, seed=3):
    """Equal keys give equal scores, so every weight is 1/n: out = mean of V.
    Scale 0 gives the same for any keys."""
    rng = np.random.default_rng(seed)
    q, kp, vp, tab, cl = _case(rng, 2, 2, 2, 64, 16, [37, 9], "f16")
    V = decode(vp, "f16")
    same = kp.copy()
    same[:] = kp[0, 0, 0]
    for keys, scale in ((same, 0.125), (kp, 0.0)):
        got = orc.paged_attention(q, keys, vp, tab, cl, scale, "f16")
        for s in range(2):
            n = int(cl[s])
            rows = np.stack([V[tab[s, t // 16], :, t % 16, :] for t in range(n)])
            for h in range(2):
                assert np.abs(got[s, h] - rows[:, h, :].mean(axis=0)).max() <= ATOL


def pin_two_token_closed_form(orc):
    """q = e0, k0 = 0, k1 = e0, scale 1: scores (0, 1), weights (1, e)/(1 + e)."""
    D, bs = 16, 16
    one = np.float16(1.0).view(np.uint16)
    q = np.zeros((1, 1, D), dtype=np.uint16)
    q[0, 0, 0] = one
    kp = np.zeros((2, 1, bs, D), dtype=np.uint16)
    kp[1, 0, 1, 0] = one                     # token 1 lives in block 1, slot 1
    vp = np.zeros((2, 1, bs, D), dtype=np.uint16)
    v0 = np.arange(D, dtype=np.float16)
    v1 = (-np.arange(D, dtype=np.float16)) * np.float16(0.5)
    vp[1, 0, 0] = v0.view(np.uint16)
    vp[1, 0, 1] = v1.view(np.uint16)
    tab = np.array([[1]], dtype=np.int32)
    got = orc.paged_attention(q, kp, vp, tab, np.array([2], np.int32), 1.0, "f16")
    e = math.e
    want = (v0.astype(np.float64) + e * v1.astype(np.float64)) / (1.0 + e)
    assert np.abs(got[0, 0] - want).max() <= ATOL


def pin_block_permutation(orc, seed=4):
    """Physical placement is irrelevant: permuting blocks (and the tables with
    them) gives bit-identical output."""
    rng = np.random.default_rng(seed)
    for B, H, Hkv, D, bs, ctx, dt in SHAPES:
        q, kp, vp, tab, cl = _case(rng, B, H, Hkv, D, bs, ctx, dt)
        pi = rng.permutation(kp.shape[0])
        kp2 = np.empty_like(kp)
        vp2 = np.empty_like(vp)
        kp2[pi] = kp
        vp2[pi] = vp
        tab2 = np.where(tab >= 0, pi[np.maximum(tab, 0)], -1).astype(np.int32)
        a = orc.paged_attention(q, kp, vp, tab, cl, 0.1, dt)
        b = orc.paged_attention(q, kp2, vp2, tab2, cl, 0.1, dt)
        assert np.array_equal(a, b)


def pin_shared_equals_duplicated(orc, seed=5):
    """Two sequences reading the same physical blocks give the same result as when
    one of them reads a byte copy of those blocks."""
    rng = np.random.default_rng(seed)
    q, kp, vp, tab, cl = _case(rng, 2, 4, 2, 64, 16, [45, 45], "bf16", extra_blocks=6)
    q[1] = q[0]
    shared = tab.copy()
    shared[1] = shared[0]
    dup = tab.copy()
    for j in range(3):          # sequence 1's own blocks become copies of 0's
        kp[dup[1, j]] = kp[dup[0, j]]
        vp[dup[1, j]] = vp[dup[0, j]]
    a = orc.paged_attention(q, kp, vp, shared, cl, 0.125, "bf16")
    b = orc.paged_attention(q, kp, vp, dup, cl, 0.125, "bf16")
    assert np.array_equal(a, b)
    assert np.array_equal(a[0], a[1])


def pin_tail_slots_ignored(orc, seed=6):
    """Unwritten slots past context_len (NaN here) never reach the output."""
    rng = np.random.default_rng(seed)
    for B, H, Hkv, D, bs, ctx, dt in SHAPES:
        q, kp, vp, tab, cl = _case(rng, B, H, Hkv, D, bs, ctx, dt)
        a = orc.paged_attention(q, kp, vp, tab, cl, 0.1, dt)
        nan = np.uint16(0x7e00 if dt == "f16" else 0x7fc0)
        for s, n in enumerate(cl):
            if n % bs:
                b = tab[s, n // bs]
                kp[b, :, n % bs:, :] = nan
                vp[b, :, n % bs:, :] = nan
        b = orc.paged_attention(q, kp, vp, tab, cl, 0.1, dt)
        assert np.isfinite(b).all() and np.array_equal(a, b)


def pin_gqa_mapping(orc):
    """With H=6, Hkv=3 (groups of 2) and one token, head h returns KV head h//2's V."""
    D, bs = 16, 16
    q = np.zeros((1, 6, D), dtype=np.uint16)
    kp = np.zeros((1, 3, bs, D), dtype=np.uint16)
    vp = np.zeros((1, 3, bs, D), dtype=np.uint16)
    for kvh in range(3):
        vp[0, kvh, 0, :] = np.full(D, kvh + 1, dtype=np.float16).view(np.uint16)
    got = orc.paged_attention(q, kp, vp, np.array([[0]], np.int32), np.array([1], np.int32),
                              1.0, "f16")
    for h in range(6):
        assert np.array_equal(got[0, h], np.full(D, h // 2 + 1, dtype=np.float64))


def pin_empty_context(orc):
    q, kp, vp, tab, cl = _case(np.random.default_rng(7), 2, 2, 2, 16, 16, [0, 3], "f16")
    got = orc.paged_attention(q, kp, vp, tab, cl, 0.25, "f16")
    assert np.array_equal(got[0], np.zeros_like(got[0])) and np.abs(got[1]).sum() > 0


def pin_reshape_and_cache(orc, seed=8):
    rng = np.random.default_rng(seed)
    NB, Hkv, bs, D, T = 6, 3, 16, 32, 20
    kp = rng.integers(0, 65536, (NB, Hkv, bs, D), dtype=np.uint16)
    vp = rng.integers(0, 65536, (NB, Hkv, bs, D), dtype=np.uint16)
    k = rng.integers(0, 65536, (T, Hkv, D), dtype=np.uint16)
    v = rng.integers(0, 65536, (T, Hkv, D), dtype=np.uint16)
    slots = rng.choice(NB * bs, T, replace=False).astype(np.int64)
    slots[3] = -1                                   # skipped token
    ek, ev = kp.copy(), vp.copy()
    keep = slots >= 0
    ek[slots[keep] // bs, :, slots[keep] % bs, :] = k[keep]
    ev[slots[keep] // bs, :, slots[keep] % bs, :] = v[keep]
    orc.reshape_and_cache(k, v, kp, vp, slots)
    assert np.array_equal(kp, ek) and np.array_equal(vp, ev)


def pin_copy_blocks(orc, seed=9):
    rng = np.random.default_rng(seed)
    pools = [rng.integers(0, 256, (10, 3, 4, 8), dtype=np.uint8) for _ in range(3)]
    bb = 3 * 4 * 8
    pairs = np.array([[1, 7], [4, 2], [1, 9]], dtype=np.int64)
    want = [p.copy() for p in pools]
    for w in want:
        for s, d in pairs:
            w[d] = w[s]
    orc.copy_blocks(pools, pairs, bb)
    for p, w in zip(pools, want):
        assert np.array_equal(p, w)


def pin_swap_blocks(orc, seed=11):
    """Cross-pool block copies vs numpy slice assignment; the source is untouched."""
    rng = np.random.default_rng(seed)
    src = [rng.integers(0, 256, (9, 2, 4, 8), dtype=np.uint8) for _ in range(2)]
    dst = [rng.integers(0, 256, (5, 2, 4, 8), dtype=np.uint8) for _ in range(2)]
    bb = 2 * 4 * 8
    pairs = np.array([[7, 0], [2, 4], [8, 1]], dtype=np.int64)
    want = [d.copy() for d in dst]
    before = [x.copy() for x in src]
    for w, x in zip(want, src):
        for a, b in pairs:
            w[b] = x[a]
    orc.swap_blocks(dst, src, pairs, bb)
    for d, w in zip(dst, want):
        assert np.array_equal(d, w)
    for x, b in zip(src, before):
        assert np.array_equal(x, b)


def _torch_e4m3_codes(x: np.ndarray) -> np.ndarray:
    """float32 -> E4M3 codes through torch's own float8_e4m3fn cast (in-range values)."""
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.float8_e4m3fn)
    return t.view(torch.uint8).numpy()


def pin_e4m3_decode(orc):
    codes = np.arange(256, dtype=np.uint8)
    got = orc.e4m3_to_double(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(np.isnan(got), np.isnan(ref)) and np.isnan(got).sum() == 2
    m = ~np.isnan(ref)
    assert np.array_equal(got[m], ref[m])
    assert got[0x7e] == 448.0 and got[0x01] == 2.0 ** -9 and got[0x08] == 2.0 ** -6


def pin_e4m3_encode(orc, seed=12):
    rng = np.random.default_rng(seed)
    x = np.concatenate([rng.standard_normal(3000) * s for s in (1e-3, 0.05, 1.0, 20.0, 120.0)])
    x = np.clip(x, -440.0, 440.0).astype(np.float32)
    codes = np.arange(256, dtype=np.uint8)
    vals = orc.e4m3_to_double(codes)
    finite = codes[~np.isnan(vals)]
    mids = []                                   # exact midpoints between neighbours: ties to even
    pos = np.sort(vals[(vals >= 0) & ~np.isnan(vals)])
    mids = ((pos[1:] + pos[:-1]) / 2).astype(np.float32)
    x = np.concatenate([x, mids, -mids, vals[~np.isnan(vals)].astype(np.float32)])
    assert np.array_equal(orc.e4m3_encode(x), _torch_e4m3_codes(x))
    # saturation (no infinities in E4M3): past 448 the code is +-448
    big = np.array([448.0, 449.0, 463.9, 464.0, 1e6, -500.0, np.inf, -np.inf], dtype=np.float32)
    assert list(orc.e4m3_encode(big)) == [0x7e, 0x7e, 0x7e, 0x7e, 0x7e, 0xfe, 0x7e, 0xfe]
    # every finite code round-trips
    assert np.array_equal(orc.e4m3_encode(vals[finite].astype(np.float32)), finite)


def _fp8_case(rng, B, H, Hkv, D, bs, ctx, dtype):
    q, kp, vp, tab, cl = _case(rng, B, H, Hkv, D, bs, ctx, dtype)
    k8 = rng.integers(0, 256, kp.shape, dtype=np.uint8)
    v8 = rng.integers(0, 256, vp.shape, dtype=np.uint8)
    for a in (k8, v8):                          # no NaN codes in the cache
        a[(a & 0x7f) == 0x7f] = 0x10
    return q, k8, v8, tab, cl


def pin_fp8_attention_bruteforce(orc, seed=13):
    """fp8 attention = attention over the dequantised cache (numpy dequantisation)."""
    rng = np.random.default_rng(seed)
    for B, H, Hkv, D, bs, ctx, dt in SHAPES:
        q, k8, v8, tab, cl = _fp8_case(rng, B, H, Hkv, D, bs, ctx, dt)
        ks, vs = 0.37, 1.9
        got = orc.paged_attention_fp8(q, k8, v8, tab, cl, 1.0 / math.sqrt(D), dt, ks, vs)
        deq = lambda a, sc: torch.from_numpy(a).view(torch.float8_e4m3fn).to(torch.float64).numpy() * sc
        ref = contiguous_attention(decode(q, dt), deq(k8, ks), deq(v8, vs), tab, cl, 1.0 / math.sqrt(D))
        # random codes span the whole E4M3 range (|v| up to 448 * vs): relative bound
        assert np.abs(got - ref).max() <= ATOL * max(1.0, np.abs(ref).max())


def pin_fp8_cache_write(orc, seed=14):
    """Quantising write: code = E4M3(x / scale) with the division in float32."""
    rng = np.random.default_rng(seed)
    NB, Hkv, bs, D, T = 5, 2, 16, 32, 12
    for dt in ("f16", "bf16"):
        k = _rand_bits(rng, (T, Hkv, D), dt)
        v = _rand_bits(rng, (T, Hkv, D), dt)
        kp = rng.integers(0, 256, (NB, Hkv, bs, D), dtype=np.uint8)
        vp = rng.integers(0, 256, (NB, Hkv, bs, D), dtype=np.uint8)
        slots = rng.choice(NB * bs, T, replace=False).astype(np.int64)
        ks, vs = np.float32(0.0213), np.float32(0.75)
        ek, ev = kp.copy(), vp.copy()
        kx = (decode(k, dt).astype(np.float32) / ks).astype(np.float32)
        vx = (decode(v, dt).astype(np.float32) / vs).astype(np.float32)
        ek[slots // bs, :, slots % bs, :] = _torch_e4m3_codes(np.clip(kx, -448, 448))
        ev[slots // bs, :, slots % bs, :] = _torch_e4m3_codes(np.clip(vx, -448, 448))
        orc.reshape_and_cache_fp8(k, v, kp, vp, slots, dt, float(ks), float(vs))
        assert np.array_equal(kp, ek) and np.array_equal(vp, ev)


def pin_int8_codes(orc, seed=16):
    """INT8 (excess-128) codes: every byte decodes to byte - 128; the encoder is
    numpy's round-half-to-even clipped to [-127, 127], with exact ties, the
    saturation points, NaN (stored as zero) and infinities."""
    codes = np.arange(256, dtype=np.uint8)
    assert np.array_equal(orc.int8_to_double(codes), codes.astype(np.float64) - 128.0)
    rng = np.random.default_rng(seed)
    x = np.concatenate([rng.standard_normal(1500) * s for s in (0.3, 3.0, 40.0, 200.0)])
    x = np.concatenate([x, np.arange(-130, 130) + 0.5, np.arange(-130, 131)]).astype(np.float32)
    want = (np.clip(np.rint(x), -127, 127).astype(np.int64) + 128).astype(np.uint8)
    assert np.array_equal(orc.int8_encode(x), want)
    special = np.array([np.nan, np.inf, -np.inf, 127.49, -127.5, 1e30], dtype=np.float32)
    assert list(orc.int8_encode(special)) == [128, 255, 1, 255, 1, 255]


def _dequant_kv8(codes, kv_format, scales):
    """Codes [NB][Hkv][bs][D] -> float64 values with one scale per KV head: E4M3
    through torch's float8_e4m3fn, INT8 as byte - 128."""
    if kv_format == "e4m3":
        v = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    else:
        v = codes.astype(np.float64) - 128.0
    return v * np.asarray(scales, dtype=np.float64)[None, :, None, None]


def _head_scales(rng, n, base):
    """n per-head scales spanning up to 100x around `base`."""
    return base * 10.0 ** rng.uniform(-1.0, 1.0, n)


def pin_kv8_attention_bruteforce(orc, seed=17):
    """Attention over an 8-bit cache with per-KV-head scales (E4M3 and INT8) =
    the brute force over the numpy-dequantised cache."""
    rng = np.random.default_rng(seed)
    for fmt in ("e4m3", "int8"):
        for B, H, Hkv, D, bs, ctx, dt in SHAPES:
            q, k8, v8, tab, cl = _fp8_case(rng, B, H, Hkv, D, bs, ctx, dt)
            ks, vs = _head_scales(rng, Hkv, 0.05), _head_scales(rng, Hkv, 0.05)
            got = orc.paged_attention_kv8(q, k8, v8, tab, cl, 1.0 / math.sqrt(D), dt, fmt, ks, vs)
            ref = contiguous_attention(decode(q, dt), _dequant_kv8(k8, fmt, ks), _dequant_kv8(v8, fmt, vs), tab, cl,
                                       1.0 / math.sqrt(D))
            assert np.abs(got - ref).max() <= ATOL * max(1.0, np.abs(ref).max()), (fmt, B, H, Hkv)


def pin_kv8_cache_write(orc, seed=18):
    """Quantising write with per-KV-head scales: code = encode(x / scale[h]) with
    the division in float32; E4M3 through torch's cast, INT8 through numpy."""
    rng = np.random.default_rng(seed)
    NB, Hkv, bs, D, T = 5, 3, 16, 32, 12
    for fmt in ("e4m3", "int8"):
        for dt in ("f16", "bf16"):
            k = _rand_bits(rng, (T, Hkv, D), dt)
            v = _rand_bits(rng, (T, Hkv, D), dt)
            kp = rng.integers(0, 256, (NB, Hkv, bs, D), dtype=np.uint8)
            vp = rng.integers(0, 256, (NB, Hkv, bs, D), dtype=np.uint8)
            slots = rng.choice(NB * bs, T, replace=False).astype(np.int64)
            slots[2] = -1
            ks = _head_scales(rng, Hkv, 0.02).astype(np.float32)
            vs = _head_scales(rng, Hkv, 0.02).astype(np.float32)
            ek, ev = kp.copy(), vp.copy()
            keep = slots >= 0
            for pool, x, sc in ((ek, k, ks), (ev, v, vs)):
                y = (decode(x, dt).astype(np.float32) / sc[None, :, None]).astype(np.float32)
                if fmt == "e4m3":
                    codes = _torch_e4m3_codes(np.clip(y, -448, 448))
                else:
                    codes = (np.clip(np.rint(y), -127, 127).astype(np.int64) + 128).astype(np.uint8)
                pool[slots[keep] // bs, :, slots[keep] % bs, :] = codes[keep]
            orc.reshape_and_cache_kv8(k, v, kp, vp, slots, dt, fmt, ks, vs)
            assert np.array_equal(kp, ek) and np.array_equal(vp, ev), (fmt, dt)


def _block_scales(rng, NB, Hkv, base):
    """[NB][Hkv] scales spanning up to 100x around `base`."""
    return base * 10.0 ** rng.uniform(-1.0, 1.0, (NB, Hkv))


def pin_kv8_blocks_attention_bruteforce(orc, seed=19):
    """Attention over an 8-bit cache with one scale per (physical block, KV
    head) = the brute force over the cache dequantised by numpy, block by
    block (each element times the scale of its own block and head)."""
    rng = np.random.default_rng(seed)
    for fmt in ("e4m3", "int8"):
        for B, H, Hkv, D, bs, ctx, dt in SHAPES:
            q, k8, v8, tab, cl = _fp8_case(rng, B, H, Hkv, D, bs, ctx, dt)
            NB = k8.shape[0]
            ks, vs = _block_scales(rng, NB, Hkv, 0.05), _block_scales(rng, NB, Hkv, 0.05)
            got = orc.paged_attention_kv8(q, k8, v8, tab, cl, 1.0 / math.sqrt(D), dt, fmt, ks, vs)
            kd = _dequant_kv8(k8, fmt, np.ones(Hkv)) * ks[:, :, None, None]
            vd = _dequant_kv8(v8, fmt, np.ones(Hkv)) * vs[:, :, None, None]
            ref = contiguous_attention(decode(q, dt), kd, vd, tab, cl, 1.0 / math.sqrt(D))
            assert np.abs(got - ref).max() <= ATOL * max(1.0, np.abs(ref).max()), (fmt, B, H, Hkv)


def pin_kv8_blocks_cache_write(orc, seed=20):
    """Quantising write with one scale per (block, KV head): code =
    encode(x / scale[block of the slot][h]) with the division in float32."""
    rng = np.random.default_rng(seed)
    NB, Hkv, bs, D, T = 6, 3, 16, 32, 40
    for fmt in ("e4m3", "int8"):
        for dt in ("f16", "bf16"):
            k = _rand_bits(rng, (T, Hkv, D), dt)
            v = _rand_bits(rng, (T, Hkv, D), dt)
            kp = rng.integers(0, 256, (NB, Hkv, bs, D), dtype=np.uint8)
            vp = rng.integers(0, 256, (NB, Hkv, bs, D), dtype=np.uint8)
            slots = rng.choice(NB * bs, T, replace=False).astype(np.int64)
            slots[5] = -1
            ks = _block_scales(rng, NB, Hkv, 0.02).astype(np.float32)
            vs = _block_scales(rng, NB, Hkv, 0.02).astype(np.float32)
            ek, ev = kp.copy(), vp.copy()
            for t in range(T):
                if slots[t] < 0:
                    continue
                b, o = int(slots[t]) // bs, int(slots[t]) % bs
                for pool, x, sc in ((ek, k, ks), (ev, v, vs)):
                    y = (decode(x[t], dt).astype(np.float32) / sc[b][:, None]).astype(np.float32)
                    if fmt == "e4m3":
                        codes = _torch_e4m3_codes(np.clip(y, -448, 448))
                    else:
                        codes = (np.clip(np.rint(y), -127, 127).astype(np.int64) + 128).astype(np.uint8)
                    pool[b, :, o, :] = codes
            orc.reshape_and_cache_kv8(k, v, kp, vp, slots, dt, fmt, ks, vs)
            assert np.array_equal(kp, ek) and np.array_equal(vp, ev), (fmt, dt)


def pin_slot_mapping(orc, seed=10):
    rng = np.random.default_rng(seed)
    bs, B, W = 16, 5, 6
    tables = rng.permutation(B * W).reshape(B, W).astype(np.int32)
    seq_ids, positions, want = [], [], []
    for s in range(B):
        order = [tables[s, j] * bs + o for j in range(W) for o in range(bs)]  # token order
        for pos in rng.choice(W * bs, 7, replace=False):
            seq_ids.append(s)
            positions.append(int(pos))
            want.append(order[pos])
    got = orc.slot_mapping(tables, seq_ids, positions, bs)
    assert np.array_equal(got, np.array(want, dtype=np.int64))


ALL_PINS = [pin_decode_f16, pin_decode_bf16, pin_bruteforce, pin_sdpa, pin_random_shapes, pin_single_token,
            pin_equal_keys, pin_two_token_closed_form, pin_block_permutation,
            pin_shared_equals_duplicated, pin_tail_slots_ignored, pin_gqa_mapping,
            pin_empty_context, pin_reshape_and_cache, pin_copy_blocks, pin_swap_blocks, pin_slot_mapping,
            pin_e4m3_decode, pin_e4m3_encode, pin_fp8_attention_bruteforce, pin_fp8_cache_write,
            pin_int8_codes, pin_kv8_attention_bruteforce, pin_kv8_cache_write,
            pin_kv8_blocks_attention_bruteforce, pin_kv8_blocks_cache_write]
