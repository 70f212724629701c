"""pa_decode_shared: decode that streams blocks shared by several sequences'
tables once per group of sequences.

The result must be the definition (the oracle, fp64) within the dtype's
tolerance, equal within tolerance to pa_decode / pa_decode_append on the same
inputs, deterministic, and untouched by NaN in slots no sequence covers. The
work list must also show the grouping the header describes: the number of
units is checked against a direct count from the block tables.
"""
from __future__ import annotations

import math

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_372_b200 as pa
from paged_kv_cache_372_b200 import inputs, workloads
from tests import gpu_harness as H
from tests import margins
from tests.bruteforce import bits_of

pytestmark = pytest.mark.gpu


# ------------------------------------------------------------------------------
def sharing_case(seed, heads, kv_heads, head_dim, block_size, dtype, append):
    """Sequences with shared leading blocks in several patterns, in shuffled order:
    a large group with one common prefix, nested sharing, a pair that diverges
    after its first block, (without append) identical tables, an empty
    sequence, a sequence shorter than a block, and unrelated sequences."""
    rng = np.random.default_rng(seed)
    gen = inputs.generator(seed)
    bs = block_size
    NB = 600
    order = inputs.permutation(NB, gen)
    pos = [0]

    def fresh(n):
        out = order[pos[0]:pos[0] + n]
        pos[0] += n
        assert len(out) == n
        return list(out)

    seqs = []  # (table, ctx)

    def add(table, ctx):
        assert ctx <= len(table) * bs
        seqs.append((table, ctx))

    prefix = fresh(5)
    for _ in range(12):
        suf = int(rng.integers(1, 3 * bs))
        add(prefix + fresh(-(-suf // bs)), 5 * bs + suf)
    pb, mid = fresh(3), fresh(2)
    r = int(rng.integers(1, bs))
    add(pb + mid + fresh(1), 5 * bs + r)
    add(pb + mid + fresh(2), 6 * bs + r)
    add(pb + fresh(2), 3 * bs + r + 1)
    pc = fresh(1)
    add(pc + fresh(2), bs + bs + 3)
    add(pc + fresh(1), bs + 5)
    if not append:
        same = fresh(4)
        add(list(same), 4 * bs)
        add(list(same), 4 * bs)
        add(list(same), 4 * bs - 3)
        add(prefix[:1], bs - 3)  # shares block 0 but holds no full block
    add(fresh(1), 0)
    add(fresh(1), bs - 2)
    for _ in range(5):
        n = int(rng.integers(1, 40))
        add(fresh(n), int(rng.integers((n - 1) * bs + 1, n * bs + 1)))
    perm = rng.permutation(len(seqs))
    seqs = [seqs[i] for i in perm]

    B = len(seqs)
    W = max(len(t) for t, _ in seqs)
    tables = np.full((B, W), -1, dtype=np.int32)
    for i, (t, _) in enumerate(seqs):
        tables[i, :len(t)] = t
    ctx = np.array([c for _, c in seqs], dtype=np.int32)

    kp = inputs.normal((NB, kv_heads, bs, head_dim), dtype, gen)
    vp = inputs.normal((NB, kv_heads, bs, head_dim), dtype, gen)
    # Poison every slot no sequence covers (its content must not matter).
    valid = np.zeros((NB, bs), dtype=bool)
    for (t, c) in seqs:
        for j in range(c):
            valid[t[j // bs], j % bs] = True
    bad = torch.from_numpy(~valid)[:, None, :, None].expand(NB, kv_heads, bs, head_dim)
    kp[bad] = float("nan")
    vp[bad] = float("nan")
    q = inputs.normal((B, heads, head_dim), dtype, gen)
    case = dict(kp=kp, vp=vp, q=q, tables=tables, ctx=ctx, scale=1.0 / math.sqrt(head_dim), dtype=dtype,
                seqs=seqs, bs=bs, heads=heads, kv_heads=kv_heads)
    if append:
        case["k_new"] = inputs.normal((B, kv_heads, head_dim), dtype, gen)
        case["v_new"] = inputs.normal((B, kv_heads, head_dim), dtype, gen)
        case["slots"] = np.array([t[(c - 1) // bs] * bs + (c - 1) % bs if c > 0 else -1 for t, c in seqs],
                                 dtype=np.int64)
    return case


def expected_entries(case, P, append):
    """Work-list entries (per KV head) of the grouping the header describes,
    counted directly from the tables."""
    bs, seqs = case["bs"], case["seqs"]
    cap = 16 // (case["heads"] // case["kv_heads"])

    def nfull(c):
        p = c - 1 if append else c
        return p // bs if p > 0 else 0

    keys = sorted(((t[0] if nfull(c) > 0 else 2**31 - 1), i) for i, (t, c) in enumerate(seqs))
    shared = [0] * len(seqs)
    n = 0
    i = 0
    while i < len(keys):
        j = i
        while j < len(keys) and keys[j][0] == keys[i][0]:
            j += 1
        if keys[i][0] == 2**31 - 1:
            j = i + 1
        for lead in range(i, j, cap):
            members = [keys[k][1] for k in range(lead, min(lead + cap, j))]
            if len(members) < 2:
                continue
            lt, lc = seqs[members[0]]
            sh = nfull(lc)
            for m in members[1:]:
                mt, mc = seqs[m]
                lim = min(nfull(mc), nfull(lc))
                lcp = 0
                while lcp < lim and mt[lcp] == lt[lcp]:
                    lcp += 1
                sh = min(sh, lcp)
            for m in members:
                shared[m] = sh * bs
            n += -(-sh * bs // P)
        i = j
    for k, (_, c) in enumerate(seqs):
        n += -(-(c - shared[k]) // P)
    return n, sum(1 for s in shared if s > 0)


def run_shared(case, P, append, workspace=None):
    dev = torch.device("cuda")
    kp, vp = case["kp"].to(dev), case["vp"].to(dev)
    q = case["q"].to(dev)
    out = torch.full_like(q, float("nan"))  # every row must be written
    B, H_, D = q.shape
    mx = int(case["ctx"].max())
    if workspace is None:
        workspace = pa.alloc_workspace(B, H_, case["kv_heads"], D, case["bs"], mx, P, dev, shared=True)
    kw = {}
    if append:
        kw = dict(k_new=case["k_new"].to(dev), v_new=case["v_new"].to(dev))
    pa.pa_decode_shared(out, q, kp, vp, torch.from_numpy(case["tables"]).to(dev),
                        torch.from_numpy(case["ctx"]).to(dev), case["scale"], mx, P, workspace, **kw)
    torch.cuda.synchronize()
    assert pa.pa_device_errors() == 0
    return out, kp, vp, workspace


def run_plain(case, P, append):
    dev = torch.device("cuda")
    kp, vp = case["kp"].to(dev), case["vp"].to(dev)
    q = case["q"].to(dev)
    out = torch.full_like(q, float("nan"))  # every row must be written
    mx = int(case["ctx"].max())
    tab, ctx = torch.from_numpy(case["tables"]).to(dev), torch.from_numpy(case["ctx"]).to(dev)
    if append:
        pa.pa_decode_append(out, q, case["k_new"].to(dev), case["v_new"].to(dev), kp, vp, tab, ctx,
                            case["scale"], mx, P)
    else:
        pa.pa_decode(out, q, kp, vp, tab, ctx, case["scale"], mx, P)
    torch.cuda.synchronize()
    assert pa.pa_device_errors() == 0
    return out, kp, vp


def run_oracle(case, append):
    kp, vp = bits_of(case["kp"]).copy(), bits_of(case["vp"]).copy()
    if append:
        oracle.reshape_and_cache(bits_of(case["k_new"]), bits_of(case["v_new"]), kp, vp, case["slots"])
    ref = oracle.paged_attention(bits_of(case["q"]), kp, vp, case["tables"], case["ctx"], case["scale"],
                                 case["dtype"])
    return ref, kp, vp


SHAPES = [  # (heads, kv_heads, head_dim, block_size, dtype)
    (8, 8, 128, 16, "f16"),
    (8, 4, 64, 32, "bf16"),
    (16, 4, 128, 16, "bf16"),
    (16, 2, 128, 64, "f16"),
    (4, 4, 64, 64, "bf16"),
    (8, 2, 64, 16, "f16"),
]


@pytest.mark.parametrize("append", [False, True])
@pytest.mark.parametrize("shape", SHAPES)
def test_sharing_patterns_match_oracle(shape, append):
    heads, kv_heads, D, bs, dtype = shape
    case = sharing_case(7 + bs + D, heads, kv_heads, D, bs, dtype, append)
    ref, okp, ovp = run_oracle(case, append)
    for P in (0, 2 * bs):
        out, kp, vp, ws = run_shared(case, P, append)
        err = H.max_err(out, ref)
        assert err <= H.TOL[dtype], (shape, P, err)
        margins.record(f"shared {heads}/{kv_heads} D={D} bs={bs} {dtype} P={P or 'auto'}"
                       f"{' append' if append else ''}", err, H.TOL[dtype])
        if append:
            assert H.pools_equal(kp, vp, okp, ovp)
        # The plan grouped the sequences as described (units per KV head).
        Pr = pa.pa_decode_shared_partition_size(len(case["ctx"]), heads, kv_heads, D, bs, int(case["ctx"].max()), P)
        n_expect, n_shared = expected_entries(case, Pr, append)
        assert int(ws[4:8].view(torch.int32).item()) == n_expect
        assert n_shared >= 10  # sequences that share blocks do share units (G = 8 included: 2 per unit)
        # Same inputs through the plain path.
        plain, pkp, pvp = run_plain(case, P, append)
        assert float((plain.float() - out.float()).abs().max()) <= H.TOL[dtype]
        if append:
            # bitwise: unused slots hold NaN
            assert torch.equal(pkp.view(torch.int16), kp.view(torch.int16))
            assert torch.equal(pvp.view(torch.int16), vp.view(torch.int16))


def test_deterministic():
    case = sharing_case(3, 16, 4, 128, 16, "bf16", False)
    a = run_shared(case, 32, False)[0]
    b = run_shared(case, 32, False)[0]
    assert torch.equal(a, b)


@pytest.mark.parametrize("name", ["beam", "beam256"])
@pytest.mark.parametrize("fused", [True, False])
def test_beam_workloads(name, fused):
    wl = workloads.build(name, 0, steps=3)
    kp, vp = H.to_gpu(wl)
    okp, ovp = H.oracle_state(wl)
    for i in range(len(wl.steps)):
        out = H.gpu_step_shared(wl, i, kp, vp, fused=fused)
        ref = H.oracle_step(wl, i, okp, ovp)
        torch.cuda.synchronize()
        assert pa.pa_device_errors() == 0
        assert H.pools_equal(kp, vp, okp, ovp), f"pools differ after step {i}"
        err = H.max_err(out, ref)
        assert err <= H.TOL[wl.dtype]
        margins.record(f"shared {name}{' fused' if fused else ''} {wl.dtype}", err, H.TOL[wl.dtype])


def test_without_sharing_equals_plain_decode():
    """No shared blocks: every unit is an ordinary one and the partitions are
    pa_decode's, so the unnormalised partials are the same; the merges differ
    only in the order of their fp32 sums (pa_decode: in the attention kernel,
    in one level up to 8 partitions and two beyond; here: in the separate
    merge launch), so the results agree up to that rounding."""
    wl = workloads.llama3_8b(1, num_seqs=24)
    st = wl.steps[0]
    dev = torch.device("cuda")
    kp, vp = wl.k_pool.to(dev), wl.v_pool.to(dev)
    q = st.q.to(dev)
    tab = torch.from_numpy(st.block_tables).to(dev)
    for ctx_np in (np.minimum(st.context_lens, 8 * 128), st.context_lens):
        ctx = torch.from_numpy(np.ascontiguousarray(ctx_np)).to(dev)
        mx = int(ctx_np.max())
        a, b = torch.full_like(q, float("nan")), torch.full_like(q, float("nan"))
        pa.pa_decode(a, q, kp, vp, tab, ctx, wl.scale, mx, 128)
        pa.pa_decode_shared(b, q, kp, vp, tab, ctx, wl.scale, mx, 128)
        torch.cuda.synchronize()
        assert float((a.float() - b.float()).abs().max()) <= H.TOL[wl.dtype]


def test_more_sequences_than_one_grouping():
    """1100 sequences (more than the grouping plan's 1024): the call runs as two
    chunks, sharing within each, and matches the oracle and pa_decode."""
    from paged_kv_cache_372_b200 import inputs
    gen = inputs.generator(404)
    B, heads, kvh, D, bs, NB = 1100, 8, 2, 64, 16, 2400
    rng = np.random.default_rng(404)
    perm = inputs.permutation(NB, gen)
    tables = np.full((B, 3), -1, dtype=np.int32)
    ctx = np.zeros(B, dtype=np.int32)
    nxt = 0
    for i in range(0, B, 2):  # pairs with one shared full block and a private second one
        shared = perm[nxt]
        nxt += 1
        for j in (i, i + 1):
            tables[j, 0] = shared
            tables[j, 1] = perm[nxt]
            nxt += 1
            ctx[j] = bs + int(rng.integers(1, bs + 1))
    case = dict(kp=inputs.normal((NB, kvh, bs, D), "f16", gen), vp=inputs.normal((NB, kvh, bs, D), "f16", gen),
                q=inputs.normal((B, heads, D), "f16", gen), tables=tables, ctx=ctx, scale=D ** -0.5, dtype="f16",
                bs=bs, heads=heads, kv_heads=kvh)
    ref, _, _ = run_oracle(case, False)
    n0 = pa.pa_launch_count()
    out = run_shared(case, 0, False)[0]
    assert pa.pa_launch_count() - n0 == 6  # per chunk: grouping plan, attention, merge launch
    assert not torch.isnan(out).any()
    err = H.max_err(out, ref)
    assert err <= H.TOL["f16"], err
    plain = run_plain(case, 0, False)[0]
    assert float((plain.float() - out.float()).abs().max()) <= H.TOL["f16"]


def whole_unit_case(group):
    """Three sequences with identical tables whose whole 64-token context is one
    shared unit (at partitions longer than that), next to a sequence with one
    partition of its own and one with several."""
    from paged_kv_cache_372_b200 import inputs
    gen = inputs.generator(90 + group)
    bs, D, kvh = 16, 128, 2
    heads = kvh * group
    NB = 64
    tables = np.full((5, 8), -1, dtype=np.int32)
    same = [3, 17, 9, 40]
    tables[0, :4] = same
    tables[1, :4] = same
    tables[2, :4] = same
    tables[3, :2] = [5, 6]
    tables[4, :8] = [20, 21, 22, 23, 24, 25, 26, 27]
    ctx = np.array([64, 64, 64, 20, 128], dtype=np.int32)
    return dict(kp=inputs.normal((NB, kvh, bs, D), "f16", gen), vp=inputs.normal((NB, kvh, bs, D), "f16", gen),
                q=inputs.normal((5, heads, D), "f16", gen), tables=tables, ctx=ctx, scale=D ** -0.5, dtype="f16",
                bs=bs, heads=heads, kv_heads=kvh)


@pytest.mark.parametrize("group", [1, 2, 4, 8])
def test_whole_context_in_one_shared_unit(group):
    """A member whose only partial is a shared unit's still has it normalised
    into the output (by the merge launch); the sequence with one partition of
    its own is written directly."""
    case = whole_unit_case(group)
    ref, _, _ = run_oracle(case, False)
    for P in (256, 32):
        out = run_shared(case, P, False)[0]
        assert not torch.isnan(out).any()
        err = H.max_err(out, ref)
        assert err <= H.TOL["f16"], (P, err)
