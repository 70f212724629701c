"""Runs a workload step by step on the GPU (through the C ABI) and in the oracle.

Both sides start from the same seeded pools and follow the same plan: copy
blocks, write the new tokens, attend. The GPU side uses only the binding of
libpa_b200; the oracle side uses only ``oracle``.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
import paged_kv_cache_372_b200 as pa
from tests.bruteforce import bits_of

TOL = {"f16": 2e-3, "bf16": 1e-2}


def to_gpu(wl):
    return wl.k_pool.cuda(), wl.v_pool.cuda()


def gpu_step(wl, step, kp, vp, partition_size=None, workspace=None):
    st = wl.steps[step]
    dev = kp.device
    if len(st.copy_pairs):
        pa.pa_copy_blocks([kp, vp], torch.from_numpy(st.copy_pairs).to(dev))
    pa.pa_reshape_and_cache(st.k_new.to(dev), st.v_new.to(dev), kp, vp,
                            torch.from_numpy(st.slot_mapping).to(dev))
    q = st.q.to(dev)
    out = torch.full_like(q, float("nan"))  # every row must be written
    P = wl.partition_size if partition_size is None else partition_size
    pa.pa_decode(out, q, kp, vp, torch.from_numpy(st.block_tables).to(dev),
                 torch.from_numpy(st.context_lens).to(dev), wl.scale,
                 int(st.context_lens.max()), P, workspace)
    return out


def oracle_state(wl):
    return bits_of(wl.k_pool).copy(), bits_of(wl.v_pool).copy()


def oracle_step(wl, step, kp, vp, threads=0):
    st = wl.steps[step]
    if len(st.copy_pairs):
        oracle.copy_blocks([kp, vp], st.copy_pairs, wl.block_bytes)
    oracle.reshape_and_cache(bits_of(st.k_new), bits_of(st.v_new), kp, vp, st.slot_mapping)
    return oracle.paged_attention(bits_of(st.q), kp, vp, st.block_tables, st.context_lens,
                                  wl.scale, wl.dtype, threads)


def max_err(gpu_out: torch.Tensor, ref: np.ndarray) -> float:
    g = gpu_out.float().cpu().double().numpy()
    assert np.isfinite(g).all(), "non-finite GPU output"
    return float(np.abs(g - ref).max())


def pools_equal(kp_gpu, vp_gpu, kp_ref, vp_ref) -> bool:
    return (np.array_equal(bits_of(kp_gpu.cpu()), kp_ref)
            and np.array_equal(bits_of(vp_gpu.cpu()), vp_ref))


def gpu_step_fused(wl, step, kp, vp, partition_size=None, workspace=None):
    """The same step with the fused append + decode entry point: copies, then
    any extra (prefill) tokens through pa_reshape_and_cache, then
    pa_decode_append for each sequence's new token."""
    st = wl.steps[step]
    dev = kp.device
    B = st.q.shape[0]
    bs = wl.block_size
    for s in range(B):  # the workloads append each sequence's token at its last position
        n = int(st.context_lens[s])
        assert st.slot_mapping[s] == st.block_tables[s, (n - 1) // bs] * bs + (n - 1) % bs
    if len(st.copy_pairs):
        pa.pa_copy_blocks([kp, vp], torch.from_numpy(st.copy_pairs).to(dev))
    if len(st.slot_mapping) > B:
        pa.pa_reshape_and_cache(st.k_new[B:].to(dev), st.v_new[B:].to(dev), kp, vp,
                                torch.from_numpy(st.slot_mapping[B:]).to(dev))
    q = st.q.to(dev)
    out = torch.full_like(q, float("nan"))  # every row must be written
    P = wl.partition_size if partition_size is None else partition_size
    pa.pa_decode_append(out, q, st.k_new[:B].contiguous().to(dev), st.v_new[:B].contiguous().to(dev), kp, vp,
                        torch.from_numpy(st.block_tables).to(dev), torch.from_numpy(st.context_lens).to(dev),
                        wl.scale, int(st.context_lens.max()), P, workspace)
    return out


def gpu_step_shared(wl, step, kp, vp, partition_size=None, workspace=None, fused=True):
    """The same step through pa_decode_shared: copies, extra tokens, then the
    shared-prefix decode, appending each sequence's new token (fused) or with
    every new token written by pa_reshape_and_cache first."""
    st = wl.steps[step]
    dev = kp.device
    B = st.q.shape[0]
    if len(st.copy_pairs):
        pa.pa_copy_blocks([kp, vp], torch.from_numpy(st.copy_pairs).to(dev))
    first = B if fused else 0
    if len(st.slot_mapping) > first:
        pa.pa_reshape_and_cache(st.k_new[first:].to(dev), st.v_new[first:].to(dev), kp, vp,
                                torch.from_numpy(st.slot_mapping[first:]).to(dev))
    q = st.q.to(dev)
    out = torch.full_like(q, float("nan"))  # every row must be written
    P = wl.partition_size if partition_size is None else partition_size
    kw = {}
    if fused:
        kw = dict(k_new=st.k_new[:B].contiguous().to(dev), v_new=st.v_new[:B].contiguous().to(dev))
    pa.pa_decode_shared(out, q, kp, vp, torch.from_numpy(st.block_tables).to(dev),
                        torch.from_numpy(st.context_lens).to(dev), wl.scale, int(st.context_lens.max()), P,
                        workspace, **kw)
    return out
