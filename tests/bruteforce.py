"""Independent checks for the oracle (never used on the product path).

``contiguous_attention`` rebuilds each sequence's contiguous K/V cache (the
per-request layout that paging replaces, "别再让GPU内存拖后腿了..." section 1,
NaiveKVCache) with a numpy gather, then takes softmax(scale * q K^T) V with
numpy matmuls. It shares no code with the C oracle: element decoding here goes
through numpy's own float16 / float32 types.
"""
from __future__ import annotations

import numpy as np
import torch


def decode(bits: np.ndarray, dtype: str) -> np.ndarray:
    """16-bit patterns -> float64 through numpy's types (not the oracle's decoder)."""
    bits = np.asarray(bits, dtype=np.uint16)
    if dtype in ("f16", "fp16", "float16"):
        return bits.view(np.float16).astype(np.float64)
    with np.errstate(invalid="ignore"):
        return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def bits_of(t: torch.Tensor) -> np.ndarray:
    """Raw 16-bit patterns of a CPU fp16/bf16 tensor."""
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def contiguous_attention(q, k_pool, v_pool, block_tables, context_lens, scale):
    """All float64 arrays. Returns out [B][H][D]."""
    B, H, D = q.shape
    NB, Hkv, bs, _ = k_pool.shape
    G = H // Hkv
    out = np.zeros((B, H, D), dtype=np.float64)
    for s in range(B):
        n = int(context_lens[s])
        if n == 0:
            continue
        pos = np.arange(n)
        blocks = np.asarray(block_tables[s])[pos // bs]
        K = k_pool[blocks, :, pos % bs, :]          # [n][Hkv][D] contiguous cache
        V = v_pool[blocks, :, pos % bs, :]
        for h in range(H):
            x = scale * (K[:, h // G, :] @ q[s, h])
            w = np.exp(x - x.max())
            out[s, h] = (w / w.sum()) @ V[:, h // G, :]
    return out


def sdpa_attention(q, k_pool, v_pool, block_tables, context_lens, scale):
    """The same result through torch's scaled_dot_product_attention in fp64 (CPU),
    with each KV head repeated over its query-head group."""
    B, H, D = q.shape
    NB, Hkv, bs, _ = k_pool.shape
    G = H // Hkv
    out = np.zeros((B, H, D), dtype=np.float64)
    for s in range(B):
        n = int(context_lens[s])
        if n == 0:
            continue
        idx = [(int(block_tables[s][t // bs]), t % bs) for t in range(n)]
        K = torch.from_numpy(np.stack([k_pool[b, :, o, :] for b, o in idx], axis=1))  # [Hkv][n][D]
        V = torch.from_numpy(np.stack([v_pool[b, :, o, :] for b, o in idx], axis=1))
        K = K.repeat_interleave(G, dim=0).unsqueeze(0)
        V = V.repeat_interleave(G, dim=0).unsqueeze(0)
        qq = torch.from_numpy(q[s]).reshape(1, H, 1, D)
        o = torch.nn.functional.scaled_dot_product_attention(qq, K, V, scale=scale)
        out[s] = o.reshape(H, D).numpy()
    return out
