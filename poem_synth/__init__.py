"""Seeded synthetic inputs for POEM block-sparse attention prefill.

This module only draws inputs.  It holds none of the method's arithmetic
(no softmax, no block statistics, no selection), so both the CUDA library's
tests and the fp64 oracle can take their inputs from it.

Everything is drawn on the CPU from ``torch.Generator().manual_seed(seed)`` in
a fixed order, so a (recipe, seed) pair always yields the same bytes.

Recipes (the layer shapes come from the method's evaluation models; the value
distributions are synthetic stand-ins for the long-context prefill workloads,
which need model weights and datasets that are not used here):

* ``single_head``: one head, N tokens, head dim 64; Q, K, V i.i.d. N(0, 1) in
  fp32, then K scaled by 2 so that the scaled logits q.k/sqrt(64) have
  standard deviation 2.
* ``heavy_block_layer``: a GQA layer (e.g. 32/8 heads, d = 128).  Z ~ N(0, 1)
  for Q, K, V.  Per KV head g: a unit direction u_g on the 8 lowest-frequency
  rotary pairs (16 dims), a heavy-block set (each key block independently with
  probability 0.1) and a strength beta_g ~ U[4, 6].  Every query head of the
  group gets + a u_g and every key in a heavy block + a u_g with
  a^2 = beta_g sqrt(d), which adds about beta_g to the scaled logit of heavy
  keys.  Rotary embedding (rotate-half pairing, given base, no frequency
  rescaling) is applied to Q and K.  V = Z_v + mu[g, block], with
  mu ~ N(0, 0.5^2) per (KV head, block, dim).  Converted to bf16.
* ``contrast_layer``: the heavy-block layer's Q and K (same draws), but
  value offsets chosen so that block mass and block deviation disagree: no
  offset on ordinary blocks; a fraction ``flat_frac`` of the heavy blocks keep
  no offset (high mass, value near the dense output); the other heavy blocks,
  taken in id order, form pairs with opposite offsets +c w, -c w (w a random
  unit vector per pair, c = ``pair_offset``), whose deviations cancel in the
  output; ordinary blocks are "deviant" with probability ``deviant_prob`` and
  get an offset of norm ``deviant_offset`` along a random unit vector.
* ``iid_layer``: Q, K, V i.i.d. N(0, 1), converted to bf16.
* ``random_block_lists``: per (head, tile i) the mandatory sink and diagonal
  blocks {0, i}, then blocks drawn uniformly without replacement from
  {1 .. i-1} up to max(|mandatory|, round(density * (i + 1))) blocks in total.
"""
from __future__ import annotations

import hashlib
import math

import numpy as np
import torch


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """Raw bf16 bit patterns of a bf16 tensor, as a uint16 numpy array."""
    assert t.dtype == torch.bfloat16
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def to_f64(t: torch.Tensor) -> np.ndarray:
    return t.to(torch.float64).contiguous().numpy()


def digest(*tensors: torch.Tensor) -> str:
    """SHA-256 over the raw bytes of the given tensors (generator drift check)."""
    h = hashlib.sha256()
    for t in tensors:
        a = t.contiguous()
        if a.dtype == torch.bfloat16:
            a = a.view(torch.int16)
        h.update(a.numpy().tobytes())
    return h.hexdigest()


def single_head(n_tokens: int = 1024, head_dim: int = 64, seed: int = 0, k_gain: float = 2.0):
    """Single-head fp32 recipe: returns dict(q, k, v) of shape [N, 1, d] fp32."""
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(n_tokens, 1, head_dim, generator=g, dtype=torch.float32)
    k = torch.randn(n_tokens, 1, head_dim, generator=g, dtype=torch.float32) * k_gain
    v = torch.randn(n_tokens, 1, head_dim, generator=g, dtype=torch.float32)
    return {"q": q, "k": k, "v": v}


def _rope_tables(n_tokens: int, head_dim: int, base: float):
    half = head_dim // 2
    inv = base ** (-(torch.arange(half, dtype=torch.float64) * 2.0 / head_dim))
    ang = torch.arange(n_tokens, dtype=torch.float64)[:, None] * inv[None, :]
    return torch.cos(ang).to(torch.float32), torch.sin(ang).to(torch.float32)


def _apply_rope_(x: torch.Tensor, cos: torch.Tensor, sin: torch.Tensor, chunk: int = 8192):
    """In-place rotate-half rotary embedding of x [N, H, d] (fp32)."""
    n, _, d = x.shape
    half = d // 2
    for s in range(0, n, chunk):
        e = min(n, s + chunk)
        c = cos[s:e, None, :]
        si = sin[s:e, None, :]
        x1 = x[s:e, :, :half].clone()
        x2 = x[s:e, :, half:].clone()
        x[s:e, :, :half] = x1 * c - x2 * si
        x[s:e, :, half:] = x2 * c + x1 * si


def heavy_block_layer(n_tokens: int, n_q_heads: int = 32, n_kv_heads: int = 8, head_dim: int = 128,
                      block: int = 128, rope_base: float = 500000.0, seed: int = 0,
                      heavy_prob: float = 0.1, beta_range=(4.0, 6.0), mu_std: float = 0.5,
                      n_dir_pairs: int = 8):
    """Heavy-block GQA recipe (module docstring).  Returns dict with bf16
    q [N, Hq, d], k, v [N, Hkv, d] and the drawn structure (heavy mask, beta)."""
    assert n_tokens % block == 0 and n_q_heads % n_kv_heads == 0 and head_dim % 2 == 0
    g = torch.Generator().manual_seed(seed)
    T = n_tokens // block
    G = n_q_heads // n_kv_heads
    half = head_dim // 2
    q = torch.randn(n_tokens, n_q_heads, head_dim, generator=g, dtype=torch.float32)
    k = torch.randn(n_tokens, n_kv_heads, head_dim, generator=g, dtype=torch.float32)
    v = torch.randn(n_tokens, n_kv_heads, head_dim, generator=g, dtype=torch.float32)
    # Per KV head direction on the lowest-frequency rotary pairs (largest pair index).
    pairs = torch.arange(half - n_dir_pairs, half)
    dims = torch.cat([pairs, pairs + half])
    u = torch.zeros(n_kv_heads, head_dim, dtype=torch.float32)
    comp = torch.randn(n_kv_heads, dims.numel(), generator=g, dtype=torch.float32)
    comp = comp / comp.norm(dim=1, keepdim=True)
    u[:, dims] = comp
    heavy = torch.rand(n_kv_heads, T, generator=g) < heavy_prob
    beta = beta_range[0] + (beta_range[1] - beta_range[0]) * torch.rand(n_kv_heads, generator=g)
    mu = torch.randn(n_kv_heads, T, head_dim, generator=g, dtype=torch.float32) * mu_std
    a = torch.sqrt(beta * math.sqrt(head_dim))  # a^2 = beta * sqrt(d)
    for gi in range(n_kv_heads):
        shift = (a[gi] * u[gi]).to(torch.float32)
        q[:, gi * G:(gi + 1) * G, :] += shift
        tok = heavy[gi].repeat_interleave(block)
        k[tok, gi, :] += shift
        v[:, gi, :] += mu[gi].repeat_interleave(block, dim=0)
    cos, sin = _rope_tables(n_tokens, head_dim, rope_base)
    _apply_rope_(q, cos, sin)
    _apply_rope_(k, cos, sin)
    return {
        "q": q.to(torch.bfloat16),
        "k": k.to(torch.bfloat16),
        "v": v.to(torch.bfloat16),
        "heavy": heavy,
        "beta": beta,
    }


def contrast_layer(n_tokens: int, n_q_heads: int = 32, n_kv_heads: int = 8, head_dim: int = 128,
                   block: int = 128, rope_base: float = 500000.0, seed: int = 0, heavy_prob: float = 0.1,
                   beta_range=(4.0, 6.0), flat_frac: float = 0.5, pair_offset: float = 3.0,
                   deviant_prob: float = 0.05, deviant_offset: float = 6.0):
    """Mass/deviation contrast recipe (module docstring).  Q and K are those of
    heavy_block_layer with the same arguments; returns dict with bf16 q, k, v and
    the drawn structure (heavy, flat, pair_sign, deviant masks)."""
    x = heavy_block_layer(n_tokens, n_q_heads, n_kv_heads, head_dim, block=block, rope_base=rope_base, seed=seed,
                          heavy_prob=heavy_prob, beta_range=beta_range)
    g = torch.Generator().manual_seed(seed + 7919)
    T = n_tokens // block
    heavy = x["heavy"]
    v = torch.randn(n_tokens, n_kv_heads, head_dim, generator=g, dtype=torch.float32)
    flat = torch.zeros(n_kv_heads, T, dtype=torch.bool)
    sign = torch.zeros(n_kv_heads, T, dtype=torch.int8)
    deviant = torch.zeros(n_kv_heads, T, dtype=torch.bool)
    mu = torch.zeros(n_kv_heads, T, head_dim, dtype=torch.float32)
    for gi in range(n_kv_heads):
        hb = torch.nonzero(heavy[gi]).flatten()
        keep_flat = torch.rand(hb.numel(), generator=g) < flat_frac
        flat[gi, hb[keep_flat]] = True
        paired = hb[~keep_flat]
        for a in range(0, paired.numel() - 1, 2):
            w = torch.randn(head_dim, generator=g)
            w = w / w.norm()
            mu[gi, paired[a]] = pair_offset * w
            mu[gi, paired[a + 1]] = -pair_offset * w
            sign[gi, paired[a]] = 1
            sign[gi, paired[a + 1]] = -1
        light = torch.nonzero(~heavy[gi]).flatten()
        dv = light[torch.rand(light.numel(), generator=g) < deviant_prob]
        for b in dv.tolist():
            w = torch.randn(head_dim, generator=g)
            mu[gi, b] = deviant_offset * w / w.norm()
        deviant[gi, dv] = True
        v[:, gi, :] += mu[gi].repeat_interleave(block, dim=0)
    return {"q": x["q"], "k": x["k"], "v": v.to(torch.bfloat16), "heavy": heavy, "flat": flat,
            "pair_sign": sign, "deviant": deviant}


def iid_layer(n_tokens: int, n_q_heads: int = 32, n_kv_heads: int = 8, head_dim: int = 128, seed: int = 0):
    """Q, K, V i.i.d. N(0, 1) in bf16."""
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(n_tokens, n_q_heads, head_dim, generator=g, dtype=torch.float32).to(torch.bfloat16)
    k = torch.randn(n_tokens, n_kv_heads, head_dim, generator=g, dtype=torch.float32).to(torch.bfloat16)
    v = torch.randn(n_tokens, n_kv_heads, head_dim, generator=g, dtype=torch.float32).to(torch.bfloat16)
    return {"q": q, "k": k, "v": v}


def random_block_lists(n_q_heads: int, n_tiles: int, density: float, seed: int = 0,
                       local_block: bool = False):
    """CSR block lists (row r = h * n_tiles + i) with ascending ids.

    Mandatory: {0, i} (plus i-1 when ``local_block``).  The rest are drawn
    uniformly without replacement from the other causal blocks until the row
    holds max(|mandatory|, round(density * (i + 1))) blocks."""
    rng = np.random.Generator(np.random.PCG64(seed))
    counts = np.zeros(n_q_heads * n_tiles, dtype=np.int64)
    lists = []
    for h in range(n_q_heads):
        for i in range(n_tiles):
            mand = [0] if i == 0 else [0, i]
            if local_block and i >= 2:
                mand = [0, i - 1, i]
            hi = i - 1 if (local_block and i >= 2) else i  # pool: 1 .. hi-1
            pool = np.arange(1, max(hi, 1), dtype=np.int64)
            total = max(len(mand), int(round(density * (i + 1))))
            extra = min(total - len(mand), pool.size)
            pick = rng.choice(pool, size=extra, replace=False) if extra > 0 else np.zeros(0, np.int64)
            row = np.sort(np.concatenate([np.array(mand, dtype=np.int64), pick]))
            lists.append(row)
            counts[h * n_tiles + i] = row.size
    row_ptr = np.zeros(n_q_heads * n_tiles + 1, dtype=np.int32)
    row_ptr[1:] = np.cumsum(counts)
    col_idx = np.concatenate(lists).astype(np.int32)
    return row_ptr, col_idx
