"""Seeded synthetic inputs shaped like the workloads on the TurboQuant pages.

This module holds input generation only, none of the quantizer's arithmetic.
Both the CUDA path (tests, bench) and the oracle are fed from here.

Recipes (the pages name Llama-3.1-8B KV caches and OpenAI-3 embedding search,
which are not available; these synthetic tensors stand in for them):

* ``gaussian_rows(n, d, norm_range=(0.5, 2))``: rows with iid N(0,1) direction
  rescaled to a norm drawn from U[lo, hi]; with ``norm_range=None`` the raw
  Gaussian rows; with ``unit=True`` L2-normalised rows (embedding search).
* ``kv_keys(heads, tokens, dim)``: bf16 keys with iid N(0,1) entries and, per
  head, ``outliers`` distinct channels (drawn from the seed) multiplied by
  ``outlier_scale`` before the round to bf16 (round-to-nearest-even).
* ``kv_queries(q_heads, kv_heads, dim)``: bf16 decode queries, one token per
  query head, with the outlier channels of their KV head (GQA grouping
  q_head -> q_head // (q_heads // kv_heads)).

Every generator takes ``seed`` and ``device``; the values depend on both
(torch uses different generators on CPU and CUDA), so a comparison between
two implementations must draw its inputs once and hand the same tensor to
both.
"""
import torch


def _gen(seed, device):
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def gaussian_rows(n, d, seed=1, device="cpu", norm_range=(0.5, 2.0), unit=False,
                  dtype=torch.float32):
    g = _gen(seed, device)
    x = torch.randn(n, d, generator=g, device=device, dtype=torch.float32)
    if unit or norm_range is not None:
        x = x / x.norm(dim=1, keepdim=True).clamp_min(1e-30)
    if not unit and norm_range is not None:
        lo, hi = norm_range
        s = torch.rand(n, 1, generator=g, device=device, dtype=torch.float32) * (hi - lo) + lo
        x = x * s
    return x.to(dtype)


def outlier_channels(heads, dim, seed=1, outliers=4):
    """Per-head outlier channel indices, [heads, outliers] int64 (CPU)."""
    g = _gen(int(seed) + 7919, "cpu")
    return torch.stack([torch.randperm(dim, generator=g)[:outliers] for _ in range(heads)])


def kv_keys(heads, tokens, dim, seed=1, device="cpu", outliers=4, outlier_scale=20.0):
    """Keys [heads, tokens, dim] bf16 (batch 1 folded away)."""
    g = _gen(seed, device)
    k = torch.randn(heads, tokens, dim, generator=g, device=device, dtype=torch.float32)
    ch = outlier_channels(heads, dim, seed, outliers).to(device)
    for h in range(heads):
        k[h][:, ch[h]] *= outlier_scale
    return k.to(torch.bfloat16)


def kv_queries(q_heads, kv_heads, dim, seed=2, device="cpu", outliers=4, outlier_scale=20.0,
               key_seed=1):
    """Decode queries [kv_heads, q_heads // kv_heads, dim] bf16, grouped by KV head."""
    g = _gen(seed, device)
    per = q_heads // kv_heads
    q = torch.randn(kv_heads, per, dim, generator=g, device=device, dtype=torch.float32)
    ch = outlier_channels(kv_heads, dim, key_seed, outliers).to(device)
    for h in range(kv_heads):
        q[h][:, ch[h]] *= outlier_scale
    return q.to(torch.bfloat16)


def sample_rows(n, count, seed=3):
    """A sorted seeded sample of row indices in [0, n) (CPU int64)."""
    g = _gen(seed, "cpu")
    count = min(count, n)
    return torch.randperm(n, generator=g)[:count].sort().values


def random_records(n, words, seed=11, norm_range=(0.5, 2.0), rnorm_range=(0.0, 0.5)):
    """Uniformly random code records for search tests that need no encoder:
    `words` uint32 words per record (every bit pattern is a valid record of
    the packed layouts), plus per-record norms.  Returns (codes [n, words]
    uint32 numpy, xnorm [n] fp32, rnorm [n] fp32) on the CPU."""
    import numpy as np
    g = _gen(seed, "cpu")
    w = np.empty((n, words), dtype=np.uint32)
    step = max(1, (1 << 22) // max(words, 1))  # rows per draw (bounded host memory)
    for r0 in range(0, n, step):
        r1 = min(n, r0 + step)
        w[r0:r1] = torch.randint(0, 1 << 32, (r1 - r0, words), generator=g,
                                 dtype=torch.int64).numpy().astype(np.uint32)
    lo, hi = norm_range
    xn = torch.rand(n, generator=g) * (hi - lo) + lo
    rlo, rhi = rnorm_range
    rn = torch.rand(n, generator=g) * (rhi - rlo) + rlo
    return w, xn.numpy().astype("float32"), rn.numpy().astype("float32")
