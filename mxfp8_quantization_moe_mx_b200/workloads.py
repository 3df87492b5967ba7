"""Seeded synthetic inputs for the quantization path (shared by tests, smoke and bench).

This module only draws random numbers and assembles tensors; it contains none of the
method's arithmetic (no block maxima, no scales, no E4M3/E8M0 encoding).  Every
tensor comes back as a contiguous CPU ``torch.bfloat16`` tensor (or int32 offsets),
generated with ``torch.Generator`` seeded explicitly, so the same seed gives the
same bytes on any machine with this torch build.

Shapes and value mixes follow the workloads the source pages measure:
  * the Llama4 debug configuration on the torchtitan mxfp8 all-to-all page
    ("[mxfp8 MoE training] Support mxfp8 all to all in expert parallel",
    Performance): dim 5120, seq_len 8192, local batch 8, 16 experts, so the
    dispatch payload is (8 * 8192, 5120) bf16 tokens;
  * the per-group rowwise scaling tables on the torchao page ("[moe training] fix
    uncoalesced global accesses in per group rowwise scaling kernel",
    Performance): input (16640, 5120) bf16 with 16, 32, 64 or 128 groups.
Value distributions (lognormal row/feature scales, outliers, subnormals, values at
and above the E4M3 maximum, all-zero blocks, empty and Zipf-sized groups) are the
recipe written down in the repository's design notes; the pages print no values.
"""
from __future__ import annotations

import torch

# Seeds: config i uses SEED_BASE + i.
SEED_BASE = 1000


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator()
    g.manual_seed(int(seed))
    return g


def _bf16(x: torch.Tensor) -> torch.Tensor:
    return x.to(torch.bfloat16).contiguous()


def uniform_group_offsets(g: torch.Generator, M: int, G: int) -> torch.Tensor:
    """Exclusive end offsets of G contiguous groups whose sizes are a multinomial
    draw of M tokens over G equally likely experts."""
    pick = torch.randint(0, G, (M,), generator=g)
    sizes = torch.bincount(pick, minlength=G)
    return torch.cumsum(sizes, 0).to(torch.int32)


def zipf_group_offsets(g: torch.Generator, M: int, G: int, n_empty: int,
                       s: float = 1.2) -> torch.Tensor:
    """G groups, n_empty of them (chosen at random) empty; the others get weights
    proportional to rank**-s (ranks assigned in random order) and sizes drawn as a
    multinomial of M tokens over those weights."""
    perm = torch.randperm(G, generator=g)
    empty = perm[:n_empty]
    live = perm[n_empty:]
    ranks = torch.randperm(live.numel(), generator=g).to(torch.float64) + 1.0
    w = ranks.pow(-s)
    pick = torch.multinomial(w, M, replacement=True, generator=g)
    live_sizes = torch.bincount(pick, minlength=live.numel())
    sizes = torch.zeros(G, dtype=torch.int64)
    sizes[live] = live_sizes
    sizes[empty] = 0
    return torch.cumsum(sizes, 0).to(torch.int32)


# ---- configuration 0: tiny correctness case -------------------------------------------

def tiny(seed: int = SEED_BASE + 0, rows: int = 256, cols: int = 512):
    """X (256, 512): N(0,1); 1% of the entries (exact count, no repeats) times 100;
    the 1x32 block at row 17, columns 64..95 set to zero.  Offsets [a, a, b, 256]
    with 1 <= a < b <= 255 drawn uniformly, so group 1 is empty."""
    g = _gen(seed)
    x = torch.randn(rows, cols, generator=g)
    n = rows * cols
    k = (n + 50) // 100
    idx = torch.randperm(n, generator=g)[:k]
    x.view(-1)[idx] *= 100.0
    x[17, 64:96] = 0.0
    ab = torch.randperm(rows - 1, generator=g)[:2] + 1
    a, b = int(ab.min()), int(ab.max())
    offs = torch.tensor([a, a, b, rows], dtype=torch.int32)
    return {"x": _bf16(x), "offs": offs}


# ---- configuration 1: MXFP8 dispatch payload --------------------------------------------

def dispatch(seed: int = SEED_BASE + 1, rows: int = 65536, cols: int = 5120,
             n_groups: int = 16):
    """Tokens (local batch 8 x seq 8192, dim 5120): N(0,1) rows times a per-row
    lognormal(0,1) scale, and about 0.1% of the entries (drawn with replacement)
    times 100.  ``offs`` splits the tokens over ``n_groups`` experts with
    multinomial-uniform sizes, for the per-group step on the received tokens."""
    g = _gen(seed)
    x = torch.randn(rows, cols, generator=g)
    x *= torch.exp(torch.randn(rows, 1, generator=g))
    n = rows * cols
    idx = torch.randint(0, n, (max(1, n // 1000),), generator=g)
    x.view(-1)[idx] *= 100.0
    offs = uniform_group_offsets(g, rows, n_groups)
    return {"x": _bf16(x), "offs": offs}


# ---- configuration 2: per-group rowwise FP8 scaling ---------------------------------------

def per_group(seed: int = SEED_BASE + 2, M: int = 16640, K: int = 5120, n_groups: int = 16):
    """X (16640, 5120): N(0,1) times a per-feature lognormal(0,1) scale; group sizes
    multinomial-uniform over the M tokens."""
    g = _gen(seed)
    x = torch.randn(M, K, generator=g)
    x *= torch.exp(torch.randn(1, K, generator=g))
    offs = uniform_group_offsets(g, M, n_groups)
    return {"x": _bf16(x), "offs": offs}


# ---- configuration 3: dual-axis MXFP8 for the backward pass ----------------------------------

def dual_axis(seed: int = SEED_BASE + 3, act_rows: int = 16384, dim: int = 5120,
              experts: int = 16, hidden: int = 8192):
    """Activations (16384, 5120) and expert weights (16, 8192, 5120), both N(0, 0.02^2)."""
    g = _gen(seed)
    act = torch.randn(act_rows, dim, generator=g) * 0.02
    w = torch.randn(experts, hidden, dim, generator=g) * 0.02
    return {"act": _bf16(act), "w": _bf16(w)}


# ---- configuration 4: stress mix -------------------------------------------------------------

def stress(seed: int = SEED_BASE + 4, M: int = 131072, K: int = 5120, n_groups: int = 128,
           n_empty: int = 20):
    """X (131072, 5120) built per 1x32 block; each block draws a category:
         55%  N(0,1)
         10%  random bf16 subnormals (bit patterns 0x0001..0x007F, random sign)
         10%  N(0,1)*50 clipped to |x| <= 447, one element set to exactly +-448
         10%  N(0,1) with one element uniform in [450, 510] * 2^j, j uniform in [-4, 4]
          5%  all zero
         10%  N(0,1) times a per-block lognormal(0,1) scale
       Groups: 128, of which 20 are empty, Zipf(1.2) sizes for the rest."""
    assert K % 32 == 0
    g = _gen(seed)
    nb = M * K // 32
    x = torch.randn(nb, 32, generator=g)
    u = torch.rand(nb, generator=g)
    cat = torch.bucketize(u, torch.tensor([0.55, 0.65, 0.75, 0.85, 0.90]))
    # category 2: large values, one exactly +-448
    m2 = cat == 2
    n2 = int(m2.sum())
    blk = (x[m2] * 50.0).clamp_(-447.0, 447.0)
    pos = torch.randint(0, 32, (n2,), generator=g)
    sgn = torch.where(torch.rand(n2, generator=g) < 0.5, -1.0, 1.0)
    blk[torch.arange(n2), pos] = 448.0 * sgn
    x[m2] = blk
    # category 3: one element above the E4M3 maximum at scale 2^j
    m3 = cat == 3
    n3 = int(m3.sum())
    blk = x[m3]
    pos = torch.randint(0, 32, (n3,), generator=g)
    j = torch.randint(-4, 5, (n3,), generator=g).to(torch.float32)
    val = (450.0 + 60.0 * torch.rand(n3, generator=g)) * torch.pow(2.0, j)
    sgn = torch.where(torch.rand(n3, generator=g) < 0.5, -1.0, 1.0)
    blk[torch.arange(n3), pos] = val * sgn
    x[m3] = blk
    # category 4: all zero
    x[cat == 4] = 0.0
    # category 5: lognormal block scale
    m5 = cat == 5
    n5 = int(m5.sum())
    x[m5] = x[m5] * torch.exp(torch.randn(n5, 1, generator=g))
    xb = x.to(torch.bfloat16)
    # category 1: subnormal bit patterns, written directly as bf16 bits
    m1 = cat == 1
    n1 = int(m1.sum())
    bits = torch.randint(1, 0x80, (n1, 32), generator=g, dtype=torch.int32)
    bits |= torch.randint(0, 2, (n1, 32), generator=g, dtype=torch.int32) << 15
    xb.view(torch.int16)[m1] = bits.to(torch.int16)
    offs = zipf_group_offsets(g, M, n_groups, n_empty)
    return {"x": xb.view(M, K).contiguous(), "offs": offs}


def bf16_bits(t: torch.Tensor):
    """The uint16 bit patterns of a CPU bf16 tensor, as a numpy array (a view)."""
    import numpy as np
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)
