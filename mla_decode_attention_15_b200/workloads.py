"""Seeded synthetic inputs for MLA decode.

This module only draws random numbers and builds paged-cache bookkeeping
(lengths, page pool, block table).  It holds none of the attention arithmetic,
so both the CUDA path and the fp64 oracle can read the tensors it builds and
see identical bits.

Shapes follow the DeepSeek-R1 decode setting of the FlashMLA-ETAP pages
(technical summary, "Resultados Experimentais" and "Limitações": 16 heads per
GPU, 576-wide rows, sequences up to 64K, batch 16/32) and the absorbed-MQA
cache of the GQLA summary ("Caminho MQA-Absorvido": a 512-wide latent plus a
64-wide shared RoPE key per token).  The page size of 64 tokens is the one the
FlashMLA-ETAP blog's integration example configures.

Draw order for one workload, all from ``torch.Generator('cpu')`` seeded with
the workload's seed:
  1. per-request lengths (only for ragged workloads);
  2. Q = randn * sigma, rounded to bf16;
  3. the page pool = randn * sigma, rounded to bf16, with
     sum_b ceil(L_b / 64) + spare pages;
  4. a random permutation of the pool's page ids, dealt row-major over
     (request, logical page) into the block table (identity table: no draw);
  5. peaked rows (only where requested): per request, max(1, floor(frac*L_b))
     distinct logical rows drawn without replacement; each whole 576-wide row
     is multiplied by 8 after bf16 rounding (exact in bf16).
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, Optional, Tuple

import torch

D_QK = 576
D_V = 512
PAGE = 64
SOFTMAX_SCALE = 192 ** -0.5

_RAGGED = Tuple[str, int, int]


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic decode batch; the fields describe shapes, not arithmetic."""
    name: str
    batch: int
    s_q: int
    heads: int
    lens: Tuple  # ("fixed", L) or ("uniform", lo, hi) inclusive
    sigma: float
    table: str  # "identity" or "permuted"
    peaked_frac: float
    causal: bool
    seed: int
    spare_pages: int = 8
    description: str = ""

    @property
    def n_cols(self) -> int:
        return self.heads * self.s_q


WORKLOADS: Dict[str, Workload] = {
    w.name: w
    for w in [
        Workload("b1_l1024_h16", 1, 1, 16, ("fixed", 1024), 1.0, "identity", 0.0, False, 1000,
                 description="batch 1, s_q 1, 16 heads, KV len 1024, identity block table"),
        Workload("b16_l4096_h16", 16, 1, 16, ("fixed", 4096), 1.0, "permuted", 0.0, False, 1001,
                 description="batch 16, s_q 1, 16 heads, KV len 4096, permuted pages"),
        Workload("b16_sq2_ragged1k16k_h16_peaked", 16, 2, 16, ("uniform", 1024, 16384), 1.0,
                 "permuted", 0.01, True, 1002,
                 description="batch 16, s_q 2 causal, 16 heads, KV len U[1024,16384], "
                             "1% of rows x8, permuted pages"),
        Workload("b16_l65536_h16", 16, 1, 16, ("fixed", 65536), 1.0, "permuted", 0.0, False, 1003,
                 description="batch 16, s_q 1, 16 heads, KV len 65536 (1.21 GB latent cache), "
                             "permuted pages"),
        Workload("b32_sq2_ragged8k32k_h128", 32, 2, 128, ("uniform", 8192, 32768), 0.5,
                 "permuted", 0.0, True, 1004,
                 description="batch 32, s_q 2 causal, 128 heads, KV len U[8192,32768], "
                             "sigma 0.5, permuted pages"),
    ]
}

HEADLINE = "b16_l65536_h16"
SMALL = "b1_l1024_h16"


def _draw_lens(spec, batch: int, g: torch.Generator) -> torch.Tensor:
    kind = spec[0]
    if kind == "fixed":
        return torch.full((batch,), int(spec[1]), dtype=torch.int32)
    if kind == "uniform":
        lo, hi = int(spec[1]), int(spec[2])
        return torch.randint(lo, hi + 1, (batch,), generator=g, dtype=torch.int64).to(torch.int32)
    if kind == "list":
        return torch.tensor(list(spec[1]), dtype=torch.int32)
    raise ValueError("unknown length spec %r" % (spec,))


def build(batch: int, s_q: int, heads: int, lens, sigma: float = 1.0, table: str = "permuted",
          peaked_frac: float = 0.0, seed: int = 0, spare_pages: int = 8,
          tail_fill: Optional[float] = None, causal: bool = False, pool_device: str = "cpu") -> dict:
    """Build one batch of decode inputs on the CPU.

    ``pool_device`` other than "cpu" draws the page pool (step 3) there, from
    a generator of that device seeded with ``seed + 1``, and leaves it there;
    for multi-GB pools (sweeps, large-offset tests), whose oracle checks read
    a host copy of it.  Every other draw stays on the CPU generator.

    ``lens`` is ("fixed", L), ("uniform", lo, hi) or ("list", [L_0, ...]).
    ``tail_fill`` (tests only) overwrites the rows past L_b in each request's
    last page with alternating +/-tail_fill, values that must not affect any
    result.

    Returns a dict of CPU tensors: q [B, s_q, h, 576] bf16, kv_cache
    [num_blocks, 64, 1, 576] bf16, block_table [B, max_pages] int32 (unused
    slots -1), cache_seqlens [B] int32, plus softmax_scale and causal.
    """
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    seqlens = _draw_lens(lens, batch, g)
    pages = [(int(L) + PAGE - 1) // PAGE for L in seqlens.tolist()]
    total_pages = sum(pages)
    max_pages = max(pages) if pages else 0
    max_pages = max(max_pages, 1)
    q = (torch.randn(batch * s_q * heads * D_QK, generator=g) * sigma).to(torch.bfloat16)
    q = q.view(batch, s_q, heads, D_QK)
    num_blocks = total_pages + spare_pages
    if pool_device == "cpu":
        kv = (torch.randn(num_blocks * PAGE * D_QK, generator=g) * sigma).to(torch.bfloat16)
    else:
        gd = torch.Generator(device=pool_device)
        gd.manual_seed(int(seed) + 1)
        kv = (torch.randn(num_blocks * PAGE * D_QK, generator=gd, device=pool_device) * sigma).to(torch.bfloat16)
    kv = kv.view(num_blocks, PAGE, 1, D_QK)
    if table == "identity":
        ids = torch.arange(num_blocks, dtype=torch.int32)
    elif table == "permuted":
        ids = torch.randperm(num_blocks, generator=g).to(torch.int32)
    else:
        raise ValueError("table must be 'identity' or 'permuted'")
    block_table = torch.full((batch, max_pages), -1, dtype=torch.int32)
    k = 0
    for b, P in enumerate(pages):
        block_table[b, :P] = ids[k:k + P]
        k += P
    if peaked_frac > 0:
        for b, L in enumerate(seqlens.tolist()):
            if L <= 0:
                continue
            n = max(1, int(math.floor(peaked_frac * L)))
            rows = torch.randperm(L, generator=g)[:n]
            for t in rows.tolist():
                phys = int(block_table[b, t // PAGE])
                kv[phys, t % PAGE] = kv[phys, t % PAGE] * 8
    if tail_fill is not None:
        for b, L in enumerate(seqlens.tolist()):
            P = pages[b]
            if P == 0 or L % PAGE == 0:
                continue
            phys = int(block_table[b, P - 1])
            n_tail = PAGE - L % PAGE
            sign = torch.ones(n_tail, 1, D_QK)
            sign[1::2] = -1
            kv[phys, L % PAGE:] = (sign * tail_fill).to(torch.bfloat16)
    return dict(q=q, kv_cache=kv, block_table=block_table, cache_seqlens=seqlens,
                softmax_scale=SOFTMAX_SCALE, causal=bool(causal))


def make_inputs(workload, seed: Optional[int] = None) -> dict:
    """Inputs for a named workload (``seed`` overrides its seed, e.g. per rank)."""
    w = WORKLOADS[workload] if isinstance(workload, str) else workload
    d = build(w.batch, w.s_q, w.heads, w.lens, sigma=w.sigma, table=w.table,
              peaked_frac=w.peaked_frac, seed=w.seed if seed is None else seed,
              spare_pages=w.spare_pages, causal=w.causal)
    d["workload"] = w
    return d


# ---------------------------------------------------------------- GQA path
GQA_D_HEAD = 128
GQA_D_ROPE = 64
GQA_HEADS_PER_GROUP = 16


def build_gqa(batch: int, s_q: int, groups: int, lens, sigma: float = 1.0, seed: int = 0,
              spare_pages: int = 8, causal: bool = False, pool_device: str = "cpu") -> dict:
    """Inputs for the GQLA GQA path: a group-expanded paged cache whose
    per-token row is K_0..K_{g-1} (128 each), V_0..V_{g-1} (128 each), then the
    shared RoPE key (64); 16 query heads per group, q = [B, s_q, 16g, 192].
    Draw order as in build(): lengths, Q, pool (on ``pool_device``), block
    table permutation.  No attention arithmetic here."""
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    seqlens = _draw_lens(lens, batch, g)
    pages = [(int(L) + PAGE - 1) // PAGE for L in seqlens.tolist()]
    max_pages = max(max(pages) if pages else 0, 1)
    h = GQA_HEADS_PER_GROUP * groups
    width = 2 * groups * GQA_D_HEAD + GQA_D_ROPE
    q = (torch.randn(batch * s_q * h * (GQA_D_HEAD + GQA_D_ROPE), generator=g) * sigma).to(torch.bfloat16)
    q = q.view(batch, s_q, h, GQA_D_HEAD + GQA_D_ROPE)
    num_blocks = sum(pages) + spare_pages
    n = num_blocks * PAGE * width
    if pool_device == "cpu":
        kv = (torch.randn(n, generator=g) * sigma).to(torch.bfloat16)
    else:
        gd = torch.Generator(device=pool_device)
        gd.manual_seed(int(seed) + 1)
        kv = (torch.randn(n, generator=gd, device=pool_device) * sigma).to(torch.bfloat16)
    kv = kv.view(num_blocks, PAGE, 1, width)
    ids = torch.randperm(num_blocks, generator=g).to(torch.int32)
    block_table = torch.full((batch, max_pages), -1, dtype=torch.int32)
    k = 0
    for b, P in enumerate(pages):
        block_table[b, :P] = ids[k:k + P]
        k += P
    return dict(q=q, kv_cache=kv, block_table=block_table, cache_seqlens=seqlens,
                softmax_scale=SOFTMAX_SCALE, causal=bool(causal), groups=groups)


ABSORB_D_NOPE, ABSORB_D_ROPE, ABSORB_D_LATENT, ABSORB_D_V_HEAD = 128, 64, 512, 128


def build_absorb(tokens: int, heads: int, seed: int = 0, sigma: float = 1.0) -> dict:
    """Inputs for the absorbed projections (GQLA summary, "Caminho
    MQA-Absorvido"), all bf16 on the CPU, drawn in this order from one CPU
    generator: q_in [T, h, 192] = randn * sigma; w_uk [h, 128, 512] = randn /
    sqrt(128); o [T, h, 512] = randn * sigma; w_uv [h, 512, 128] = randn /
    sqrt(512).  The weight scales keep the products near unit variance, as a
    trained projection's would be; the weights themselves are random."""
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))

    def draw(shape, scale):
        return (torch.randn(math.prod(shape), generator=g) * scale).to(torch.bfloat16).view(*shape)

    q_in = draw((tokens, heads, ABSORB_D_NOPE + ABSORB_D_ROPE), sigma)
    w_uk = draw((heads, ABSORB_D_NOPE, ABSORB_D_LATENT), 1.0 / math.sqrt(ABSORB_D_NOPE))
    o = draw((tokens, heads, ABSORB_D_LATENT), sigma)
    w_uv = draw((heads, ABSORB_D_LATENT, ABSORB_D_V_HEAD), 1.0 / math.sqrt(ABSORB_D_LATENT))
    return dict(q_in=q_in, w_uk=w_uk, o=o, w_uv=w_uv)
