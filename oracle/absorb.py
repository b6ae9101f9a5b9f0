"""fp64 oracle for the absorbed projections around the decode path: TEST
INFRASTRUCTURE (imported only by tests/ and bench.py's reference legs).

GQLA technical summary (gist.science, pt, 2605.15250), "Caminho MQA-Absorvido":
the up-projections are absorbed into the query and output projections, so
every head attends to the compact latent cache directly.  For one head h
with query part q_nope_h (128) and the head's up-projections W_UK_h (128 x 512,
keys) and W_UV_h (512 x 128, values):

  q_lat_h = q_nope_h . W_UK_h          (the latent query, 512 wide; the score
                                        q_lat_h . c equals q_nope_h . (W_UK_h c)
                                        for a latent row c)
  out_h   = O_h . W_UV_h               (O_h: the 512-wide attention output over
                                        latent rows; out_h the head's 128-wide
                                        value-space output)

Both are a per-head matrix product, written with numpy in fp64 (bf16 inputs are
converted exactly).
"""
from __future__ import annotations

import numpy as np
import torch


def _f64(x):
    if isinstance(x, torch.Tensor):
        return x.detach().cpu().double().numpy()
    return np.asarray(x, dtype=np.float64)


def absorb_q(q_in, w_uk, d_nope: int = 128):
    """q_in [T, h, d_nope + d_rope] (the head's group part then its RoPE part),
    w_uk [h, d_nope, 512]  ->  q [T, h, 512 + d_rope]: the latent query
    q_nope . W_UK followed by the unchanged RoPE part."""
    q = _f64(q_in)
    w = _f64(w_uk)
    lat = np.einsum("thk,hkn->thn", q[..., :d_nope], w)
    return np.concatenate([lat, q[..., d_nope:]], axis=-1)


def absorb_o(o, w_uv):
    """o [T, h, 512], w_uv [h, 512, d_out]  ->  [T, h, d_out] = O . W_UV per head."""
    return np.einsum("thk,hkn->thn", _f64(o), _f64(w_uv))
