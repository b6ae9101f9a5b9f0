"""B200-native (sm_100a) absorbed-MQA MLA decode in the transposed order.

The product is the C-ABI library ``libmla_decode.so`` (include/mla_decode.h):
``mla_decode_get_schedule`` (split-KV plan), ``mla_decode_fwd`` (persistent
TMA + tcgen05 decode kernel, then the LSE combine), ``mla_decode_combine``,
the GQA path over a group-expanded cache (``mla_gqa_decode_*``), the absorbed
projections around the decode (``mla_absorb_q`` / ``mla_absorb_o``) and the
merge of per-rank results for split-KV across GPUs
(``mla_decode_combine_ranks``; ``kv_split`` holds the page split and the
exchange).  ``binding`` is the ctypes binding; ``workloads`` holds the seeded
synthetic inputs.  Importing this package does not load the library: the
first call does, and raises if it has not been built.
"""
from .binding import (  # noqa: F401
    GqaDecoder,
    MlaDecoder,
    MlaDecodeError,
    absorb_o,
    absorb_q,
    make_absorb_dims,
    make_dims,
    make_gqa_dims,
    mla_absorb_o,
    mla_absorb_q,
    mla_decode,
    mla_decode_combine,
    mla_decode_combine_ranks,
    mla_decode_fwd,
    mla_decode_fwd_noalloc,
    mla_decode_get_schedule,
    mla_decode_get_schedule_host,
    mla_decode_get_status,
    mla_decode_schedule_bytes,
    mla_decode_strerror,
    mla_decode_version,
    mla_decode_workspace_bytes,
    mla_gqa_decode_combine,
    mla_gqa_decode_fwd,
    mla_gqa_decode_get_schedule,
    mla_gqa_decode_get_schedule_host,
    mla_gqa_decode_schedule_bytes,
    mla_gqa_decode_workspace_bytes,
)
