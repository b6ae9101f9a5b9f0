"""B200-native (sm_100a) absorbed-MQA MLA decode in the transposed order.

The product is the C-ABI library ``libmla_decode.so`` (include/mla_decode.h):
``mla_decode_get_schedule`` (split-KV plan), ``mla_decode_fwd`` (persistent
TMA + tcgen05 decode kernel, then the LSE combine) and
``mla_decode_combine``.  ``binding`` is its ctypes binding; ``workloads``
holds the seeded synthetic inputs.  Importing this package does not load the
library: the first call does, and raises if it has not been built.
"""
from .binding import (  # noqa: F401
    MlaDecoder,
    MlaDecodeError,
    make_dims,
    mla_decode,
    mla_decode_combine,
    mla_decode_fwd,
    mla_decode_fwd_noalloc,
    mla_decode_get_schedule,
    mla_decode_get_schedule_host,
    mla_decode_get_status,
    mla_decode_schedule_bytes,
    mla_decode_strerror,
    mla_decode_version,
    mla_decode_workspace_bytes,
)
