"""B200-native (sm_100a) per-rank hot path of context-parallel attention.

* ``fwd``       non-causal attention with LSE (tcgen05 / TMEM / TMA kernel for bf16)
* ``merge``     exact (O, LSE) merge of two key-chunk partials (Ring Attention step)
* ``seq2head``  Ulysses sequence shards -> head groups over P virtual ranks
* ``head2seq``  the inverse permute
* ``ring_attention`` / ``ulysses_attention``  the two per-rank compositions
* ``UlyssesHostPass``  a whole Ulysses layer from host shards to host O/LSE, copies
  pipelined with the attention inside the library (cpattn_ulysses_host)

All compute runs in ``libcpattn.so`` (C ABI in ``include/cpattn.h``); this package only
marshals arguments.  ``workloads`` holds the seeded synthetic inputs.
"""

from ._binding import (  # noqa: F401
    BF16,
    F32,
    CpattnError,
    device_error,
    fwd,
    fwd_accumulate,
    fwd_split,
    split_suggest,
    split_workspace_bytes,
    ulysses_fwd,
    ulysses_fwd_split,
    ulysses_workspace_bytes,
    ulysses_host,
    head2seq,
    lib,
    library_path,
    merge,
    rmsnorm,
    selftest_exp2,
    selftest_wait_timeout,
    seq2head,
    seq2head_qkv,
    seq2head_qkv_norm,
    status_str,
    version,
)
from .paths import (  # noqa: F401
    UlyssesHostPass,
    UlyssesPlan,
    UlyssesStreamer,
    ring_attention,
    ulysses_attention,
)
