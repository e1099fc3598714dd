"""B200-native (sm_100a) hot path of DiT denoising: joint image+text attention
with rotary embedding (BF16 and FP8) and the First-Block-Cache gate.

The compute runs in ``libdit.so`` (hand-written CUDA for sm_100a, C ABI in
``include/dit.h``); this package is the thin Python binding over it.
"""
from ._binding import (  # noqa: F401
    DitError,
    FBCacheGate,
    attention,
    attention_workspace,
    fbcache_gate,
    fbcache_gate_finalize,
    fbcache_gate_ref_update,
    fbcache_gate_sums,
    fp8_workspace_views,
    lib,
    read_error,
    rope_apply,
    rope_tables,
    selftest_wait_timeout,
    probe_unit_rates,
)
