"""B200-native (sm_100a) WKV7: the RWKV-7 generalized delta rule behind a C ABI.

``wkv7_fwd`` / ``wkv7_step`` (and their State Anomaly Neutralization forms
``wkv7_sane_fwd`` / ``wkv7_sane_step``, and the Gated DeltaNet ``wkv7_gdn_fwd`` /
``wkv7_gdn_step``) call libwkv7.so (hand-written CUDA kernels);
``synth`` draws the seeded synthetic workloads.  Importing this package does
not load the CUDA library; the first call does, and fails loudly if it is
missing.
"""
from .wkv7 import (WKV7Error, gated_delta_net, generalized_delta_rule, library,  # noqa: F401
                   status_string, wkv7_bwd, wkv7_fwd, wkv7_gdn_bwd, wkv7_gdn_fwd,
                   wkv7_gdn_step, wkv7_get_last_error, wkv7_sane_fwd, wkv7_sane_step,
                   wkv7_step)

__all__ = ["wkv7_fwd", "wkv7_step", "wkv7_bwd", "generalized_delta_rule", "wkv7_sane_fwd",
           "wkv7_sane_step", "wkv7_gdn_fwd",
           "wkv7_gdn_step", "wkv7_gdn_bwd", "gated_delta_net", "wkv7_get_last_error",
           "library", "status_string", "WKV7Error"]
