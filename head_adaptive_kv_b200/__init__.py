"""B200-native decode hot path of HARD-KV's Cascade Cache.

Five steps per (sequence, KV head): score the sparse tier against the current
query, Logits Calibration, a clamped per-head Top-p budget, order-preserving
compaction into a static layout (Rewrite Cache / Flatten Index), and cascade
decode attention over the dense, compacted-sparse and condensed tiers. All of it
runs in ``libhkv.so`` (hand-written CUDA for sm_100a, C ABI in ``include/hkv.h``);
the ``hkv`` module only marshals arguments. ``workloads`` makes seeded inputs.
"""
_EXPORTS = {
    "FLAT_SUM", "PAD_MAX", "Cut", "HkvError", "Problem", "StepOutputs", "Tier", "Workspace",
    "calibrate", "cascade_decode", "compact", "debug_withhold_publish", "launch_count", "score",
    "set_wait_limit_ns", "step", "status_string", "topp_select",
}


def __getattr__(name):
    if name in _EXPORTS:
        from . import hkv  # loads libhkv.so; raises if it is missing

        return getattr(hkv, name)
    raise AttributeError(name)
