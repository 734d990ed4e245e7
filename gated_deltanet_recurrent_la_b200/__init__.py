"""B200-native recurrent-state step for linear attention (Gated DeltaNet family).

The compute path is liblastate.so (hand-written CUDA for sm_100a behind a C ABI,
include/la_state.h).  `gated_deltanet_recurrent_la_b200.lastate` is its thin Python
binding; `workloads` generates seeded synthetic inputs.
"""
__all__ = ["lastate", "workloads"]


def __getattr__(name):
    if name in ("lastate", "workloads"):
        import importlib
        return importlib.import_module(f"{__name__}.{name}")
    raise AttributeError(name)
