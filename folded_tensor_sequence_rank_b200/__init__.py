"""TSP (Tensor + Sequence Parallelism) per-rank dense-layer forward for B200.

The CUDA library and its binding live in `folded_tensor_sequence_rank_b200.tsp`
(imported on first use); `folded_tensor_sequence_rank_b200.inputs` draws the
seeded synthetic inputs.
"""
__all__ = ["tsp", "inputs"]


def __getattr__(name):
    if name in ("tsp", "inputs"):
        import importlib
        return importlib.import_module(f"{__name__}.{name}")
    raise AttributeError(name)
