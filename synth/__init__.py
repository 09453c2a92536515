"""Seeded synthetic inputs (weights, KV prefixes, token ids) and model shapes.

Shared by the tests, the benchmark and the oracle's callers.  Holds none of the
method's arithmetic: only shapes and random draws.
"""
from .configs import FULL, LAYER, TINY, WORKLOADS, ModelConfig, Workload  # noqa: F401
from .weights import (LAYER_TENSORS, layer_shapes, make_kv_prefix, make_layer, make_selfcond,  # noqa: F401
                      make_tokens, make_weights, tensor_seed, to_f64)
