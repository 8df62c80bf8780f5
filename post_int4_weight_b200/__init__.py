"""AWQ INT4 weight quantisation hot path for B200 (sm_100a).

Activation statistics, the per-linear alpha grid search for the AWQ scale,
group-wise symmetric INT4 quantisation with the AutoAWQ GEMM packing, and the
optional output-space scoring, each a hand-written CUDA kernel behind the
C ABI declared in ``include/awq.h``.  ``post_int4_weight_b200.awq`` is the
Python binding (argument marshalling only).
"""
from .workloads import WORKLOADS, Workload, SearchGroup  # noqa: F401

__all__ = ["WORKLOADS", "Workload", "SearchGroup"]
