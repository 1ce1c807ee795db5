"""Seeded synthetic inputs shared by the CUDA path's tests/bench and the CPU oracle.

This package holds no attention arithmetic: it only names the workloads and
draws their random inputs, so that both sides see identical bf16 bit patterns.
"""

from .workloads import (WORKLOADS, Workload, head_subset, make_grad_output, make_inputs, make_inputs_fp8, make_inputs_fp8kv,
                        quantize_e4m3)

__all__ = ["WORKLOADS", "Workload", "make_inputs", "make_inputs_fp8", "make_inputs_fp8kv", "quantize_e4m3", "make_grad_output",
           "head_subset"]
