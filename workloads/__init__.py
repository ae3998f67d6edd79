"""Seeded synthetic inputs for paged decode attention.

This package only *produces inputs*: context lengths, block tables, slot
mappings, copy-on-write pairs and random tensor values.  It holds none of the
method's arithmetic (no gather, no softmax, no scatter, no block copy), so the
CPU oracle and the CUDA path can both be fed from it without sharing any code
that computes a result.
"""

from .configs import CONFIGS, WorkloadConfig, get_config  # noqa: F401
from .gen import (Workload, build_workload, device_values, host_values, poison_unread_slots,  # noqa: F401
                  unread_slots)
