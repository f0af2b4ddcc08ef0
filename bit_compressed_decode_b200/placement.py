"""Which layers of a weight-streamed stack keep their blobs in HBM.

"FlexGen Guide: High-Throughput LLM Offloading on One GPU", section 1 (Three-Tier Storage
Hierarchy): the policy places a fraction of the weights on the GPU and streams the rest from CPU
memory. Here the fraction is the largest number of layers whose blobs fit the device memory left
after the stack's other needs, and those layers are spread evenly over the stack, so the copy of
each streamed layer overlaps the compute of the resident layer before it (fg_stack_create keeps a
layer whose blob is in device memory resident: no copy, no staging buffer). No linear program: the
pages' LP placement optimiser is out of scope.
"""
from __future__ import annotations


def resident_count(free_bytes: int, blob_bytes: int, num_layers: int, reserve_bytes: int = 0) -> int:
    """Layers whose blobs fit in `free_bytes` of device memory minus `reserve_bytes`."""
    if blob_bytes <= 0 or num_layers < 0:
        raise ValueError("bad placement arguments")
    room = free_bytes - reserve_bytes
    return max(0, min(num_layers, room // blob_bytes))


def spread(resident: int, num_layers: int) -> list[bool]:
    """`resident` of `num_layers` layers marked resident, spread evenly: layer l is resident when
    floor((l + 1) R / n) > floor(l R / n)."""
    if not 0 <= resident <= num_layers:
        raise ValueError("resident layers out of range")
    return [(l + 1) * resident // num_layers > l * resident // num_layers for l in range(num_layers)]
