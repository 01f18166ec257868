"""epx: B200-native (sm_100a) MoE token dispatch and combine.

The compute path is libepx.so (hand-written CUDA, C ABI in include/epx.h);
``combine_ep_layout_07_b200.epx`` is its argument-marshalling binding.
``combine_ep_layout_07_b200.workloads`` draws the seeded synthetic inputs.
"""
from .epx import (EpxError, Layout, combine_epilogue, combine_local_reduce,  # noqa: F401
                  combine_reduce, dispatch, dispatch_expand, expand_index, layout,
                  read_totals, roundtrip_device_bytes, roundtrip_host, roundtrip_host_noalloc,
                  standin_expert, standin_expert_gather)
