"""B200-native (sm_100a) data-parallel hot path of ZeRO stages 1 and 2.

    from zero_partitioned_optimizer_plan_b200 import libzero   # binding of libzero.so
    from zero_partitioned_optimizer_plan_b200 import synth     # seeded synthetic inputs

The C ABI is include/libzero.h; the CUDA kernels and the native runtime (planner, bucket
scheduler) are under csrc/ and build into the in-tree libzero.so
(``python -m zero_partitioned_optimizer_plan_b200.build``).
"""
