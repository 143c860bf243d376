"""B200-native DeepSeekMoE layer forward: a C-ABI library of sm_100a kernels and its binding.

The binding (`fine_grained_mixture_route_b200.moe`) loads the shared library on first use;
importing the package itself loads nothing, so the seeded input generator
(`fine_grained_mixture_route_b200.workloads`) can be imported on machines without a GPU.
"""
