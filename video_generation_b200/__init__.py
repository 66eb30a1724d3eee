"""B200-native affine autoregressive flow (STARFlow-V AF block) -- CUDA library + thin binding.

``video_generation_b200.flow`` loads libaf.so (built by ``video_generation_b200.build``)
and exposes af_forward, af_inverse_jacobi, flow_stack_forward and flow_stack_inverse.
"""
