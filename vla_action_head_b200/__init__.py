"""vla_action_head_b200: the NVFP4 linear layer of a VLA action head on B200 (sm_100a).

The compute path is the C-ABI library libnvfp4.so built from csrc/ (hand-written sm_100a
CUDA); `nvfp4` is its thin Python binding (argument marshalling only).
"""
