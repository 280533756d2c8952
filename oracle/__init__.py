"""CPU oracle for the NVFP4 linear layer (test infrastructure only).

Only tests/, __graft_entry__.smoke() and bench.py's CPU baseline may import this
package.  It shares no code with the CUDA path.
"""
