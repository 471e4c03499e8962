"""B200-native chunk-causal attention layer of UnStep's causal video DiT step.

The compute path is ``libunstep.so`` (hand-written sm_100a CUDA behind a C ABI, see
``include/unstep.h``); :mod:`causal_video_diffusion_b200.binding` marshals torch tensors into
its calls.  Importing this package loads nothing; the binding loads the library on first use and
raises if it is missing.
"""
__version__ = "0.1.0"
