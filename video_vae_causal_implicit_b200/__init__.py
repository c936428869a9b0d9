"""B200-native causal Conv3D (Wan-style WanCausalConv3d) and residual block.

The compute lives in the CUDA library ``libcc3d.so`` (built for sm_100a);
``cc3d`` holds the thin ctypes binding over its C ABI.  ``synth`` draws the
seeded synthetic inputs.  The library is loaded on first use, so importing
the package never needs a GPU.
"""
__all__ = ["cc3d", "synth"]
