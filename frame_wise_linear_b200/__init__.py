"""B200-native Video Delta Attention (VDA) forward.

The CUDA library (``libvda.so``, built from ``csrc/``) is loaded on first use
by :mod:`frame_wise_linear_b200.vda`; importing this package alone loads
nothing, so that :mod:`frame_wise_linear_b200.synth` stays usable without a
built library.
"""
