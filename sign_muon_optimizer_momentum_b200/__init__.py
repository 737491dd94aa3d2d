"""B200-native Sign-Muon optimizer step.

The compute path is the C-ABI library ``libsignmuon.so`` (hand-written CUDA
for sm_100a) exposed through the thin ctypes binding in ``_lib``; PyTorch is
used only for device memory, streams and seeded input generation.  Importing
the package does not load the library; the first call into ``_lib`` does, and
fails loudly if it has not been built.
"""
__all__ = ["synthetic"]
