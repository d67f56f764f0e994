"""W8A8 CausalConv3d for the Qwen-Image / Wan VAE decoder on B200 (sm_100a).

The compute path is the CUDA library ``libqvae.so`` (sources in ``csrc/``,
C declarations in ``include/qvae.h``).  ``qvae`` is a thin ctypes binding with
the same entry-point names; ``synth`` draws the seeded synthetic inputs.
Importing the package loads nothing; ``qvae.lib()`` loads the library and
fails loudly when it is missing.
"""
__all__ = ["qvae", "synth"]
