"""libkda: B200-native KDA forward scan with modality-aware short convolution.

The compute lives in the CUDA shared library ``libkda.so`` (C ABI, see
``include/kda.h``); ``kda`` is its thin Python binding and ``sequence_parallel`` runs
the sequence-parallel forward over ``torch.distributed``.  Importing this package does
not load the library, so the input generators work on machines without a GPU.
"""
__all__ = ["inputs", "kda", "sequence_parallel"]
