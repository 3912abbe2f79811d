"""B200-native hot path of Doge's Dynamic Mask Attention (DMA).

The compute lives in the C-ABI library ``libdma.so`` (CUDA, sm_100a); the
binding in :mod:`doge_dynamic_mask_b200.dma` only marshals arguments.  Import
that module to use the library: it raises if the library is not built.
"""
__version__ = "0.1.0"
