"""B200 (sm_100a) implementation of FlexQ's group-quantized W6A6 / W6A8 linear layer.

The compute path is the CUDA library ``libflexq.so`` (C ABI in include/flexq.h);
``flexq`` is its thin Python binding and ``inputs`` draws seeded synthetic
inputs.  Importing the package does not load the library; the first call does,
and raises if it has not been built.
"""
