"""SWAT sliding-window attention on B200 (sm_100a).

The compute path is the C-ABI library ``libswat.so`` (hand-written CUDA);
``binding`` marshals torch tensors into its calls. Importing this package
does not load the library; the first call does, and fails loudly if the
library is missing.
"""
