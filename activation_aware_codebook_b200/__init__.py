"""B200-native AAAC (activation-aware adaptive codebook) layer fit.

The compute path is the C-ABI library ``libaaac.so`` (hand-written sm_100a
CUDA kernels, csrc/); ``binding`` marshals torch tensors into its calls.
``synth`` draws the seeded synthetic inputs.
"""
