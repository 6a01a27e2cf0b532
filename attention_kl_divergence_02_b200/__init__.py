"""libstreamkl: a B200-native (sm_100a) fused attention KL divergence.

Forward: per query row KL(P1||P2) with P_t = softmax(scale * Q_t K_t^T), computed in one
pass over key tiles without materialising P1 or P2, plus the two log-sum-exp vectors.
Backward: gradients of sum_i g_i KL_i with P1 fixed (mode 1) or P2 fixed (mode 2),
recomputing the probabilities tile by tile from the saved LSEs.

The compute runs in the CUDA library ``libstreamkl.so`` behind a C ABI
(``include/streamkl.h``); ``attention_kl_divergence_02_b200.binding`` marshals torch
tensors into that ABI.  Importing this package loads nothing; the binding loads the
library on first use and raises if it is missing.
"""
__all__ = ["binding", "inputs"]
