"""B200-native decode hot path: fused 4-bit dequant-GEMV, paged GQA decode
attention, MoE routing and greedy argmax behind the ``bw_*`` C ABI.

Importing the package loads nothing; ``token_decode_b200.bw`` loads the
compiled library (``libbw.so``) and fails loudly when it is missing.
"""
__all__ = ["synth"]
