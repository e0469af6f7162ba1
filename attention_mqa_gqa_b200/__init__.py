"""B200-native (sm_100a) fused attention forward for grouped query heads.

One C-ABI library (``libattn_b200.so``, declared in ``include/attn_b200.h``)
computes softmax(scale * Q K^T) V where many query heads share few K/V heads:
MHA/GQA/MQA at head_dim 128 or 512, and absorbed-MLA decode over cached
576-wide latent rows whose first 512 columns are the values.  The Python
module ``binding`` only marshals arguments into that library.
"""
