"""B200-native block-compressed attention (LBCA / HCA form).

The compute path is the C-ABI library ``liblbca.so`` (hand-written CUDA for
sm_100a); ``block_compressed_long_b200.lbca`` is its thin ctypes binding and
``block_compressed_long_b200.synth`` draws seeded synthetic inputs.
"""
