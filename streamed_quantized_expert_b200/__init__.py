"""B200-native streamed, quantized routed-expert FFN.

The compute path is the C-ABI library ``libmoe.so`` (hand-written CUDA for
sm_100a) declared in ``include/moe.h``; ``ops`` is its thin ctypes binding.
``synth`` draws the seeded synthetic inputs.
"""
