"""Parallax attention (softmax attention with a covariance correction) for B200.

The compute path is the C-ABI library ``libplx.so`` built from ``csrc/`` for
sm_100a; ``plx`` (imported lazily) is its thin ctypes binding.
"""
