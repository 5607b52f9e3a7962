"""B200 (sm_100a) ring-chunked attention and Ulysses layout transforms.

The compute lives in ``libra_b200.so`` (hand-written CUDA for sm_100a behind the
C ABI of ``include/ra.h``).  ``sequence_parallelism_attn_b200.ra`` is the thin
ctypes binding with the same entry-point names; it loads the library on first
use and raises if it is missing -- there is no fallback path.  ``dist`` carries the path
across GPUs (NCCL through torch.distributed) and ``autograd`` pairs every forward with its
backward for training.
"""
__all__ = ["ra", "synth", "dist", "autograd"]
