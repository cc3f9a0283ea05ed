"""B200 (sm_100a) Mixture-of-Experts layer forward behind a C ABI.

route -> dispatch -> grouped expert FFN -> combine, in hand-written CUDA
kernels (libmoe.so, declared in include/moe.h).  ``api`` is the Python face
of that ABI; ``inputs`` draws the seeded synthetic workloads.  Importing the
package does not load the library: the first call into ``api`` does, and it
fails loudly if the library has not been built.
"""

__all__ = ["api", "inputs", "build"]
