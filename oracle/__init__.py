"""Float64 CPU oracle of the RG-LRU layer: test infrastructure only.

Only tests/, the smoke check and the bench's CPU-baseline leg import this
package. The CUDA library never does, and has no CPU fallback through it.
"""
