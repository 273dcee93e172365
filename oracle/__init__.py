"""fp64 CPU oracle of the tensor-parallel MLP block with biases.

TEST INFRASTRUCTURE ONLY: imported by the tests, by ``__graft_entry__.smoke()``
and by the CPU-baseline leg of ``bench.py``; never by the CUDA library or its
Python binding.
"""
