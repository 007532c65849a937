"""libsparseattn: block-sparse attention with in-softmax block approximation on B200.

The compute path is the C-ABI shared library ``libsparseattn.so`` built from
``csrc/`` for sm_100a; ``binding`` marshals torch tensors to its entry points.
Importing this package loads nothing; ``binding.load()`` loads the library and
raises if it has not been built.
"""

__all__ = ["binding", "workloads"]
