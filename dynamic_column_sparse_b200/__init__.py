"""Column-sparse cross-step deltas (Chipmunk-style) on B200: C-ABI CUDA library + thin binding.

``dynamic_column_sparse_b200.chipmunk`` holds the binding (imports torch);
``dynamic_column_sparse_b200.synth`` the seeded input generator (numpy only).
"""
__version__ = "0.1.0"
