"""Hierarchical local attention (UltraGen) for NVIDIA B200, sm_100a.

``ug`` is the ctypes binding of the C-ABI library libug.so (built in-tree by
``block_sparse_local_raster_b200.build``); ``workloads`` holds the workload
geometries and seeded input generators.  Importing the package loads nothing;
the library is loaded by the first binding call and its absence is an error.
"""
