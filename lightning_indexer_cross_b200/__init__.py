"""B200-native (sm_100a) IndexCache decode hot path.

The compute lives in ``libindexcache.so`` (C ABI, ``include/indexcache.h``):
lightning indexer, top-k, sparse MLA decode with sink and gate, and the F/S
layer-stack driver. ``_abi`` binds it with ctypes under the same names;
``ops`` is a thin torch-tensor front end. ``workloads`` draws the seeded
synthetic inputs. Importing ``_abi``/``ops`` fails if the library has not
been built; there is no fallback implementation.
"""
__all__ = ["workloads", "ops", "_abi", "build"]
