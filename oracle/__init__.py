"""CPU oracle for the HySparse hybrid block (test infrastructure only).

Only the tests, the package smoke check and the benchmark's CPU-baseline leg
may import this package.  The product path never does: it shares no code with
it and fails loudly when its own CUDA library is missing.
"""
from .hsref import (build, use_library, full_rows, topk_rows, sparse_rows, block_rows, max_threads,
                    set_threads, library_path)

__all__ = ["build", "use_library", "full_rows", "topk_rows", "sparse_rows", "block_rows", "max_threads",
           "set_threads", "library_path"]
