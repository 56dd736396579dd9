"""fp64 CPU oracle for deferred-RoPE attention over a shared paged KV cache.

TEST INFRASTRUCTURE ONLY: the test suite, the smoke check and the benchmark's
CPU-baseline leg are the only callers.  The CUDA library neither imports nor
links anything here, and nothing here imports the CUDA library.

The arithmetic lives in ``lazy_oracle.c`` (plain C99, double precision); this
module compiles it with gcc on first use and wraps it with ctypes.
"""
from .oracle import (  # noqa: F401
    build,
    load_library,
    lib_path,
    bf16_to_f64,
    f64_to_bf16,
    pack_word,
    unpack_word,
    pack_meta,
    rope,
    llama31_theta,
    alibi_slopes,
    kv_write,
    expand_table,
    attend,
    rope_rows_bf16,
    num_threads,
    set_num_threads,
)
