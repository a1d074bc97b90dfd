"""B200-native ExTernD decomposition: greedy sequential-deflation ALS that
factors an fp32 matrix A (m x n) into B diag(D) C with ternary B, C and
inner rank k = mu * min(m, n), plus its block-ALS and importance-weighted
variants.  The compute runs in the CUDA library ``libexternd.so`` (sm_100a);
``externd`` is the ctypes binding to its C ABI."""

__all__ = ["externd", "workloads"]
