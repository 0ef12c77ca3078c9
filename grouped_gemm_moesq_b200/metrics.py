"""Work accounting for the grouped GEMM and the MoE layer (host only).

Effective throughput follows the paper's kernel benchmark (App. D.2):
TFLOP/s_eff = 2 * M * K * sum_g N_g / (t * 1e12), counting the dense
contraction even though the sparse MMA skips half of it.  Algorithmic bytes
count what a kernel must move at least once: the packed weights of the
experts that receive tokens (11 * M * K / 32 bytes each: E2M1 values K/4,
pair mask K/16 and UE4M3 scales K/32 per row, paper App. A Eq. 7), the NVFP4
activations (K/2 codes + K/32 scales per row) and the bf16 output.
"""
from __future__ import annotations


def token_pattern(n: int, groups: int):
    """Per-expert token counts {N, 3N/4, N/2, N/4} repeated over `groups`
    experts (paper, App. D.2)."""
    base = [n, 3 * n // 4, n // 2, n // 4]
    return [base[g % 4] for g in range(groups)]


def effective_tflops(M: int, K: int, counts, seconds: float) -> float:
    return 2.0 * M * K * sum(counts) / (seconds * 1e12)


def packed_weight_bytes(M: int, K: int) -> int:
    """Bytes of one packed expert linear (values + mask + scales)."""
    return 11 * M * K // 32


def gemm_algorithmic_bytes(M: int, K: int, counts) -> int:
    """Minimum HBM bytes of one grouped sparse GEMM launch."""
    touched = sum(1 for c in counts if c > 0)
    rows = sum(counts)
    return (touched * packed_weight_bytes(M, K) + touched * 4     # weights + alpha inputs
            + rows * (K // 2 + K // 32)                           # NVFP4 activations
            + rows * M * 2)                                       # bf16 output


def gemm_flops(M: int, K: int, counts) -> float:
    """Dense-equivalent flops (2 M K per routed row)."""
    return 2.0 * M * K * sum(counts)
