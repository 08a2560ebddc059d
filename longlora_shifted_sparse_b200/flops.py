"""FLOP accounting for S2-Attn.

Counting convention: each of the two per-group contractions (Q K^T and P V) costs
2 * G * G * d FLOPs per (batch, head, group) without a mask; a causal mask halves it.
So forward = 4 * B * H * N * G * d (/ 2 when causal), and backward = 2.5 x forward.
The ratio to dense attention is N / G ("LongLoRA and Shifted Sparse Attention (S^2-Attn)",
mechanism claim: M = N / G groups cut attention FLOPs M-fold).
"""


def attention_fwd_flops(B: int, N: int, H: int, d: int, G: int, causal: bool = True) -> float:
    f = 4.0 * B * H * N * G * d
    return f / 2 if causal else f


def attention_bwd_flops(B: int, N: int, H: int, d: int, G: int, causal: bool = True) -> float:
    return 2.5 * attention_fwd_flops(B, N, H, d, G, causal)


def toy_dense_ops(L: int, D: int) -> int:
    """The pages' toy operation count for full attention: L^2 * D
    ("LongLoRA: Efficient 100k Context LLM Fine-Tuning Guide", Step 2)."""
    return L * L * D


def toy_s2_ops(L: int, G: int, D: int) -> int:
    """The same page's toy count for shifted sparse attention: L * G * D."""
    return L * G * D
