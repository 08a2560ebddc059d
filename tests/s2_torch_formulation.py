"""An independent statement of S2-Attn built from library routines, used only to pin the oracle.

It follows the pages' tensor formulation instead of the oracle's row/index arithmetic:
RoPE as complex multiplication x * exp(i m theta / s) (the RoFormer closed form), the
shift as ``torch.roll`` of whole tensors, the group fold as a reshape into the batch
dimension, and the per-group attention as ``torch.nn.functional.scaled_dot_product_attention``
(fp64, CPU). Sources: "LongLoRA and Shifted Sparse Attention (S^2-Attn)" (definition
paragraph), "LongLoRA: Efficient 100k Context LLM Fine-Tuning Guide" (How Shifted Short
Attention Works; Implementation, Step 1), "LoRA for Long-Context Adaptation" (RoPE and
position interpolation sections).
"""
from __future__ import annotations

import torch
import torch.nn.functional as F


def rope_complex(x: torch.Tensor, s: float, base: float = 10000.0) -> torch.Tensor:
    """x [B, N, H, d] real fp64 -> rotated copy; pair (2i, 2i+1) is one complex number."""
    B, N, H, d = x.shape
    pos = torch.arange(N, dtype=torch.float64) / s
    theta = base ** (-torch.arange(0, d, 2, dtype=torch.float64) / d)
    ang = pos[:, None] * theta[None, :]
    rot = torch.polar(torch.ones_like(ang), ang)  # [N, d/2] complex
    z = torch.view_as_complex(x.reshape(B, N, H, d // 2, 2).contiguous())
    return torch.view_as_real(z * rot[None, :, None, :]).reshape(B, N, H, d)


def _grouped(q, k, v, G, causal):
    B, H, N, d = q.shape
    fold = lambda t: t.reshape(B * H * (N // G), G, d)
    o = F.scaled_dot_product_attention(fold(q), fold(k), fold(v), is_causal=causal)
    return o.reshape(B, H, N, d)


def _grouped_lse(q, k, G, causal):
    B, H, N, d = q.shape
    fold = lambda t: t.reshape(B * H * (N // G), G, d)
    sc = fold(q) @ fold(k).transpose(1, 2) / (d ** 0.5)
    if causal:
        keep = torch.ones(G, G, dtype=torch.bool).tril()
        sc = sc.masked_fill(~keep, float("-inf"))
    return torch.logsumexp(sc, dim=-1).reshape(B, H, N)


def s2attn(q, k, v, G: int, s: float, base: float = 10000.0, causal: bool = True,
           with_lse: bool = False):
    """q [B,N,Hq,d], k/v [B,N,Hkv,d] fp64 tensors -> o [B,N,Hq,d] (and lse [B,Hq,N])."""
    Hq, Hkv = q.shape[2], k.shape[2]
    R = Hq // Hkv
    qh = rope_complex(q, s, base).transpose(1, 2)
    kh = rope_complex(k, s, base).transpose(1, 2).repeat_interleave(R, dim=1)
    vh = v.transpose(1, 2).repeat_interleave(R, dim=1)
    half = Hq // 2
    sh = G // 2
    roll_fwd = lambda t: torch.roll(t, shifts=-sh, dims=2)
    roll_back = lambda t: torch.roll(t, shifts=sh, dims=2)
    o_std = _grouped(qh[:, :half], kh[:, :half], vh[:, :half], G, causal)
    o_sh = roll_back(_grouped(roll_fwd(qh[:, half:]), roll_fwd(kh[:, half:]),
                              roll_fwd(vh[:, half:]), G, causal))
    o = torch.cat([o_std, o_sh], dim=1).transpose(1, 2)
    if not with_lse:
        return o
    l_std = _grouped_lse(qh[:, :half], kh[:, :half], G, causal)
    l_sh = roll_back(_grouped_lse(roll_fwd(qh[:, half:]), roll_fwd(kh[:, half:]), G, causal))
    return o, torch.cat([l_std, l_sh], dim=1)


def dense_causal(q, k, v, s: float, base: float = 10000.0):
    """Textbook dense causal attention over the whole sequence (the pages' inference mode)."""
    Hq, Hkv = q.shape[2], k.shape[2]
    R = Hq // Hkv
    qh = rope_complex(q, s, base).transpose(1, 2)
    kh = rope_complex(k, s, base).transpose(1, 2).repeat_interleave(R, dim=1)
    vh = v.transpose(1, 2).repeat_interleave(R, dim=1)
    return F.scaled_dot_product_attention(qh, kh, vh, is_causal=True).transpose(1, 2)
