"""Byte accounting for the Fathom scan.

The paper argues in bytes per token (yeyulingfeng.com article, sections
"先算一笔字节账" and "方法一"/"方法二"): a block of 64 tokens of one channel
stores four 64-bit plane words and one fp16 scale, and a scan that reads t
planes of a channel pays t bits per token plus the channel's scale, 16 bits
shared by 64 tokens.  These helpers turn plans into bytes; the benchmark
uses them for the algorithmic-byte side of its roofline.
"""
from __future__ import annotations

BLOCK = 64          # tokens per scale block
PLANES = 4          # bit planes per channel (4-bit codes)
SCALE_BITS = 16     # one fp16 scale per block per channel


def index_bytes_per_token(D: int) -> float:
    """Bytes the full index stores per token per KV head: D channels x
    (4 plane bits + 16/64 scale bits)."""
    return D * (PLANES + SCALE_BITS / BLOCK) / 8.0


def read_bits_per_token(plane_bits: int, n_active: int) -> float:
    """Bits a scan reads per token for one group: its plane bits plus one
    scale per active channel shared by the block's 64 tokens."""
    return plane_bits + n_active * SCALE_BITS / BLOCK


def fixed_scan_bits(r: int, bits: int = PLANES) -> float:
    """Per-token bits of a fixed-depth scan of r channels at ``bits`` bits."""
    return read_bits_per_token(r * bits, r)


def scan_bytes(n: int, plane_bits: int, n_active: int, G: int = 4, D: int = 128,
               query_bytes: bool = True) -> int:
    """Algorithmic bytes one group's scan must read: n*(sum t_j)/8 plane
    bytes + one 2-byte scale per active channel per block, plus the
    group's fp32 queries."""
    nb = (n + BLOCK - 1) // BLOCK
    b = (n * plane_bits) // 8 + n_active * 2 * nb
    if query_bytes:
        b += G * D * 4
    return b


def token_major_scan_bytes(n: int, n_active: int, G: int = 4, D: int = 128, query_bytes: bool = True) -> int:
    """Bytes one group's scan of a token-major 4-bit copy moves: whole rows
    of D/2 bytes per token (whatever the number of channels read) plus one
    2-byte scale per active channel per block and the group's queries."""
    nb = (n + BLOCK - 1) // BLOCK
    b = n * D // 2 + n_active * 2 * nb
    if query_bytes:
        b += G * D * 4
    return b


def step_scan_bytes(n: int, plan_bits, plan_active, G: int = 4, D: int = 128) -> int:
    """Algorithmic bytes over all groups of one step."""
    return sum(scan_bytes(n, int(b), int(a), G, D) for b, a in zip(plan_bits, plan_active))


def dense_kv_bytes(layers: int, kv_heads: int, D: int, n: int, elem_bytes: int = 2) -> int:
    """Bytes of a dense K and V cache read once."""
    return 2 * layers * kv_heads * D * n * elem_bytes


def per_token_index_bytes(layer_heads: int, n: int, bytes_per_token: float) -> float:
    """Bytes of a per-token index of the given width over all layer-heads."""
    return layer_heads * n * bytes_per_token
