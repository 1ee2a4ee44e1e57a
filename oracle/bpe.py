"""Effective bits per KV element of a quantized cache format.

TEST INFRASTRUCTURE ONLY (see the package docstring).

Follows "Dual-QK: Sharp Queries and Flat Keys for Prunable 2-bit KV Caches",
§4.1 (capacity BPE describes the stored cache; bandwidth BPE the KV data read
per decoding step with channel selection; both include quantization metadata
and the BF16-protected sink and recent tokens) and Table 1 (the printed BPE
values at a 128K context and 40% query-channel sparsity).

A format is described per token and KV head:
  k_quant_channels   key channels stored at `bits` (the rest of the 128 key
                     channels are stored as BF16 "protected" channels)
  k_meta_bits        key scale/zero bits per token
  v_meta_bits        value scale/zero bits per token
  protected_tokens   tokens kept entirely in BF16 (keys and values)
Reads at sparsity s touch k = ceil((1-s) d) key channels (protected BF16 key
channels count among them), all value channels and all metadata.
"""
from __future__ import annotations

import dataclasses
import math

D = 128


@dataclasses.dataclass(frozen=True)
class Format:
    bits: int
    k_quant_channels: int
    k_meta_bits: int
    v_meta_bits: int
    protected_tokens: int = 0


def _k_selected(sparsity: float, d: int = D) -> int:
    return int(math.ceil((1.0 - sparsity) * d - 1e-9))


def stored_bits_per_token(f: Format) -> float:
    k_bf16 = D - f.k_quant_channels
    return (f.k_quant_channels * f.bits + k_bf16 * 16 + f.k_meta_bits
            + D * f.bits + f.v_meta_bits)


def read_bits_per_token(f: Format, sparsity: float) -> float:
    k = _k_selected(sparsity)
    k_bf16 = D - f.k_quant_channels          # protected channels, always read
    k_q = k - k_bf16
    return k_q * f.bits + k_bf16 * 16 + f.k_meta_bits + D * f.bits + f.v_meta_bits


def capacity_bpe(f: Format, n_ctx: int) -> float:
    p = f.protected_tokens
    bits = (n_ctx - p) * stored_bits_per_token(f) + p * 2 * D * 16
    return bits / (n_ctx * 2 * D)


def bandwidth_bpe(f: Format, n_ctx: int, sparsity: float) -> float:
    p = f.protected_tokens
    k = _k_selected(sparsity)
    bits = (n_ctx - p) * read_bits_per_token(f, sparsity) + p * (k + D) * 16
    return bits / (n_ctx * 2 * D)


# The pages' own formats.
DUAL_QK_PAGES = Format(bits=2, k_quant_channels=127, k_meta_bits=32, v_meta_bits=32,
                       protected_tokens=64 + 256)
OSCAR_PAGES = Format(bits=2, k_quant_channels=128, k_meta_bits=32, v_meta_bits=32,
                     protected_tokens=64 + 256)
# The group-32 layout built here: four fp16 scale/zero pairs per token for keys
# and for values, channel 0 of the key in BF16, no protected tokens.
GROUP32_INT2 = Format(bits=2, k_quant_channels=127, k_meta_bits=4 * 32, v_meta_bits=4 * 32)
GROUP32_INT4 = Format(bits=4, k_quant_channels=127, k_meta_bits=4 * 32, v_meta_bits=4 * 32)
