"""Seeded synthetic inputs and the decoder shapes they follow.

This module holds no arithmetic of the quantised matmul: it only draws the
float32 weights and activations that both the CUDA path and the CPU oracle are
fed, and names the shapes of the workloads.

Shapes: the decoder is a Qwen3-0.6B-style backbone with hidden size 1024 and
28 blocks whose KV cache holds 8 heads of 128 ("MOSS-Transcribe-Diarize --
LiteRT (TFLite)", section "Files"; the architecture section of the evermx
article names the Qwen3-0.6B-style decoder). The per-projection [out, in]
shapes below follow from those sizes; the tied embedding / lm_head has a
151,936-token vocabulary.

Value distributions: weights ~ N(0, 0.02^2), activations ~ N(0, 1), both
float32, drawn on the CPU with ``torch.Generator().manual_seed(seed)`` so that
every process sees identical bytes.
"""

from __future__ import annotations

import torch

HIDDEN = 1024
N_LAYERS = 28
WEIGHT_STD = 0.02

#: (name, N = out features, K = in features) of one decoder block's linears.
DECODER_PROJ = (
    ("q", 2048, 1024),
    ("k", 1024, 1024),
    ("v", 1024, 1024),
    ("o", 1024, 2048),
    ("gate", 3072, 1024),
    ("up", 3072, 1024),
    ("down", 1024, 3072),
)

#: Tied embedding / lm_head projection [vocab, hidden].
LM_HEAD = (151936, 1024)

LM_HEAD_SEED = 99999
X_SEED = 7


def layer_seed(layer: int, proj_index: int) -> int:
    """Seed of projection ``proj_index`` (q,k,v,o,gate,up,down = 0..6) of block ``layer``."""
    return 1000 * layer + proj_index


def weight(n: int, k: int, seed: int, std: float = WEIGHT_STD) -> torch.Tensor:
    """float32 [n, k] ~ N(0, std^2) on the CPU, seeded."""
    g = torch.Generator().manual_seed(seed)
    return torch.randn(n, k, generator=g, dtype=torch.float32) * std


def activations(m: int, k: int, seed: int) -> torch.Tensor:
    """float32 [m, k] ~ N(0, 1) on the CPU, seeded."""
    g = torch.Generator().manual_seed(seed)
    return torch.randn(m, k, generator=g, dtype=torch.float32)


def raw_codes(n: int, k: int, bits: int, seed: int) -> tuple[torch.Tensor, torch.Tensor]:
    """Uniformly random packed bytes and random finite binary16 scale bit patterns.

    Exercises every code a container may hold, including -8 / -128, which the
    quantiser itself never emits. Returns (packed uint8 [n, k*bits/8],
    scale bit patterns as int16 [n, k/32]); the scales are N(0, 0.01^2) values
    rounded by torch to float16 (sign included).
    """
    g = torch.Generator().manual_seed(seed)
    packed = torch.randint(0, 256, (n, k * bits // 8), generator=g, dtype=torch.int32).to(torch.uint8)
    scales = (torch.randn(n, k // 32, generator=g, dtype=torch.float32) * 0.01).to(torch.float16)
    return packed, scales.view(torch.int16)
