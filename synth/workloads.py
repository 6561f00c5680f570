"""Workload shapes and input recipes for the low-bit linears of FLUX.2-Klein-4B.

Token counts follow the latent geometry of the Bonsai Image pipeline: an image of
H x W pixels gives (H/16)(W/16) image tokens, and the text stream is padded to 512
tokens (mlx-vlm Bonsai article, component architecture section). The hidden width
3072 (MLP ratio 3) is a representative size; the text-encoder widths 2560 / 9728
are the Qwen3 encoder's (same article). Every tensor is drawn from ``synth``'s
counter-based generator, so inputs are identical wherever they are rebuilt.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import List, Optional

import numpy as np


@dataclass(frozen=True)
class LinearSpec:
    name: str
    M: int
    K: int
    N: int
    bits: int
    group_size: int
    p0: float = 1.0 / 3.0          # P(code == 0) for ternary codes
    scale_lo: float = 0.005
    scale_hi: float = 0.02
    zero_lo: float = 6.0           # 4-bit zero points, in code units
    zero_hi: float = 9.0
    seed: int = 0
    stream_base: int = 0           # added to every per-tensor stream id

    @property
    def flops(self) -> int:
        return 2 * self.M * self.K * self.N

    def algorithmic_bytes(self) -> int:
        """Packed W + scales (+ zeros) + X + Y, each moved once."""
        groups = self.K // self.group_size
        w = self.N * self.K * self.bits // 8
        sz = groups * self.N * 2 * (2 if self.bits == 4 else 1)
        return w + sz + self.M * self.K * 2 + self.M * self.N * 2

    def with_m(self, M: int, name: Optional[str] = None) -> "LinearSpec":
        d = dict(self.__dict__)
        d["M"] = M
        if name:
            d["name"] = name
        return LinearSpec(**d)


@dataclass
class Problem:
    spec: LinearSpec
    x_bf16: np.ndarray             # uint16 bit patterns, [M][K]
    codes: np.ndarray              # int8, [N][K]
    scales: np.ndarray             # float16, [K/g][N]
    zeros: Optional[np.ndarray]    # float16, [K/g][N] (bits == 4 only)


def make_problem(spec: LinearSpec, with_x: bool = True) -> Problem:
    from . import STREAM_CODES, STREAM_SCALES, STREAM_X, STREAM_ZEROS, codes, normal_bf16, uniform_f16

    s = spec.seed
    b = spec.stream_base
    G = spec.K // spec.group_size
    x = normal_bf16(s, b + STREAM_X, (spec.M, spec.K)) if with_x else None
    c = codes(s, b + STREAM_CODES, (spec.N, spec.K), spec.bits, spec.p0)
    sc = uniform_f16(s, b + STREAM_SCALES, (G, spec.N), spec.scale_lo, spec.scale_hi)
    z = None
    if spec.bits == 4:
        z = uniform_f16(s, b + STREAM_ZEROS, (G, spec.N), spec.zero_lo, spec.zero_hi)
    return Problem(spec, x, c, sc, z)


# ---------------------------------------------------------------------------------------------
# Named workloads
# ---------------------------------------------------------------------------------------------
D = 3072           # transformer hidden width (representative)
TE_H, TE_I = 2560, 9728   # Qwen3 text-encoder hidden / intermediate


def chain_linears(image_hw: int = 1024, text_tokens: int = 512, d: int = D,
                  n_double: int = 5, n_single: int = 20) -> List[LinearSpec]:
    """One denoise step's linear chain: 5 double-stream blocks (separate image and text
    QKV, out, MLP-up, MLP-down) then 20 single-stream blocks (fused QKV+MLP-in, fused out).

    Ternary codes with P(0)=0.4, group 128. Inputs of linear slot ``s`` of block ``blk``
    are drawn with seed ``blk`` and streams ``100*(s+1) + tensor id``, so every linear
    has fresh activations and its own weights.
    """
    m_img = (image_hw // 16) * (image_hw // 16)
    m_all = m_img + text_tokens
    out: List[LinearSpec] = []
    common = dict(bits=2, group_size=128, p0=0.4, scale_lo=0.005, scale_hi=0.02)
    blk = 0
    for _ in range(n_double):
        slot = 0
        for stream_name, m in (("img", m_img), ("txt", text_tokens)):
            for lname, k, n in (("qkv", d, 3 * d), ("out", d, d), ("mlp_up", d, 3 * d), ("mlp_down", 3 * d, d)):
                out.append(LinearSpec(f"double{blk}.{stream_name}.{lname}", m, k, n, seed=blk,
                                      stream_base=100 * (slot + 1), **common))
                slot += 1
        blk += 1
    for _ in range(n_single):
        out.append(LinearSpec(f"single{blk}.qkv_mlp_in", m_all, d, 6 * d, seed=blk, stream_base=100, **common))
        out.append(LinearSpec(f"single{blk}.out", m_all, 4 * d, d, seed=blk, stream_base=200, **common))
        blk += 1
    return out


def chain_linears_separate_qkv(image_hw: int = 1024, text_tokens: int = 512, d: int = D,
                               n_double: int = 5, n_single: int = 20) -> List[LinearSpec]:
    """One denoise step with the transformer's unfused projection layout: each double-stream
    block has separate image Q, K, V (d -> d each), out, MLP-up, MLP-down, and the text stream's
    add-Q, add-K, add-V, add-out, MLP-up, MLP-down (12 linears); single-stream blocks keep their
    fused QKV+MLP-in and out (2 linears). 5 x 12 + 20 x 2 = 100 linears (card: 100 low-bit linear
    layers, Q/K/V and add-Q/K/V among them). Seeds and streams follow chain_linears."""
    m_img = (image_hw // 16) * (image_hw // 16)
    m_all = m_img + text_tokens
    out: List[LinearSpec] = []
    common = dict(bits=2, group_size=128, p0=0.4, scale_lo=0.005, scale_hi=0.02)
    blk = 0
    for _ in range(n_double):
        slot = 0
        for stream_name, m in (("img", m_img), ("txt", text_tokens)):
            for lname, k, n in (("q", d, d), ("k", d, d), ("v", d, d), ("out", d, d), ("mlp_up", d, 3 * d),
                                ("mlp_down", 3 * d, d)):
                out.append(LinearSpec(f"double{blk}.{stream_name}.{lname}", m, k, n, seed=blk,
                                      stream_base=100 * (slot + 1), **common))
                slot += 1
        blk += 1
    for _ in range(n_single):
        out.append(LinearSpec(f"single{blk}.qkv_mlp_in", m_all, d, 6 * d, seed=blk, stream_base=100, **common))
        out.append(LinearSpec(f"single{blk}.out", m_all, 4 * d, d, seed=blk, stream_base=200, **common))
        blk += 1
    return out


def text_encoder_mlp_layers(tokens: int, layers: int = 4) -> List[LinearSpec]:
    """The Qwen3 text encoder's MLP linears for `layers` layers (gate and up 2560 -> 9728, down
    9728 -> 2560; uint4, group 64 per the mlx article's component architecture). The layer count
    is representative, not taken from the pages."""
    common = dict(bits=4, group_size=64, scale_lo=0.002, scale_hi=0.01)
    out: List[LinearSpec] = []
    for layer in range(layers):
        for j, (lname, k, n) in enumerate((("gate", TE_H, TE_I), ("up", TE_H, TE_I), ("down", TE_I, TE_H))):
            out.append(LinearSpec(f"te{layer}.{lname}{tokens}", tokens, k, n, seed=layer,
                                  stream_base=10 * (j + 1), **common))
    return out


def klein_linears_small_m(tokens: int, bits: int) -> List[LinearSpec]:
    """The six distinct linear shapes of a denoise step (double-stream QKV d -> 3d, out d -> d,
    MLP-up d -> 3d, MLP-down 3d -> d; single-stream QKV+MLP-in d -> 6d, out 4d -> d) at a handful
    of tokens, as a decode-style or text-stream call would run them: ternary (P(0) = 0.4) or
    binary codes, group 128."""
    fmt = dict(bits=bits, group_size=128, p0=0.4, scale_lo=0.005, scale_hi=0.02)
    name = "ternary" if bits == 2 else "binary"
    out: List[LinearSpec] = []
    for j, (lname, k, n) in enumerate((("qkv", D, 3 * D), ("out", D, D), ("mlp_up", D, 3 * D), ("mlp_down", 3 * D, D),
                                       ("qkv_mlp_in", D, 6 * D), ("single_out", 4 * D, D))):
        out.append(LinearSpec(f"{lname}_m{tokens}_{name}", tokens, k, n, seed=tokens, stream_base=10 * (j + 1), **fmt))
    return out


WORKLOADS = {
    # tiny ternary, uniform codes, group 64
    "tiny_ternary_g64": [LinearSpec("tiny", 64, 256, 512, bits=2, group_size=64, p0=1.0 / 3.0)],
    # ternary fused-QKV at a 512x512 image: 1024 image + 512 text tokens
    "qkv_512sq_ternary_g128": [LinearSpec("qkv512", 1536, D, 3 * D, bits=2, group_size=128, p0=0.4)],
    # binary MLP up / down at a 1024x1024 image: 4096 image + 512 text tokens
    "mlp_1024sq_binary_g128": [
        LinearSpec("mlp_up1024", 4608, D, 3 * D, bits=1, group_size=128),
        LinearSpec("mlp_down1024", 4608, 3 * D, D, bits=1, group_size=128, stream_base=10),
    ],
    # Qwen3 text-encoder linears, asymmetric uint4, group 64
    "te_m512_uint4_g64": [
        LinearSpec("te_up512", 512, TE_H, TE_I, bits=4, group_size=64, scale_lo=0.002, scale_hi=0.01),
        LinearSpec("te_down512", 512, TE_I, TE_H, bits=4, group_size=64, scale_lo=0.002, scale_hi=0.01,
                   stream_base=10),
    ],
    "te_m16_uint4_g64": [
        LinearSpec("te_up16", 16, TE_H, TE_I, bits=4, group_size=64, scale_lo=0.002, scale_hi=0.01),
        LinearSpec("te_down16", 16, TE_I, TE_H, bits=4, group_size=64, scale_lo=0.002, scale_hi=0.01,
                   stream_base=10),
    ],
    # one denoise step's 80 ternary linears at a 1024x1024 image
    "klein_step_chain_1024sq_ternary_g128": chain_linears(),
    # its largest linear on its own: a single-stream block's fused QKV + MLP-in (profiling case)
    "klein_single_qkv_mlp_in_1024sq_ternary_g128": [chain_linears()[40]],
    # the same step with separate Q/K/V and add-Q/K/V projections: 100 linears
    "klein_step_linears100_1024sq_ternary_g128": chain_linears_separate_qkv(),
    # four text-encoder MLP layers (gate, up, down) at 512 and at 16 tokens
    "te_mlp4_m512_uint4_g64": text_encoder_mlp_layers(512),
    "te_mlp4_m16_uint4_g64": text_encoder_mlp_layers(16),
    # the small-M kernel's sustained rate: one uint4 linear at 16 tokens with a K long enough
    # (40 steps of 512) that start-up is amortized; not a model shape
    "smallm_steady_m16_uint4_g64": [LinearSpec("steady16", 16, 20480, 9472, bits=4, group_size=64,
                                               scale_lo=0.002, scale_hi=0.01)],
    # the transformer's ternary and binary linear shapes at 1, 4 and 16 tokens (HBM-bound)
    **{f"klein_linears_m{m}_{'ternary' if b == 2 else 'binary'}_g128": klein_linears_small_m(m, b)
       for b in (2, 1) for m in (1, 4, 16)},
}
