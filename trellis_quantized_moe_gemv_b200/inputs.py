"""Seeded synthetic inputs for the trellis-coded MoE path.

This module only draws random numbers with the shapes and distributions of the
workloads; it holds none of the method's arithmetic (no decode, rotation, routing or
matrix product).  Both the CUDA path (tests, benchmark) and the CPU oracle read the
same arrays from here.

Workloads (named by what they are):
  * ``single_256``      one 256x256 matrix, K=2, x fp16 N(0,1), batch 1.
  * ``proj_1024x4096``  one 1024x4096 (out x in) expert projection at K = 2, 3, 4,
                        bf16 activations N(0,1), batches 1, 4, 16.
  * ``moe_decode_t16``  384 experts, D=4096, F=1024, top-8 routing from N(0,1)
                        logits, 16 tokens; widths 368 / 15 / 1 experts at K = 2/3/4
                        assigned by a seeded permutation (95.9 / 4.0 / 0.1 %, as in the
                        TrellisMX K2 Mix card's 14,731 / 608 / 21 of 15,360).
  * ``moe_prefill_t8192`` same layer shape, every expert K=3, 8192 tokens; logits
                        log p_e + Gumbel(0,1) with p_e proportional to rank_e^-1.1
                        (rank = seeded permutation of 1..384), so the top-8 is a
                        Plackett-Luce draw with Zipf(1.1) expert popularity.
  * ``moe_sweep``       the decode layer's widths at 1, 8, 64, 256, 2048, 16384 tokens,
                        N(0,1) logits.

Conventions of the stored format (16x16 tiles of 8*K uint32 words each, tiles in
row-major order, per-width groups with ascending expert ids) are those of the C-ABI
header; this module only fills such arrays with uniform random words.
"""
from dataclasses import dataclass, field
from typing import Optional, List

import numpy as np

E_EXPERTS = 384
D_HIDDEN = 4096
F_INTER = 1024
TOP_K = 8
WIDTH_SPLIT_DECODE = {2: 368, 3: 15, 4: 1}
SWEEP_TOKENS = (1, 8, 64, 256, 2048, 16384)
ZIPF_EXPONENT = 1.1


def words_per_matrix(rows: int, cols: int, K: int) -> int:
    """uint32 words of a rows x cols trellis matrix at K bits per weight."""
    return (rows // 16) * (cols // 16) * 8 * K


def random_bits(rng: np.random.Generator, rows: int, cols: int, K: int, count: int = 1):
    """Uniform random bit streams for `count` matrices: uint32 [count, words]."""
    n = words_per_matrix(rows, cols, K)
    raw = rng.bytes(4 * n * count)
    return np.frombuffer(raw, dtype=np.uint32).reshape(count, n).copy()


def random_scales(rng: np.random.Generator, shape) -> np.ndarray:
    """fp16 per-output-channel scales drawn from U[0.5, 1.5]."""
    return rng.uniform(0.5, 1.5, size=shape).astype(np.float16)


def to_bf16_values(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bfloat16 (ties to even); returns float32
    arrays whose values are exactly representable in bfloat16."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000
    return u.astype(np.uint32).view(np.float32)


def bf16_bits(x_bf16_values: np.ndarray) -> np.ndarray:
    """uint16 bit patterns of float32 values that are exact bfloat16 numbers."""
    return (np.ascontiguousarray(x_bf16_values, dtype=np.float32).view(np.uint32) >> 16).astype(np.uint16)


def random_activations(rng: np.random.Generator, shape, dtype: str = "bf16") -> np.ndarray:
    """N(0,1) activations rounded to bf16 or fp16; returned as float32 (bf16) or
    float16 (fp16) arrays of the exact rounded values."""
    x = rng.standard_normal(size=shape).astype(np.float32)
    if dtype == "bf16":
        return to_bf16_values(x)
    if dtype == "f16":
        return x.astype(np.float16)
    raise ValueError(dtype)


def normal_logits(rng: np.random.Generator, T: int, E: int = E_EXPERTS) -> np.ndarray:
    """Router logits N(0,1), float32 [T, E]."""
    return rng.standard_normal(size=(T, E)).astype(np.float32)


def zipf_gumbel_logits(rng: np.random.Generator, T: int, E: int = E_EXPERTS,
                       s: float = ZIPF_EXPONENT) -> np.ndarray:
    """Router logits log p_e + Gumbel(0,1), p_e proportional to rank_e^-s with rank a
    seeded permutation of 1..E; float32 [T, E]."""
    rank = rng.permutation(E) + 1
    p = rank.astype(np.float64) ** (-s)
    p /= p.sum()
    gumbel = rng.gumbel(0.0, 1.0, size=(T, E))
    return (np.log(p)[None, :] + gumbel).astype(np.float32)


@dataclass
class WidthGroup:
    """Experts of one width, in ascending global id, and their stored arrays."""
    K: int
    ids: np.ndarray            # int32 [n], ascending
    gate: np.ndarray           # uint32 [n, F/16 * D/16 * 8K]
    up: np.ndarray             # uint32 [n, F/16 * D/16 * 8K]
    down: np.ndarray           # uint32 [n, D/16 * F/16 * 8K]
    s_gate: np.ndarray         # fp16 [n, F]
    s_up: np.ndarray           # fp16 [n, F]
    s_down: np.ndarray         # fp16 [n, D]


@dataclass
class SyntheticLayer:
    E: int
    D: int
    F: int
    expert_bits: np.ndarray    # int32 [E]: K of every expert
    groups: List[WidthGroup] = field(default_factory=list)
    name: str = ""
    seed: int = 0
    # Layer sign vectors of the two-sided transform (int8, +1/-1), shared by every
    # expert: x [D], gu [F], h [F], y [D]; None for the input-side-only layer.
    signs: Optional[dict] = None
    # codebook of the bit streams: "t16" or "pair_e4m3" (same stored layout, K bits per weight)
    codebook: str = "t16"


def width_map(rng: np.random.Generator, E: int, split: dict) -> np.ndarray:
    """Assign widths to experts by a seeded permutation: the first split[2] experts of
    the permutation get K=2, the next split[3] K=3, the rest K=4."""
    assert sum(split.values()) == E
    order = rng.permutation(E)
    bits = np.empty(E, dtype=np.int32)
    start = 0
    for K in sorted(split):
        bits[order[start:start + split[K]]] = K
        start += split[K]
    return bits


def make_layer(seed: int, E: int = E_EXPERTS, D: int = D_HIDDEN, F: int = F_INTER,
               split: dict = None, uniform_K: int = None, name: str = "",
               codebook: str = "t16") -> SyntheticLayer:
    """A synthetic trellis-coded MoE layer with uniform random bit streams and U[0.5,1.5]
    fp16 scales.  Either `split` (experts per width) or `uniform_K` is given; `codebook`
    names how the streams are read ("t16" or "pair_e4m3")."""
    rng = np.random.default_rng(seed)
    if uniform_K is not None:
        expert_bits = np.full(E, uniform_K, dtype=np.int32)
    else:
        expert_bits = width_map(rng, E, split)
    layer = SyntheticLayer(E=E, D=D, F=F, expert_bits=expert_bits, name=name, seed=seed, codebook=codebook)
    for K in (2, 3, 4):
        ids = np.nonzero(expert_bits == K)[0].astype(np.int32)
        if ids.size == 0:
            continue
        n = ids.size
        layer.groups.append(WidthGroup(
            K=K, ids=ids,
            gate=random_bits(rng, F, D, K, n), up=random_bits(rng, F, D, K, n),
            down=random_bits(rng, D, F, K, n),
            s_gate=random_scales(rng, (n, F)), s_up=random_scales(rng, (n, F)),
            s_down=random_scales(rng, (n, D))))
    return layer


# ----------------------------------------------------------------------------- workloads

def single_256(seed: int = 1001):
    """One 256x256 matrix at K=2, fp16 x N(0,1) [1, 256]."""
    rng = np.random.default_rng(seed)
    bits = random_bits(rng, 256, 256, 2)[0]
    scales = random_scales(rng, 256)
    x = random_activations(rng, (1, 256), "f16")
    return dict(rows=256, cols=256, K=2, bits=bits, scales=scales, x=x)


def proj_1024x4096(K: int, batch: int, seed: int = 1002):
    """One 1024x4096 projection at width K with bf16 x N(0,1) [batch, 4096]."""
    rng = np.random.default_rng(seed * 100 + K * 10 + batch)
    bits = random_bits(rng, 1024, 4096, K)[0]
    scales = random_scales(rng, 1024)
    x = random_activations(rng, (batch, 4096), "bf16")
    return dict(rows=1024, cols=4096, K=K, bits=bits, scales=scales, x=x)


def moe_decode_t16(seed: int = 1003, T: int = 16, E: int = E_EXPERTS, D: int = D_HIDDEN,
                   F: int = F_INTER, split: dict = None):
    """Mixed-width decode layer (368/15/1 experts at K=2/3/4), 16 tokens."""
    split = split or WIDTH_SPLIT_DECODE
    layer = make_layer(seed, E, D, F, split=split, name="moe_decode_t16")
    rng = np.random.default_rng(seed + 7)
    x = random_activations(rng, (T, D), "bf16")
    logits = normal_logits(rng, T, E)
    return dict(layer=layer, x=x, logits=logits, k=TOP_K)


def moe_prefill_t8192(seed: int = 1004, T: int = 8192, E: int = E_EXPERTS,
                      D: int = D_HIDDEN, F: int = F_INTER):
    """All-K=3 layer, 8192 tokens with Zipf(1.1)-skewed top-8 routing."""
    layer = make_layer(seed, E, D, F, uniform_K=3, name="moe_prefill_t8192")
    rng = np.random.default_rng(seed + 7)
    x = random_activations(rng, (T, D), "bf16")
    logits = zipf_gumbel_logits(rng, T, E)
    return dict(layer=layer, x=x, logits=logits, k=TOP_K)


def moe_sweep_tokens(T: int, seed: int = 1005, layer: SyntheticLayer = None):
    """Decode-width layer at T tokens with N(0,1) logits (the batch sweep)."""
    layer = layer or make_layer(seed, split=WIDTH_SPLIT_DECODE, name="moe_sweep")
    rng = np.random.default_rng(seed * 1000 + T)
    x = random_activations(rng, (T, layer.D), "bf16")
    logits = normal_logits(rng, T, layer.E)
    return dict(layer=layer, x=x, logits=logits, k=TOP_K)


def random_signs(rng: np.random.Generator, n: int) -> np.ndarray:
    """Uniform random +1/-1 (int8) of length n."""
    return np.where(rng.integers(0, 2, size=n) == 1, 1, -1).astype(np.int8)


def with_signs(layer: SyntheticLayer, seed: int) -> SyntheticLayer:
    """The same layer carrying seeded layer sign vectors (x, gu, h, y)."""
    rng = np.random.default_rng(seed)
    layer.signs = dict(x=random_signs(rng, layer.D), gu=random_signs(rng, layer.F),
                       h=random_signs(rng, layer.F), y=random_signs(rng, layer.D))
    return layer


def small_layer(seed: int, E: int = 12, D: int = 256, F: int = 128, split: dict = None,
                uniform_K: int = None, codebook: str = "t16"):
    """A small layer for fast parity tests (dimensions multiples of 128)."""
    if split is None and uniform_K is None:
        split = {2: E - 3, 3: 2, 4: 1}
    return make_layer(seed, E, D, F, split=split, uniform_K=uniform_K, name="small", codebook=codebook)


def moe_prefill_t8192_fp8(seed: int = 1006, T: int = 8192, E: int = E_EXPERTS,
                          D: int = D_HIDDEN, F: int = F_INTER):
    """The prefill layer shape with pair-trellis (E4M3) streams, every expert K=3, 8192
    tokens with Zipf(1.1)-skewed top-8 routing."""
    layer = make_layer(seed, E, D, F, uniform_K=3, name="moe_prefill_t8192_fp8", codebook="pair_e4m3")
    rng = np.random.default_rng(seed + 7)
    x = random_activations(rng, (T, D), "bf16")
    logits = zipf_gumbel_logits(rng, T, E)
    return dict(layer=layer, x=x, logits=logits, k=TOP_K)
