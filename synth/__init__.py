"""Seeded synthetic inputs for the int4 routed-expert MoE layer.

This module is the one piece shared by the CUDA path's tests and by the CPU
oracle. It draws inputs and holds none of the layer's arithmetic: no
dequantisation, routing, union, FFN or combine happens here.

Workload shapes follow the GLM-5.2 MoE layer that the Colibri pages describe
("Come funziona" / "L'idea": 256 routed experts per MoE layer, int4 container,
shared experts always resident); the distributions (codes uniform in [-8, 7],
fp16 group-32 scales uniform in [0.005, 0.02], activations N(0, 1), router
weights N(0, 0.02)) are the workload statement's.

Two generators:

* Expert weights (int4 codes and fp16 scales) are far too large to draw on the
  host for every run (5.5 GB per layer, 87 GB for the 16-layer stack), so they
  come from a counter-based generator, SplitMix64 (Steele, Lea and Flood,
  "Fast splittable pseudorandom number generators", OOPSLA 2014; the 64-bit
  finaliser with the constants Vigna published for splitmix64).  Word ``i`` of
  a stream with key ``K`` is ``mix64(K + (i + 1) * GAMMA)``.  Any element can
  be produced independently, so the CUDA fill kernel (``synth/csrc``) and this
  numpy version produce bit-identical tensors and the oracle regenerates only
  the experts it needs.
* Small dense tensors (activations, router weights, logits, the Zipf
  permutation) come from numpy's PCG64 seeded by ``SeedSequence`` and are
  copied to the device.

Element encodings produced here (the container format):
  * codes: byte ``j`` of a code tensor is byte ``j % 8`` (little-endian) of
    word ``j // 8``.  Every byte value is equally likely, so both nibbles are
    uniform over the 16 two's-complement codes [-8, 7].
  * scales: element ``j`` takes ``u = (word_j >> 40) * 2**-24`` (exact in
    fp32), forms ``0.005f + 0.015f * u`` with two separately rounded fp32
    operations (multiply, then add) and rounds that to fp16 (nearest-even).
"""
from __future__ import annotations

import dataclasses

import numpy as np

GAMMA = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)

# Stream kinds (part of each stream's key).
GATE_Q, UP_Q, DOWN_Q, GATE_S, UP_S, DOWN_S = 1, 2, 3, 4, 5, 6
ROUTER_W, X_IN, LOGITS_IN, BIAS_PERM = 7, 8, 9, 10

SCALE_LO = np.float32(0.005)
SCALE_SPAN = np.float32(0.015)


def mix64(z: np.ndarray) -> np.ndarray:
    """SplitMix64 output finaliser on a uint64 array (wrapping arithmetic)."""
    z = np.asarray(z, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = (z ^ (z >> np.uint64(30))) * _M1
        z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def stream_key(seed: int, layer: int, kind: int) -> int:
    """64-bit key of the stream for (seed, layer, tensor kind)."""
    a = mix64(np.array([seed & 0xFFFFFFFFFFFFFFFF], dtype=np.uint64))[0]
    b = np.uint64(((layer & 0xFFFFFF) << 8) | (kind & 0xFF))
    return int(mix64(np.array([a ^ b], dtype=np.uint64))[0])


def words(key: int, start: int, count: int) -> np.ndarray:
    """Words ``start .. start+count-1`` of the SplitMix64 stream ``key``."""
    idx = np.arange(start + 1, start + count + 1, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = np.uint64(key) + idx * GAMMA
    return mix64(z)


def code_bytes(key: int, start: int, count: int) -> np.ndarray:
    """Bytes ``start .. start+count-1`` of a code tensor (uint8; int4 or int8 codes)."""
    w0 = start // 8
    w1 = (start + count + 7) // 8
    w = words(key, w0, w1 - w0)
    b = w.view(np.uint8)  # little-endian host: byte j%8 of word j//8
    off = start - w0 * 8
    return b[off:off + count].copy()


def scale_bits(key: int, start: int, count: int) -> np.ndarray:
    """fp16 bit patterns of scale elements ``start .. start+count-1`` (uint16)."""
    w = words(key, start, count)
    u = (w >> np.uint64(40)).astype(np.float32) * np.float32(2.0 ** -24)
    v = (u * SCALE_SPAN).astype(np.float32)
    v = (v + SCALE_LO).astype(np.float32)
    return v.astype(np.float16).view(np.uint16)


def _rng(seed: int, layer: int, kind: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, layer, kind])))


def f32_to_bf16_bits(v: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (nearest, ties to even); returns uint16 bits.

    Input generation only: used to store the N(0,1) activations as bf16."""
    v = np.ascontiguousarray(v, dtype=np.float32)
    u = v.view(np.uint32).astype(np.uint64)
    lsb = (u >> np.uint64(16)) & np.uint64(1)
    r = (u + np.uint64(0x7FFF) + lsb) >> np.uint64(16)
    nan = np.isnan(v)
    out = r.astype(np.uint16)
    out[nan] = 0x7FC0
    return out


def normal_bf16(seed: int, layer: int, kind: int, shape) -> np.ndarray:
    """N(0,1) activations stored as bf16 bit patterns (uint16)."""
    z = _rng(seed, layer, kind).standard_normal(size=shape, dtype=np.float32)
    return f32_to_bf16_bits(z)


def normal_f32(seed: int, layer: int, kind: int, shape, std: float) -> np.ndarray:
    z = _rng(seed, layer, kind).standard_normal(size=shape, dtype=np.float32)
    return (z * np.float32(std)).astype(np.float32)


def zipf_bias(seed: int, layer: int, n_experts: int, s: float = 1.1) -> np.ndarray:
    """Additive per-expert router bias from a Zipf(s) rank profile.

    Expert ``e`` gets rank ``r_e`` from a seeded permutation of 1..E and bias
    ``-s * ln(r_e)`` (fp32): an additive log-prior, so softmax probabilities
    scale as ``r_e ** -s``."""
    r = _rng(seed, layer, BIAS_PERM).permutation(n_experts) + 1
    return (-s * np.log(r.astype(np.float64))).astype(np.float32)


@dataclasses.dataclass(frozen=True)
class LayerShape:
    """Shape of one routed-expert MoE layer and of the batch it sees."""
    name: str
    hidden: int          # H
    inter: int           # I (expert intermediate size)
    n_experts: int       # E routed experts
    top_k: int           # k
    n_shared: int        # S shared experts (ids E .. E+S-1), weight 1.0
    tokens: int          # T
    layers: int = 1
    group: int = 32
    zipf_bias: bool = False
    logits_in: bool = False   # logits drawn i.i.d. N(0,1) instead of x @ W_r^T
    prenorm: bool = False     # stack: pre-RMSNorm and residual between layers
    bits: int = 4             # code container: int4 (two codes per byte) or int8 (one per byte)

    @property
    def n_total(self) -> int:
        return self.n_experts + self.n_shared

    def expert_bytes(self) -> int:
        """Codes + fp16 scales of one expert (gate, up and down)."""
        h, i, g = self.hidden, self.inter, self.group
        return 3 * (h * i * self.bits // 8) + 3 * (h * i // g) * 2


# The five workloads (sizes of the GLM-5.2-shaped layer; tiny case for fast parity).
TINY = LayerShape("tiny_h256_i128_e16_k2_t4", 256, 128, 16, 2, 0, 4)
DECODE_B1 = LayerShape("glm52_layer_decode_b1", 6144, 2048, 256, 8, 1, 1)
DECODE_B64 = LayerShape("glm52_layer_decode_b64_zipf", 6144, 2048, 256, 8, 1, 64, zipf_bias=True)
PREFILL_4096 = LayerShape("glm52_layer_prefill_4096", 6144, 2048, 256, 8, 1, 4096, logits_in=True)
STACK16_B4 = LayerShape("glm52_stack16_decode_b4", 6144, 2048, 256, 8, 1, 4, layers=16, prenorm=True)
# Same per-step bytes as DECODE_B1 (8 routed + 1 shared expert, 191 MB > L2) with
# only 16 routed experts resident: small enough for profiler captures.
DECODE_B1_E16 = LayerShape("glm52_layer_decode_b1_e16", 6144, 2048, 16, 8, 1, 1)
# A decode batch of 64 tokens with Zipf-biased routing over 32 routed experts
# (about 16 tokens per expert, several 16-token blocks on the popular ones;
# 0.7 GB resident): split-K units of the same shape as DECODE_B64's, for
# profiler captures.
DECODE_B64_E32 = LayerShape("glm52_layer_decode_b64_zipf_e32", 6144, 2048, 32, 8, 1, 64, zipf_bias=True)
# Batch-1 decode with the Zipf router bias of DECODE_B64: a workload whose hot
# experts recur, for the host-RAM expert tier.
DECODE_B1_ZIPF = LayerShape("glm52_layer_decode_b1_zipf", 6144, 2048, 256, 8, 1, 1, zipf_bias=True)
# Prefill tiles of the same shape as PREFILL_4096 (~128 tokens on every expert;
# 32 routed + 1 shared expert resident, 0.7 GB): for profiler captures.
PREFILL_512_E32 = LayerShape("glm52_layer_prefill_512_e32", 6144, 2048, 32, 8, 1, 512, logits_in=True)
# The same layer in the group-scaled gs64 container (one fp16 scale per 64
# codes along K; 20,054,016 bytes per expert instead of 21,233,664).
DECODE_B1_GS64 = LayerShape("glm52_layer_decode_b1_gs64", 6144, 2048, 256, 8, 1, 1, group=64)
PREFILL_4096_GS64 = LayerShape("glm52_layer_prefill_4096_gs64", 6144, 2048, 256, 8, 1, 4096, group=64,
                               logits_in=True)
# The same layer with int8 codes (the container the README requires for the MTP
# head, whose drafts are decoded in batches of 1..4): 37,748,736 + 2,359,296
# bytes per expert.
DECODE_B1_INT8 = LayerShape("glm52_layer_int8_decode_b1", 6144, 2048, 256, 8, 1, 1, bits=8)
# The prefill layer with the router logits computed in the step (x . W_r^T for
# 4096 tokens: 12.9 GFLOP in fp32) instead of given.
PREFILL_4096_ROUTER = LayerShape("glm52_layer_prefill_4096_router", 6144, 2048, 256, 8, 1, 4096)
WORKLOADS = {s.name: s for s in (TINY, DECODE_B1, DECODE_B64, PREFILL_4096, STACK16_B4, DECODE_B1_E16,
                                 DECODE_B64_E32, PREFILL_512_E32, DECODE_B1_GS64, PREFILL_4096_GS64, DECODE_B1_INT8,
                                 PREFILL_4096_ROUTER, DECODE_B1_ZIPF)}


class LayerInputs:
    """Host-side (numpy) view of one layer's seeded inputs.

    Expert tensors are produced lazily per expert so the oracle never
    materialises a whole 5.5 GB layer."""

    def __init__(self, shape: LayerShape, seed: int = 0, layer: int = 0):
        self.shape, self.seed, self.layer = shape, seed, layer
        self.keys = {k: stream_key(seed, layer, k) for k in (GATE_Q, UP_Q, DOWN_Q, GATE_S, UP_S, DOWN_S)}

    # flat element counts per expert for each tensor kind
    def per_expert(self, kind: int) -> int:
        h, i, g = self.shape.hidden, self.shape.inter, self.shape.group
        cb = h * i * self.shape.bits // 8
        return {GATE_Q: cb, UP_Q: cb, DOWN_Q: cb,
                GATE_S: i * h // g, UP_S: i * h // g, DOWN_S: h * i // g}[kind]

    def expert_codes(self, kind: int, e: int) -> np.ndarray:
        """uint8 [rows, K*bits/8] codes of expert ``e`` (gate/up: rows=I, K=H; down: rows=H, K=I)."""
        n = self.per_expert(kind)
        h, i = self.shape.hidden, self.shape.inter
        rows, k = (h, i) if kind == DOWN_Q else (i, h)
        return code_bytes(self.keys[kind], e * n, n).reshape(rows, k * self.shape.bits // 8)

    def expert_scales(self, kind: int, e: int) -> np.ndarray:
        """uint16 fp16 bits [rows, K/group] of expert ``e``."""
        n = self.per_expert(kind)
        h, i, g = self.shape.hidden, self.shape.inter, self.shape.group
        rows, k = (h, i) if kind == DOWN_S else (i, h)
        return scale_bits(self.keys[kind], e * n, n).reshape(rows, k // g)

    def router_w(self) -> np.ndarray:
        return normal_f32(self.seed, self.layer, ROUTER_W, (self.shape.n_experts, self.shape.hidden), 0.02)

    def bias(self):
        return zipf_bias(self.seed, self.layer, self.shape.n_experts) if self.shape.zipf_bias else None

    def logits(self) -> np.ndarray:
        """i.i.d. N(0,1) router logits [T, E] for the prefill workload."""
        return normal_f32(self.seed, self.layer, LOGITS_IN, (self.shape.tokens, self.shape.n_experts), 1.0)


def activations(shape: LayerShape, seed: int = 0, batch: int = 0) -> np.ndarray:
    """bf16 bits [T, H] of the layer input (batch index selects a fresh draw)."""
    return normal_bf16(seed, 1000 + batch, X_IN, (shape.tokens, shape.hidden))


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)

