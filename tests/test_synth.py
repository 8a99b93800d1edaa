"""The seeded input generator (synth/) against the published definitions it
names: SplitMix64 (Steele, Lea and Flood, OOPSLA 2014, with the splitmix64
finaliser constants) run as a sequential generator in Python integers, the
little-endian byte order of the code tensors, the scale recipe's binary32
roundings and bf16 rounding.  CPU only."""
import struct

import numpy as np
import torch

import synth

MASK = (1 << 64) - 1


def _splitmix64(state: int, n: int) -> list[int]:
    """The sequential generator: state += gamma, then the output finaliser."""
    out = []
    for _ in range(n):
        state = (state + 0x9E3779B97F4A7C15) & MASK
        z = state
        z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & MASK
        z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & MASK
        out.append(z ^ (z >> 31))
    return out


def _f32(v: float) -> float:
    return struct.unpack("<f", struct.pack("<f", v))[0]


def test_words_are_the_sequential_splitmix64_stream():
    for key in (0, 1, 0x0123456789ABCDEF, MASK, synth.stream_key(0, 3, synth.GATE_Q)):
        seq = _splitmix64(key, 40)
        assert [int(w) for w in synth.words(key, 0, 40)] == seq
        assert [int(w) for w in synth.words(key, 17, 9)] == seq[17:26]    # random access


def test_stream_keys_mix_seed_layer_and_kind():
    a = _splitmix64(0, 1)[0]             # mix64(gamma): the first output of state 0
    assert synth.mix64(np.array([0x9E3779B97F4A7C15], np.uint64))[0] == a
    keys = {synth.stream_key(s, l, k) for s in (0, 1) for l in range(4) for k in range(1, 11)}
    assert len(keys) == 2 * 4 * 10


def test_code_bytes_are_little_endian_words():
    key = synth.stream_key(5, 0, synth.UP_Q)
    w = _splitmix64(key, 6)
    want = b"".join(x.to_bytes(8, "little") for x in w)
    assert synth.code_bytes(key, 0, 48).tobytes() == want
    assert synth.code_bytes(key, 5, 30).tobytes() == want[5:35]


def test_scale_bits_follow_the_recipe():
    """u = (word >> 40) * 2^-24; v = fp32(fp32(u * 0.015f) + 0.005f); fp16(v)."""
    key = synth.stream_key(2, 1, synth.DOWN_S)
    words = _splitmix64(key, 500)
    lo, span = _f32(0.005), _f32(0.015)
    want = []
    for w in words:
        u = (w >> 40) * 2.0 ** -24
        v = _f32(_f32(u * span) + lo)
        want.append(int(np.float16(v).view(np.uint16)))   # fp32 -> fp16, nearest-even (exact input)
    got = synth.scale_bits(key, 0, 500)
    assert got.tolist() == want
    vals = got.view(np.float16).astype(np.float64)
    assert vals.min() >= 0.005 - 1e-5 and vals.max() <= 0.02 + 1e-5


def test_bf16_activations_match_torch_rounding():
    v = np.random.default_rng(3).standard_normal(5000).astype(np.float32) * np.float32(3)
    v = np.concatenate([v, np.array([np.inf, -np.inf, 0.0, -0.0, 3.3895314e38], np.float32)])
    want = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(synth.f32_to_bf16_bits(v), want)


def test_zipf_bias_is_a_log_rank_prior():
    b = synth.zipf_bias(0, 0, 256)
    ranks = np.rint(np.exp(-b.astype(np.float64) / 1.1)).astype(int)
    assert sorted(ranks.tolist()) == list(range(1, 257))
    assert np.allclose(b, (-1.1 * np.log(ranks)).astype(np.float32), rtol=0, atol=0)


def test_expert_bytes_match_the_worked_sizes():
    """Bytes of one expert (three matrices, codes + fp16 scales), the unit of
    the roofline's algorithmic bytes: 18,874,368 B of int4 codes + 2,359,296 B
    of group-32 scales at the GLM shape; 49,152 + 6,144 B for the tiny layer."""
    assert synth.DECODE_B1.expert_bytes() == 18_874_368 + 2_359_296 == 21_233_664
    assert synth.TINY.expert_bytes() == 49_152 + 6_144
    assert synth.DECODE_B1_GS64.expert_bytes() == 18_874_368 + 1_179_648      # one scale per 64 codes
    assert synth.DECODE_B1_INT8.expert_bytes() == 37_748_736 + 2_359_296      # one byte per code
    # a GLM layer with its shared expert, and the 16-layer stack, in GB
    assert round(257 * synth.DECODE_B1.expert_bytes() / 1e9, 3) == 5.457
    assert round(16 * 257 * synth.STACK16_B4.expert_bytes() / 1e9, 1) == 87.3
