"""Seeded synthetic inputs for the packed-ternary path (test and bench infrastructure).

This module only *draws inputs*: dense trits, per-row fp16 scales, bf16 activations and int8
output-head weights. It holds none of the arithmetic of the method (no packing, no transport
coding, no products, no quantisation). Both the CPU oracle and the CUDA path receive their
inputs from here, so the two never feed each other.

Random numbers come from one counter-based generator, SplitMix64 (Steele, Lea & Flood,
"Fast splittable pseudorandom number generators", OOPSLA 2014): the i-th output of a stream
with 64-bit state `key` is ``mix64(key + (i + 1) * GAMMA)``. Every element of a tensor has its
own counter ``i = row * K + col``, so any row can be regenerated on its own and the CUDA
generator in ``synth/csrc/synth_gen.cu`` (integers only) reproduces the trits and head
weights bit for bit.

Distributions follow the pages' published weight statistics:
  * trits: P(0)=0.6263, P(+1)=0.1868, P(-1)=0.1869 over the 8B ternary lane
    (discuss.pytorch.kr topic 11456, section on reading the shipped container: 62.63% zero,
    +18.677% / -18.694%); the FFN gate and down projections of (0-based) layers 1-3 of the 8B
    use P(0)=0.71 with the rest split evenly (same section: 70.48% / 72.47% in "layers 2-4";
    aiatolah.com article, "Arquitetura": "camadas 1 a 3");
  * per-row scales: fp16, uniform in [0.01, 0.05);
  * activations: bf16 of a standard normal;
  * output head: int8 uniform in [-127, 127] with a per-row fp16 scale.
Geometry (layer counts, widths, vocabulary) is the Qwen3 geometry in the model table of the
same discuss.pytorch.kr page ("three models and one container").
"""
from __future__ import annotations

from fractions import Fraction
import math

import numpy as np

GAMMA = 0x9E3779B97F4A7C15
_MASK64 = (1 << 64) - 1
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)

# stream kinds: one independent family of streams per input type
KIND_TRIT, KIND_SCALE, KIND_ACT, KIND_HEAD, KIND_HEAD_SCALE = 0, 1, 2, 3, 4

DEFAULT_SEED = 0x7E2A2026

# P(0), P(+1) as exact decimals; P(-1) is the remainder.
P_DEFAULT = ("0.6263", "0.1868")
P_SPARSE_FFN = ("0.71", "0.145")


def _mix64_int(z: int) -> int:
    z &= _MASK64
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & _MASK64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & _MASK64
    return z ^ (z >> 31)


def mix64(z: np.ndarray) -> np.ndarray:
    """SplitMix64 output mix on a uint64 array (wrapping arithmetic)."""
    z = z.astype(np.uint64, copy=True)
    with np.errstate(over="ignore"):
        z ^= z >> np.uint64(30)
        z *= _M1
        z ^= z >> np.uint64(27)
        z *= _M2
        z ^= z >> np.uint64(31)
    return z


def stream_key(seed: int, kind: int, tid: int) -> int:
    """64-bit key of the stream for (seed, kind, tensor id): a SplitMix64 output itself."""
    return _mix64_int((seed + GAMMA * (1 + (kind << 24) + tid)) & _MASK64)


def uniform_u64(key: int, counters: np.ndarray) -> np.ndarray:
    """Outputs number counters+1 of the SplitMix64 stream whose state starts at key."""
    c = counters.astype(np.uint64, copy=False)
    with np.errstate(over="ignore"):
        z = np.uint64(key) + (c + np.uint64(1)) * np.uint64(GAMMA)
    return mix64(z)


def thresholds(p: tuple[str, str]) -> tuple[int, int]:
    """Integer thresholds (T0, T1): u < T0 -> 0, T0 <= u < T1 -> +1, u >= T1 -> -1."""
    p0, pp = Fraction(p[0]), Fraction(p[1])
    t0 = math.floor(p0 * (1 << 64))
    t1 = math.floor((p0 + pp) * (1 << 64))
    return t0, t1


def _row_counters(rows: np.ndarray, K: int) -> np.ndarray:
    return (rows.astype(np.uint64)[:, None] * np.uint64(K) + np.arange(K, dtype=np.uint64)[None, :])


def trits(seed: int, tid: int, N: int, K: int, p: tuple[str, str] = P_DEFAULT,
          rows: np.ndarray | None = None, chunk_rows: int = 4096) -> np.ndarray:
    """Dense trits int8[N or len(rows), K] in {-1, 0, +1}, row-major."""
    key = stream_key(seed, KIND_TRIT, tid)
    t0, t1 = (np.uint64(v) for v in thresholds(p))
    rows = np.arange(N, dtype=np.int64) if rows is None else np.asarray(rows, dtype=np.int64)
    out = np.empty((rows.size, K), dtype=np.int8)
    for r0 in range(0, rows.size, chunk_rows):
        rr = rows[r0:r0 + chunk_rows]
        u = uniform_u64(key, _row_counters(rr, K))
        blk = np.full(u.shape, -1, dtype=np.int8)
        blk[u < t1] = 1
        blk[u < t0] = 0
        out[r0:r0 + rr.size] = blk
    return out


def _f16_uniform(key: int, n: int) -> np.ndarray:
    u = uniform_u64(key, np.arange(n, dtype=np.uint64))
    f = (u >> np.uint64(40)).astype(np.float32) * np.float32(2.0 ** -24)   # exact, in [0, 1)
    f = np.float32(0.04) * f                                               # fp32 RN
    f = np.float32(0.01) + f                                               # fp32 RN
    return f.astype(np.float16).view(np.uint16)                            # fp16 RN-even


def row_scales(seed: int, tid: int, N: int) -> np.ndarray:
    """Per-row fp16 scales (bit patterns, uint16[N]), uniform in [0.01, 0.05)."""
    return _f16_uniform(stream_key(seed, KIND_SCALE, tid), N)


def head_scales(seed: int, tid: int, V: int) -> np.ndarray:
    """Per-row fp16 scales of the int8 output head (uint16[V])."""
    return _f16_uniform(stream_key(seed, KIND_HEAD_SCALE, tid), V)


def f32_to_bf16_bits(f: np.ndarray) -> np.ndarray:
    """Round-to-nearest-even fp32 -> bf16 bit patterns (finite inputs)."""
    b = np.ascontiguousarray(f, dtype=np.float32).view(np.uint32).astype(np.uint64)
    b = (b + np.uint64(0x7FFF) + ((b >> np.uint64(16)) & np.uint64(1))) >> np.uint64(16)
    return b.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def activations(seed: int, tid: int, M: int, K: int) -> np.ndarray:
    """bf16 bit patterns uint16[M, K] of N(0,1) draws (Box-Muller in fp64, then fp32 RN, then bf16 RN)."""
    key = stream_key(seed, KIND_ACT, tid)
    n = M * K
    c = np.arange(n, dtype=np.uint64) * np.uint64(2)
    u1 = uniform_u64(key, c)
    u2 = uniform_u64(key, c + np.uint64(1))
    U1 = ((u1 >> np.uint64(11)).astype(np.float64) + 1.0) * 2.0 ** -53     # (0, 1]
    U2 = (u2 >> np.uint64(11)).astype(np.float64) * 2.0 ** -53             # [0, 1)
    z = np.sqrt(-2.0 * np.log(U1)) * np.cos(2.0 * np.pi * U2)
    return f32_to_bf16_bits(z.astype(np.float32)).reshape(M, K)


def norm_gains(seed: int, tid: int, K: int) -> np.ndarray:
    """bf16 bit patterns uint16[K] of RMSNorm gains: 1 + N(0,1) / 8, drawn from the activation
    stream family with tensor ids of their own (the pages give no gain statistics)."""
    z = bf16_bits_to_f32(activations(seed, 1_000_000 + tid, 1, K)[0]).astype(np.float64)
    return f32_to_bf16_bits((1.0 + z / 8.0).astype(np.float32))


def residual(seed: int, tid: int, M: int, K: int) -> np.ndarray:
    """fp32 [M, K] rows of N(0,1) draws: the residual stream entering a decode chain."""
    return bf16_bits_to_f32(activations(seed, 2_000_000 + tid, M, K)).astype(np.float32)


def head_weights(seed: int, tid: int, V: int, K: int, rows: np.ndarray | None = None,
                 chunk_rows: int = 4096) -> np.ndarray:
    """int8[V or len(rows), K] uniform in [-127, 127]: (u mod 255) - 127."""
    key = stream_key(seed, KIND_HEAD, tid)
    rows = np.arange(V, dtype=np.int64) if rows is None else np.asarray(rows, dtype=np.int64)
    out = np.empty((rows.size, K), dtype=np.int8)
    for r0 in range(0, rows.size, chunk_rows):
        rr = rows[r0:r0 + chunk_rows]
        u = uniform_u64(key, _row_counters(rr, K))
        out[r0:r0 + rr.size] = ((u % np.uint64(255)).astype(np.int16) - 127).astype(np.int8)
    return out


# ---------------------------------------------------------------------------------------------
# Geometry: Qwen3 shapes of the two Neutrino-1 sizes (model table, discuss.pytorch.kr topic 11456).
# A linear is (name, N = out features, K = in features). Projection order fixes tensor ids:
# tid = layer * 7 + proj.
PROJ = ("q", "k", "v", "o", "gate", "up", "down")

GEOMETRY = {
    "8b": dict(layers=36, d=4096, ffn=12288, q_heads=32, kv_heads=8, head_dim=128, vocab=151936,
               tied_head=False),
    "0.6b": dict(layers=28, d=1024, ffn=3072, q_heads=16, kv_heads=8, head_dim=128, vocab=151936,
                 tied_head=True),
}


def linear_shapes(model: str) -> list[tuple[str, int, int]]:
    g = GEOMETRY[model]
    d, f, hq, hkv, hd = g["d"], g["ffn"], g["q_heads"], g["kv_heads"], g["head_dim"]
    return [("q", hq * hd, d), ("k", hkv * hd, d), ("v", hkv * hd, d), ("o", d, hq * hd),
            ("gate", f, d), ("up", f, d), ("down", d, f)]


def trit_probs(model: str, layer: int, proj: str) -> tuple[str, str]:
    """Sparse FFN gate/down in the 8B's (0-based) layers 1-3; the published average elsewhere."""
    if model == "8b" and 1 <= layer <= 3 and proj in ("gate", "down"):
        return P_SPARSE_FFN
    return P_DEFAULT


def tensor_id(layer: int, proj: str) -> int:
    return layer * 7 + PROJ.index(proj)


def head_tensor_id(model: str) -> int:
    return GEOMETRY[model]["layers"] * 7


# Fused launches: q|k|v share their input, gate|up share theirs (Qwen3 block structure).
FUSED_GROUPS = (("qkv", ("q", "k", "v")), ("o", ("o",)), ("gate_up", ("gate", "up")), ("down", ("down",)))


def act_tensor_id(model: str, layer: int, group: str) -> int:
    """Activation stream of one fused group input (4 per layer), then the head input."""
    names = [g for g, _ in FUSED_GROUPS]
    return layer * 4 + names.index(group)


def head_act_tensor_id(model: str) -> int:
    return GEOMETRY[model]["layers"] * 4
