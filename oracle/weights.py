"""Oracle side of the counter-based weight generator (NumPy, fp64).

TEST INFRASTRUCTURE ONLY -- see oracle/__init__.py for who may use it.

The pages fix only "random init N(0, 0.02)" for the models (PHOTON
workload descriptions).  This generator is this project's published
definition of that draw; the CUDA library implements the same definition on
its own side, and the two are compared byte for byte through the library's
tensor export.

Definition (all integer arithmetic modulo 2^64):

  gamma = 0x9E3779B97F4A7C15
  mix(z):  z ^= z >> 30; z *= 0xBF58476D1CE4E5B9;
           z ^= z >> 27; z *= 0x94D049BB133111EB; z ^= z >> 31
  (mix(x + gamma*k) for k = 1, 2, ... is Vigna's SplitMix64 stream)

  tensor t (0-based, in the order of `tensor_specs`) has key
      base_t = mix(seed + gamma * (t + 1))
  element e (row-major index in the tensor's stated shape) draws
      z = mix(base_t + gamma * (e + 1))
      S = sum of the four 16-bit fields of z            (0 <= S <= 262140)
      w = fp64(S - 131070) * K,   K = (init_std * 1.7320508075688772) / 65536
  with init_std taken as its fp32 value (the type of the config field in
  the library's C ABI) and K evaluated in fp64, left to right.

  S/65536 - 2 is the Irwin-Hall sum of four uniforms on (0, 1) minus its
  mean (variance 1/3), so w has mean 0 and standard deviation init_std,
  a bounded bell-shaped stand-in for N(0, init_std^2).  Only exact integer
  operations and one fp64 multiply are involved, so every implementation
  produces the same bits.  w is then rounded to fp32 (round to nearest
  even) and, for bf16 models, from fp32 to bf16 (round to nearest even).
  RMSNorm gains are exactly 1.0 and consume a tensor index but no draws.
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

GAMMA = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)
SQRT3 = 1.7320508075688772


def mix64(z: np.ndarray) -> np.ndarray:
    """SplitMix64 output function applied elementwise to a uint64 array."""
    z = np.asarray(z, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = z ^ (z >> np.uint64(30))
        z = z * _M1
        z = z ^ (z >> np.uint64(27))
        z = z * _M2
        z = z ^ (z >> np.uint64(31))
    return z


def splitmix64_stream(state: int, n: int) -> np.ndarray:
    """First n outputs of SplitMix64 started from `state` (for the published test vectors)."""
    k = np.arange(1, n + 1, dtype=np.uint64)
    with np.errstate(over="ignore"):
        return mix64(np.uint64(state) + GAMMA * k)


def tensor_specs(cfg) -> list[tuple[str, tuple[int, ...], str]]:
    """(name, shape, kind) of every parameter tensor in generator order.

    Linear maps are stored as [out, in] and applied as y = x W^T.
    Converters are [C*d, d] with output element j*d + i (vector j, feature i).
    kind is "normal" (drawn) or "ones" (RMSNorm gain).
    """
    d, V, f = cfg.d_model, cfg.vocab, cfg.mlp_mult * cfg.d_model
    specs: list[tuple[str, tuple[int, ...], str]] = []

    def blocks(prefix: str, n: int) -> None:
        for l in range(n):
            p = f"{prefix}.{l}."
            specs.extend([
                (p + "g_attn", (d,), "ones"),
                (p + "wq", (d, d), "normal"),
                (p + "wk", (d, d), "normal"),
                (p + "wv", (d, d), "normal"),
                (p + "wo", (d, d), "normal"),
                (p + "g_mlp", (d,), "ones"),
                (p + "w1", (f, d), "normal"),
                (p + "w2", (d, f), "normal"),
            ])

    specs.append(("embed", (V, d), "normal"))
    specs.append(("chunker1", (d, cfg.C1 * d), "normal"))
    blocks("enc1", cfg.L1)
    specs.append(("enc1.g_final", (d,), "ones"))
    specs.append(("chunker2", (d, cfg.C2 * d), "normal"))
    blocks("top", cfg.Ltop)
    specs.append(("top.g_final", (d,), "ones"))
    specs.append(("converter2", (cfg.C2 * d, d), "normal"))
    blocks("dec2", cfg.Ld2)
    specs.append(("dec2.g_final", (d,), "ones"))
    specs.append(("converter1", (cfg.C1 * d, d), "normal"))
    blocks("dec1", cfg.Ld1)
    specs.append(("dec1.g_final", (d,), "ones"))
    specs.append(("head", (V, d), "normal"))
    return specs


def round_fp32_to_bf16(x32: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (nearest, ties to even); returned as float32.

    Finite inputs only (the generator never produces inf or NaN).
    """
    u = np.ascontiguousarray(x32, dtype=np.float32).view(np.uint32).astype(np.uint64)
    lsb = (u >> np.uint64(16)) & np.uint64(1)
    r = ((u + np.uint64(0x7FFF) + lsb) >> np.uint64(16)) << np.uint64(16)
    return r.astype(np.uint32).view(np.float32)


def draw_tensor(seed: int, t: int, numel: int, init_std: float, dtype: str,
                chunk: int = 1 << 18) -> np.ndarray:
    """Values of tensor t as float32 (already rounded to the storage precision)."""
    K = (float(np.float32(init_std)) * SQRT3) / 65536.0
    with np.errstate(over="ignore"):
        base = mix64(np.uint64(seed) + GAMMA * np.uint64(t + 1))
    out = np.empty(numel, dtype=np.float32)
    mask = np.uint64(0xFFFF)

    def fill(lo: int) -> None:
        # elements lo..hi-1; independent of every other range
        hi = min(numel, lo + chunk)
        e1 = np.arange(lo + 1, hi + 1, dtype=np.uint64)
        with np.errstate(over="ignore"):
            z = mix64(base + GAMMA * e1)
        s = ((z & mask) + ((z >> np.uint64(16)) & mask)
             + ((z >> np.uint64(32)) & mask) + (z >> np.uint64(48)))
        w64 = (s.astype(np.int64) - 131070).astype(np.float64) * K
        out[lo:hi] = w64.astype(np.float32)

    starts = range(0, numel, chunk)
    if len(starts) > 1:
        # NumPy releases the GIL inside these array operations
        with ThreadPoolExecutor(max_workers=min(len(starts), os.cpu_count() or 1)) as ex:
            list(ex.map(fill, starts))
    else:
        for lo in starts:
            fill(lo)
    if dtype == "bf16":
        out = round_fp32_to_bf16(out)
    return out


def make_weights(cfg, seed: int) -> dict[str, np.ndarray]:
    """All parameters as fp64 arrays holding the rounded storage values."""
    w: dict[str, np.ndarray] = {}
    for t, (name, shape, kind) in enumerate(tensor_specs(cfg)):
        n = int(np.prod(shape))
        if kind == "ones":
            v = np.ones(n, dtype=np.float64)
        else:
            v = draw_tensor(seed, t, n, cfg.init_std, cfg.dtype).astype(np.float64)
        w[name] = v.reshape(shape)
    return w
