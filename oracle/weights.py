"""Oracle side of the counter-based weight generator (NumPy, fp64).

TEST INFRASTRUCTURE ONLY -- see oracle/__init__.py for who may use it.

The pages fix only "random init N(0, 0.02)" for the models (PHOTON
workload descriptions).  This generator is this project's published
definition of that draw; the CUDA library implements the same definition on
its own side, and the two are compared byte for byte through the library's
tensor export.

Definition (integer arithmetic modulo 2^64; floating point is IEEE fp64
with round-to-nearest-even, every operation rounded on its own, no fused
multiply-add):

  gamma = 0x9E3779B97F4A7C15
  mix(z):  z ^= z >> 30; z *= 0xBF58476D1CE4E5B9;
           z ^= z >> 27; z *= 0x94D049BB133111EB; z ^= z >> 31
  (mix(x + gamma*k) for k = 1, 2, ... is Vigna's SplitMix64 stream)

  tensor t (0-based, in the order of `tensor_specs`) has key
      base_t = mix(seed + gamma * (t + 1))
  element e (row-major index in the tensor's stated shape) has key
      key_e = mix(base_t + gamma * (e + 1))
  and draws by Marsaglia's polar method: for attempt a = 0, 1, ..., 63
      x = (mix(key_e + gamma * (2a + 1)) >> 11) * 2^-52 - 1      (exact, in [-1, 1))
      y = (mix(key_e + gamma * (2a + 2)) >> 11) * 2^-52 - 1
      s = x*x + y*y
  until 0 < s < 1 (after 64 rejected attempts, which has probability
  (1 - pi/4)^64 < 1e-42, w = 0); then
      w = (x * sqrt((-2 * ln s) / s)) * sigma,   sigma = fp64 of the fp32 init_std
  (the first variable of the polar pair, a standard normal times sigma).
  ln s is evaluated as its own definition, not by a library routine:
      s = m * 2^k with m in [1, 2) (the exponent and mantissa fields);
      if m >= 0x1.6a09e667f3bcdp+0 (sqrt 2 rounded): m = m/2, k = k+1;
      f = (m - 1) / (m + 1);  ln m = 2 * atanh(f) = 2f (1 + f^2/3 + f^4/5 + ...),
      the series summed by Horner's rule over the coefficients 1/(2i+1),
      i = 11 down to 0 (each the rounded quotient), as p = p * f^2 + c_i;
      ln m = (2f) * p;   ln s = k * LN2 + ln m,   LN2 = 0x1.62e42fefa39efp-1.
  With |f| <= 0.1716 the dropped terms are below 1e-20 of ln m.
  Only exact integer steps and correctly rounded +, -, *, / and sqrt are
  involved, so every implementation that follows the definition produces
  the same bits.  w is then rounded to fp32 (round to nearest even) and, for
  bf16 models, from fp32 to bf16 (round to nearest even).  RMSNorm gains are
  exactly 1.0 and consume a tensor index but no draws.
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

GAMMA = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)
LN2 = float.fromhex("0x1.62e42fefa39efp-1")
SQRT2 = float.fromhex("0x1.6a09e667f3bcdp+0")
ATANH_COEF = [1.0 / (2 * i + 1) for i in range(12)]
MAX_ATTEMPTS = 64


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


def log_series(s: np.ndarray) -> np.ndarray:
    """ln s for positive normal fp64 s, by the exponent split and the atanh
    series of the definition above (elementwise, fp64)."""
    s = np.asarray(s, dtype=np.float64)
    bits = s.view(np.int64)
    k = ((bits >> 52) & 0x7FF) - 1023
    m = ((bits & 0x000FFFFFFFFFFFFF) | 0x3FF0000000000000).view(np.float64)
    big = m >= SQRT2
    m = np.where(big, m * 0.5, m)
    k = np.where(big, k + 1, k)
    f = (m - 1.0) / (m + 1.0)
    f2 = f * f
    p = np.full_like(f, ATANH_COEF[-1])
    for c in reversed(ATANH_COEF[:-1]):
        p = p * f2
        p = p + c
    lnm = (2.0 * f) * p
    return k.astype(np.float64) * LN2 + lnm


def _uniform_pm1(z: np.ndarray) -> np.ndarray:
    """(z >> 11) * 2^-52 - 1, exact."""
    return (z >> np.uint64(11)).astype(np.float64) * (2.0 ** -52) - 1.0


def polar_normal(keys: np.ndarray) -> np.ndarray:
    """Standard normal variables of the definition for element keys (uint64)."""
    n = keys.size
    out = np.zeros(n, dtype=np.float64)
    todo = np.arange(n)
    for att in range(MAX_ATTEMPTS):
        if todo.size == 0:
            break
        kk = keys[todo]
        with np.errstate(over="ignore"):
            x = _uniform_pm1(mix64(kk + GAMMA * np.uint64(2 * att + 1)))
            y = _uniform_pm1(mix64(kk + GAMMA * np.uint64(2 * att + 2)))
        s = x * x
        s = s + y * y
        ok = (s > 0.0) & (s < 1.0)
        sa, xa = s[ok], x[ok]
        r = np.sqrt((-2.0 * log_series(sa)) / sa)
        out[todo[ok]] = xa * r
        todo = todo[~ok]
    return out


def draw_tensor(seed: int, t: int, numel: int, init_std: float, dtype: str,
                chunk: int = 1 << 18) -> np.ndarray:
    """Values of tensor t as float32 (already rounded to the storage precision)."""
    sigma = float(np.float32(init_std))
    with np.errstate(over="ignore"):
        base = mix64(np.uint64(seed) + GAMMA * np.uint64(t + 1))
    out = np.empty(numel, dtype=np.float32)

    def fill(lo: int) -> None:
        # elements lo..hi-1; independent of every other range
        hi = min(numel, lo + chunk)
        e1 = np.arange(lo + 1, hi + 1, dtype=np.uint64)
        with np.errstate(over="ignore"):
            keys = mix64(base + GAMMA * e1)
        out[lo:hi] = (polar_normal(keys) * sigma).astype(np.float32)

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
