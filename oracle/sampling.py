"""Temperature sampling of the token decoder's output, fp64 reference.

TEST INFRASTRUCTURE ONLY -- see oracle/__init__.py for who may use it.

The PHOTON explainer's quality section describes closing the single-query
quality gap by running several slightly varied queries and combining them
(majority vote or best-of-N).  That needs a stochastic decoder; the pages do
not say which.  Reading taken here: the next token is drawn from
softmax(logits / T) with temperature T > 0 (T = 0 keeps the greedy rule).

The draw uses the Gumbel-max rule: with G_v independent standard Gumbel
variables, argmax_v (l_v / T + G_v) is distributed as softmax(l / T).  The
Gumbel variables come from a counter-based generator so that a draw depends
only on (seed, sequence, token position, vocabulary id):

  row key   K   = mix64(mix64(seed + gamma * (b + 1)) + gamma * (t + 1))
                  (mix64 = the SplitMix64 output function, gamma its
                  Weyl increment 0x9E3779B97F4A7C15), a 64-bit word;
  element   h   = MurmurHash3_x86_32 (seed 0) of the 12-byte message made of
                  K's 8 bytes and v's 4 bytes, both little-endian (Austin
                  Appleby's public hash: three 4-byte blocks, each mixed
                  with the constants 0xCC9E2D51 and 0x1B873593 and folded in
                  with rotate 13, times 5 plus 0xE6546B64; then the length 12
                  is xored in and the 32-bit finaliser applied);
  uniform   u   = (floor(h / 256) + 1/2) / 2^24, in (0, 1);
  Gumbel    G   = -ln(-ln u), with -ln u evaluated as -log1p(-(1 - u)) so
                  that u near 1 keeps its precision.

b is the sequence's row in the batch, t the token's index among the tokens
the cache has generated (chunk * C1*C2 + sub-chunk * C1 + position), v the
vocabulary id.  Ties of the perturbed values go to the lowest id, as for
greedy decoding.  The first two blocks depend on the row only, so `row_key`
returns the hash state after them and `uniforms` finishes the message per v.

The 64-bit mixes are pinned to SplitMix64's published vectors and the
element hash to scikit-learn's independent MurmurHash3 (tests).

Nucleus (top-p) sampling, a common refinement the pages do not mention
either, restricts the draw to the smallest set of most probable tokens whose
probability reaches p (ties at its edge included) and renormalises; the
Gumbel-max rule over that set has exactly that law.
"""
from __future__ import annotations

import numpy as np

from .weights import GAMMA, mix64

_F1 = np.uint32(0x85EBCA6B)
_F2 = np.uint32(0xC2B2AE35)
_MM_C1 = np.uint32(0xCC9E2D51)
_MM_C2 = np.uint32(0x1B873593)
_MM_ADD = np.uint32(0xE6546B64)


def fmix32(h: np.ndarray) -> np.ndarray:
    """MurmurHash3's 32-bit finaliser, elementwise on uint32."""
    h = np.asarray(h, dtype=np.uint32)
    with np.errstate(over="ignore"):
        h = h ^ (h >> np.uint32(16))
        h = h * _F1
        h = h ^ (h >> np.uint32(13))
        h = h * _F2
        h = h ^ (h >> np.uint32(16))
    return h


def _rotl32(x: np.ndarray, r: int) -> np.ndarray:
    return (x << np.uint32(r)) | (x >> np.uint32(32 - r))


def mm3_block(h, k) -> np.ndarray:
    """One 4-byte block of MurmurHash3_x86_32 folded into the state h (uint32)."""
    h = np.asarray(h, dtype=np.uint32)
    k = np.asarray(k, dtype=np.uint32)
    with np.errstate(over="ignore"):
        k = k * _MM_C1
        k = _rotl32(k, 15)
        k = k * _MM_C2
        h = h ^ k
        h = _rotl32(h, 13)
        h = h * np.uint32(5) + _MM_ADD
    return h


def row_key(seed: int, b: int, t: int) -> np.uint32:
    """Hash state after the row key K's two blocks (low word, then high word)."""
    with np.errstate(over="ignore"):
        k = mix64(np.uint64(seed) + GAMMA * np.uint64(b + 1))
        k = mix64(k + GAMMA * np.uint64(t + 1))
    k = int(k)
    h = mm3_block(np.uint32(0), np.uint32(k & 0xFFFFFFFF))
    return np.uint32(mm3_block(h, np.uint32(k >> 32)))


def element_hash(key: np.uint32, V: int) -> np.ndarray:
    """h_v for v = 0..V-1: the message's third block v, the length, the finaliser."""
    v = np.arange(V, dtype=np.uint32)
    return fmix32(mm3_block(np.uint32(key), v) ^ np.uint32(12))


def uniforms(key: np.uint32, V: int) -> np.ndarray:
    """u_v for v = 0..V-1, exact binary fractions in (0, 1) (fp64)."""
    h = element_hash(key, V)
    return ((h >> np.uint32(8)).astype(np.float64) + 0.5) / float(1 << 24)


def gumbel(key: np.uint32, V: int) -> np.ndarray:
    """Standard Gumbel variables G_v = -ln(-ln u_v), v = 0..V-1 (fp64)."""
    u = uniforms(key, V)
    e = -np.log1p(-(1.0 - u))   # -ln u, exact 1 - u
    return -np.log(e)


def nucleus(logits: np.ndarray, temperature: float, top_p: float) -> np.ndarray:
    """Mask of the top-p nucleus of softmax(logits / T): the smallest set of
    most probable tokens whose probability reaches top_p, with every token
    tied with its least probable member (so it is {v : p_v >= theta})."""
    z = np.asarray(logits, dtype=np.float64) / temperature
    p = np.exp(z - z.max())
    p /= p.sum()
    order = np.argsort(-p, kind="stable")
    cum = np.cumsum(p[order])
    k = int(np.searchsorted(cum, top_p * (1.0 - 1e-12)))   # first index whose mass reaches top_p
    theta = p[order[min(k, p.size - 1)]]
    return p >= theta


def sample(logits: np.ndarray, temperature: float, seed: int, b: int, t: int, top_p: float = 1.0):
    """Token drawn from softmax(logits / T) by the Gumbel-max rule; with
    top_p < 1, from that distribution restricted to its top-p nucleus and
    renormalised (the maximum runs over the nucleus only).

    Returns (token, perturbed values, -inf outside the nucleus); T > 0."""
    if not temperature > 0:
        raise ValueError("temperature must be positive")
    z = np.asarray(logits, dtype=np.float64) / temperature + gumbel(row_key(seed, b, t), logits.shape[-1])
    if top_p < 1.0:
        z = np.where(nucleus(logits, temperature, top_p), z, -np.inf)
    return int(np.argmax(z)), z
