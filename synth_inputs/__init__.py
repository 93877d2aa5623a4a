"""Seeded synthetic workloads shared by the CUDA path, the tests and the bench.

This module only describes *inputs*: the model shapes of the five PHOTON
workloads and the prompt token ids fed to them.  It contains none of the
model's arithmetic (no weights, no layers), so both the CPU oracle and the
CUDA path may import it without sharing any method code.

Sources for the shapes: PHOTON (ACL 2026), "PHOTON vertical scan" explainer,
module table and the hierarchy setting paragraph (L = 2, C1 = C2 = 4 for the
main runs, C1 = C2 = 2 for the quality-leaning runs).  Prompt distributions
are this project's reading: the pages train on The Pile, which is not
available, so token ids are drawn from a Zipf(1.1) law over the vocabulary
(p(k) proportional to k^-1.1 for rank k = 1..V, id = k - 1) or, for the tiny
byte-vocabulary model, uniformly over the 256 byte values.
"""
from __future__ import annotations

import numpy as np

# Seed of the counter-based weight generator used for every workload.
WEIGHT_SEED = 1

_BASE_600M = dict(vocab=32000, d_model=1024, n_heads=16, head_dim=64,
                  L1=4, Ltop=12, Ld1=4, Ld2=4, mlp_mult=4, dtype="bf16",
                  init_std=0.02, rope_theta=10000.0, norm_eps=1e-6)

WORKLOADS = {
    # tiny fp32 model: byte vocabulary, one layer per stack, 64 tokens decoded
    "c1": dict(vocab=256, d_model=64, n_heads=2, head_dim=32, C1=4, C2=4,
               L1=1, Ltop=1, Ld1=1, Ld2=1, mlp_mult=4, dtype="fp32",
               init_std=0.02, rope_theta=10000.0, norm_eps=1e-6,
               batch=1, prompt_len=256, decode_tokens=64,
               prompt="uniform-bytes", prompt_seed=0),
    # 600M-class bf16, 4x4 chunking, batch 64, 4096-token prompts, 512 tokens
    "c2": dict(_BASE_600M, C1=4, C2=4, batch=64, prompt_len=4096,
               decode_tokens=512, prompt="zipf1.1", prompt_seed=0),
    # same model, long context
    "c3": dict(_BASE_600M, C1=4, C2=4, batch=16, prompt_len=32768,
               decode_tokens=1024, prompt="zipf1.1", prompt_seed=0),
    # quality-leaning 2x2 chunking
    "c4": dict(_BASE_600M, C1=2, C2=2, batch=128, prompt_len=8192,
               decode_tokens=256, prompt="zipf1.1", prompt_seed=0),
    # multi-query serving: one shared prefix, many short queries
    "c5": dict(_BASE_600M, C1=4, C2=4, batch=256, prompt_len=128,
               prefix_len=16384, decode_tokens=256, prompt="zipf1.1",
               prompt_seed=1, prefix_seed=0),
}

MODEL_KEYS = ("vocab", "d_model", "n_heads", "head_dim", "C1", "C2", "L1",
              "Ltop", "Ld1", "Ld2", "mlp_mult", "dtype", "init_std",
              "rope_theta", "norm_eps")


def model_shape(name: str) -> dict:
    """The model-shape part of a named workload (plain numbers only)."""
    w = WORKLOADS[name]
    return {k: w[k] for k in MODEL_KEYS}


def zipf_probabilities(vocab: int, s: float = 1.1) -> np.ndarray:
    """p(id) for id = 0..vocab-1, proportional to (id + 1)^-s."""
    ranks = np.arange(1, vocab + 1, dtype=np.float64)
    p = ranks ** (-s)
    return p / p.sum()


def zipf_tokens(batch: int, length: int, vocab: int, seed: int,
                s: float = 1.1) -> np.ndarray:
    """int32 [batch, length] token ids drawn i.i.d. from Zipf(s) over the vocabulary."""
    rng = np.random.Generator(np.random.PCG64(seed))
    cdf = np.cumsum(zipf_probabilities(vocab, s))
    cdf[-1] = 1.0
    u = rng.random(size=(batch, length))
    ids = np.searchsorted(cdf, u, side="right")
    return np.minimum(ids, vocab - 1).astype(np.int32)


def uniform_tokens(batch: int, length: int, vocab: int, seed: int) -> np.ndarray:
    """int32 [batch, length] token ids drawn uniformly from 0..vocab-1."""
    rng = np.random.Generator(np.random.PCG64(seed))
    return rng.integers(0, vocab, size=(batch, length), dtype=np.int32)


def prompt_tokens(name: str, batch: int | None = None,
                  length: int | None = None) -> np.ndarray:
    """Prompt ids of a named workload (optionally a leading slice of its batch).

    Rows are generated for the full batch so that sequence b of a sliced
    request equals sequence b of the full workload.
    """
    w = WORKLOADS[name]
    B = w["batch"]
    T = w["prompt_len"] if length is None else length
    if w["prompt"] == "uniform-bytes":
        toks = uniform_tokens(B, T, w["vocab"], w["prompt_seed"])
    else:
        toks = zipf_tokens(B, T, w["vocab"], w["prompt_seed"])
    return toks if batch is None else toks[:batch]


def prefix_tokens(name: str) -> np.ndarray:
    """int32 [1, prefix_len] shared prefix of the multi-query workload."""
    w = WORKLOADS[name]
    return zipf_tokens(1, w["prefix_len"], w["vocab"], w["prefix_seed"])
