"""fp64 reference of a vanilla token-level Transformer of PHOTON's width.

TEST INFRASTRUCTURE ONLY -- see oracle/__init__.py for who may use it.

The PHOTON pages compare throughput per memory (TPM) against a vanilla
Transformer of similar size (explainer, 475x section, the decode-heavy
table).  This is that baseline in its plainest form: one causal pre-norm
stack over the token stream (the same blocks as PHOTON's stacks: RMSNorm,
rotate-half RoPE per token position, full multi-head attention, 4x erf-GELU
MLP, no biases), a final RMSNorm and an untied head, with a KV cache over
every token.  Weights use the same counter-based generator as the PHOTON
oracle, in the tensor order embed, blocks, final gain, head.

Decode convention: the prefill caches the first T-1 prompt tokens; every
decode step feeds one token (the last prompt token first, then the token
chosen before) at the next position and chooses the next token greedily
(lowest id on ties), so every step has the same shape.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

from .photon import LayerKV, stack
from .weights import draw_tensor


@dataclass(frozen=True)
class VanillaConfig:
    vocab: int
    d_model: int
    n_heads: int
    head_dim: int
    layers: int
    mlp_mult: int = 4
    dtype: str = "fp32"
    init_std: float = 0.02
    rope_theta: float = 10000.0
    norm_eps: float = 1e-6

    @classmethod
    def from_dict(cls, d: dict) -> "VanillaConfig":
        names = cls.__dataclass_fields__.keys()
        return cls(**{k: d[k] for k in names if k in d})


def vanilla_specs(cfg: VanillaConfig) -> list[tuple[str, tuple[int, ...], str]]:
    """(name, shape, kind) in generator order."""
    d, V, f = cfg.d_model, cfg.vocab, cfg.mlp_mult * cfg.d_model
    specs = [("embed", (V, d), "normal")]
    for l in range(cfg.layers):
        p = f"van.{l}."
        specs += [(p + "g_attn", (d,), "ones"), (p + "wq", (d, d), "normal"), (p + "wk", (d, d), "normal"),
                  (p + "wv", (d, d), "normal"), (p + "wo", (d, d), "normal"), (p + "g_mlp", (d,), "ones"),
                  (p + "w1", (f, d), "normal"), (p + "w2", (d, f), "normal")]
    specs += [("van.g_final", (d,), "ones"), ("head", (V, d), "normal")]
    return specs


def make_vanilla_weights(cfg: VanillaConfig, seed: int) -> dict[str, np.ndarray]:
    w: dict[str, np.ndarray] = {}
    for t, (name, shape, kind) in enumerate(vanilla_specs(cfg)):
        n = int(np.prod(shape))
        if kind == "ones":
            v = np.ones(n, dtype=np.float64)
        else:
            v = draw_tensor(seed, t, n, cfg.init_std, cfg.dtype).astype(np.float64)
        w[name] = v.reshape(shape)
    return w


@dataclass
class VanillaState:
    kv: list[LayerKV]       # per layer, N cached positions
    N: int                  # cached positions
    next_token: int         # the token the next decode step feeds
    tokens: list[int] = field(default_factory=list)   # every token fed or cached so far


class VanillaOracle:
    def __init__(self, cfg: VanillaConfig, seed: int, weights: dict | None = None):
        self.cfg = cfg
        self.w = make_vanilla_weights(cfg, seed) if weights is None else weights

    def forward(self, tokens, start: int, past):
        """Normed final rows and extended caches for tokens at positions start.."""
        x = self.w["embed"][np.asarray(tokens, dtype=np.int64)]
        pos = start + np.arange(x.shape[0])
        return stack(self.cfg, self.w, "van", self.cfg.layers, x, pos, past)

    def prefill(self, tokens) -> VanillaState:
        tokens = [int(t) for t in tokens]
        if len(tokens) < 2:
            raise ValueError("the prompt needs at least two tokens")
        _, kv = self.forward(tokens[:-1], 0, None)
        return VanillaState(kv=kv, N=len(tokens) - 1, next_token=tokens[-1], tokens=tokens[:-1])

    def decode_step(self, st: VanillaState, force: int | None = None):
        """Feed st.next_token; return (greedy token, logits [V])."""
        h, st.kv = self.forward([st.next_token], st.N, st.kv)
        logits = h[-1] @ self.w["head"].T
        tok = int(np.argmax(logits))
        st.tokens.append(st.next_token)
        st.N += 1
        st.next_token = tok if force is None or force < 0 else int(force)
        return tok, logits

    def logits_from_scratch(self, tokens) -> np.ndarray:
        """Next-token logits after `tokens`, with no cache (pins the cached path)."""
        h, _ = self.forward(tokens, 0, None)
        return h[-1] @ self.w["head"].T
