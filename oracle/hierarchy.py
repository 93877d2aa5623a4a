"""PHOTON with any number of levels L, fp64 reference (HierGen and RecGen).

TEST INFRASTRUCTURE ONLY -- see oracle/__init__.py for who may use it.

The explainer's architecture section writes each module for a general level
l: the Context Chunker merges C_l level-(l-1) states, a Context Encoder runs
autoregressively over each coarse stream, and a Converter and a chunk-local
Decoder go top-down.  Its RecGen section states that Theorem A.6 needs
A-hat = A only at the L -> L-1 interface, and that levels 1..L-1 lose their
encoder caches after prefill.  The main runs use L = 2, which
oracle/photon.py implements.  This module takes the same readings (R1-R8 of
the design notes) for every L >= 1:

  bottom-up   s_0 = Embed(tokens);  s_l = Encoder_l(Chunker_l(s_{l-1})),
              l = 1..L (Encoder_L is the top encoder, its outputs o_k);
  top-down    Converter_L(o_k) -> C_L conditioning positions -> Decoder_L,
              whose final-norm outputs A-hat_L are reconstructions of the
              chunk's level-(L-1) states; each A-hat_l row feeds
              Converter_{l-1} -> Decoder_{l-1} in turn, down to the token
              decoder (Decoder_1), which reads its C_1 conditioning vectors
              followed by the sub-chunk's tokens so far;
  HierGen     re-encodes the written tokens through levels 1..L-1 (their
              caches grow) and feeds Chunker_L of the level-(L-1) states to
              the top encoder;
  RecGen      feeds Chunker_L(A-hat_L) to the top encoder; no level below
              L is touched and their caches are dropped after prefill.
              It needs L >= 2 (with L = 1 the interface below the top is
              the token embedding itself, and HierGen is exact and cheap).

With L = 1 this is a single-level block model: token blocks of C_1 merged
by one linear map, a causal encoder over blocks, and a block-local token
decoder conditioned by the converter.  That is the shape of the Block
Transformer baseline the explainer compares against.  Parameter names
follow oracle/weights.py: chunker{l}, enc{l} (top for l = L), converter{l},
dec{l}, embed, head.  So for L = 2 the spec list and weights are identical
to the two-level model's.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

from .photon import LayerKV, chunker, converter, stack
from .weights import draw_tensor


@dataclass(frozen=True)
class HierConfig:
    vocab: int
    d_model: int
    n_heads: int
    head_dim: int
    chunks: tuple          # C_1 .. C_L
    enc_layers: tuple      # encoder depth of levels 1 .. L (the last is the top encoder)
    dec_layers: tuple      # decoder depth of levels 1 .. L (the first is the token decoder)
    mlp_mult: int = 4
    dtype: str = "fp32"
    init_std: float = 0.02
    rope_theta: float = 10000.0
    norm_eps: float = 1e-6

    def __post_init__(self):
        if not (len(self.chunks) == len(self.enc_layers) == len(self.dec_layers) >= 1):
            raise ValueError("chunks, enc_layers and dec_layers need one entry per level")

    @property
    def L(self) -> int:
        return len(self.chunks)

    @property
    def C(self) -> int:
        return int(np.prod(self.chunks))


def enc_name(cfg: HierConfig, l: int) -> str:
    return "top" if l == cfg.L else f"enc{l}"


def hier_specs(cfg: HierConfig) -> list[tuple[str, tuple[int, ...], str]]:
    """(name, shape, kind) of every parameter in generator order: embedding,
    then bottom-up (chunker and encoder of each level), then top-down
    (converter and decoder of each level), then the head."""
    d, V, f = cfg.d_model, cfg.vocab, cfg.mlp_mult * cfg.d_model
    specs: list[tuple[str, tuple[int, ...], str]] = []

    def blocks(prefix: str, n: int) -> None:
        for i in range(n):
            p = f"{prefix}.{i}."
            specs.extend([(p + "g_attn", (d,), "ones"), (p + "wq", (d, d), "normal"),
                          (p + "wk", (d, d), "normal"), (p + "wv", (d, d), "normal"),
                          (p + "wo", (d, d), "normal"), (p + "g_mlp", (d,), "ones"),
                          (p + "w1", (f, d), "normal"), (p + "w2", (d, f), "normal")])
        specs.append((prefix + ".g_final", (d,), "ones"))

    specs.append(("embed", (V, d), "normal"))
    for l in range(1, cfg.L + 1):
        specs.append((f"chunker{l}", (d, cfg.chunks[l - 1] * d), "normal"))
        blocks(enc_name(cfg, l), cfg.enc_layers[l - 1])
    for l in range(cfg.L, 0, -1):
        specs.append((f"converter{l}", (cfg.chunks[l - 1] * d, d), "normal"))
        blocks(f"dec{l}", cfg.dec_layers[l - 1])
    specs.append(("head", (V, d), "normal"))
    return specs


def make_hier_weights(cfg: HierConfig, seed: int) -> dict[str, np.ndarray]:
    """Parameters drawn by the counter-based generator in hier_specs order."""
    w = {}
    for t, (name, shape, kind) in enumerate(hier_specs(cfg)):
        n = int(np.prod(shape))
        v = np.ones(n) if kind == "ones" else draw_tensor(seed, t, n, cfg.init_std, cfg.dtype).astype(np.float64)
        w[name] = v.reshape(shape)
    return w


@dataclass
class HierState:
    mode: str                           # "hier" or "rec"
    caches: list                        # caches[l-1] = KV of level l's encoder (None once dropped)
    counts: list                        # counts[l-1] = entries in level l's stream
    o: np.ndarray                       # pending top output [d]
    tokens: list = field(default_factory=list)
    top_inputs: list = field(default_factory=list)   # Chunker_L outputs fed to the top encoder


@dataclass
class HierStep:
    tokens: np.ndarray      # [C] own choices, time order
    used: np.ndarray        # [C] tokens fed back (forced or own)
    logits: np.ndarray      # [C, V]
    a_hat: np.ndarray | None  # [C_L, d] Decoder_L's reconstruction (None for L = 1)
    a: np.ndarray | None    # [C_L, d] level-(L-1) encoder states of the chunk (HierGen, L >= 2)


class HierOracle:
    def __init__(self, cfg: HierConfig, seed: int, weights: dict | None = None):
        self.cfg = cfg
        self.w = make_hier_weights(cfg, seed) if weights is None else weights

    # -- bottom-up --------------------------------------------------------------
    def encode(self, l: int, lower: np.ndarray, start: int, past):
        """Chunker_l over level-(l-1) rows, then Encoder_l at positions
        start.. of its stream.  Returns (normed states, extended caches)."""
        cfg = self.cfg
        z = chunker(lower, self.w[f"chunker{l}"], cfg.chunks[l - 1])
        return stack(cfg, self.w, enc_name(cfg, l), cfg.enc_layers[l - 1], z,
                     start + np.arange(z.shape[0]), past)

    def prefill(self, tokens, mode: str) -> HierState:
        cfg = self.cfg
        if mode == "rec" and cfg.L < 2:
            raise ValueError("RecGen needs L >= 2")
        tokens = np.asarray(tokens, dtype=np.int64)
        if tokens.shape[0] <= 0 or tokens.shape[0] % cfg.C:
            raise ValueError("prompt length must be a positive multiple of C_1 * ... * C_L")
        s = self.w["embed"][tokens]
        caches, counts = [], []
        for l in range(1, cfg.L + 1):
            if l == cfg.L:
                u = chunker(s, self.w[f"chunker{l}"], cfg.chunks[l - 1])
            s, kv = self.encode(l, s, 0, None)
            caches.append(kv if (l == cfg.L or mode == "hier") else None)
            counts.append(s.shape[0] if (l == cfg.L or mode == "hier") else 0)
        return HierState(mode=mode, caches=caches, counts=counts, o=s[-1].copy(),
                         tokens=[int(t) for t in tokens], top_inputs=[r.copy() for r in u])

    # -- top-down ---------------------------------------------------------------
    def reconstruct(self, l: int, v: np.ndarray) -> np.ndarray:
        """Converter_l of one level-l vector, then Decoder_l over its C_l
        conditioning positions (chunk-local, positions 0..C_l-1); l >= 2."""
        cfg = self.cfg
        c = converter(v, self.w[f"converter{l}"], cfg.chunks[l - 1])
        out, _ = stack(cfg, self.w, f"dec{l}", cfg.dec_layers[l - 1], c, np.arange(c.shape[0]), None)
        return out

    def token_logits(self, cond: np.ndarray, prev: list) -> np.ndarray:
        cfg, w = self.cfg, self.w
        x = np.concatenate([cond] + ([w["embed"][np.asarray(prev)]] if prev else []), axis=0)
        h, _ = stack(cfg, w, "dec1", cfg.dec_layers[0], x, np.arange(x.shape[0]), None)
        return h[-1] @ w["head"].T

    def _emit(self, l: int, v: np.ndarray, force, out: list) -> None:
        """Writes the tokens under level-l vector v, depth first in time order."""
        cfg = self.cfg
        if l == 1:
            cond = converter(v, self.w["converter1"], cfg.chunks[0])
            prev: list = []
            for _ in range(cfg.chunks[0]):
                lg = self.token_logits(cond, prev)
                t = len(out)
                own = int(np.argmax(lg))
                used = own if force is None or force[t] < 0 else int(force[t])
                out.append((own, used, lg))
                prev.append(used)
            return
        for row in self.reconstruct(l, v):
            self._emit(l - 1, row, force, out)

    def decode_step(self, st: HierState, mode: str, force_tokens=None, force_a=None) -> HierStep:
        """One top-level chunk: the tokens under the pending top output, then
        the top encoder's next input (HierGen: re-encoded tokens; RecGen:
        Chunker_L of A-hat_L, or of `force_a` when given)."""
        cfg, L = self.cfg, self.cfg.L
        if mode == "hier" and any(c is None for c in st.caches[:-1]):
            raise ValueError("HierGen needs the lower encoder caches (dropped by a RecGen prefill)")
        if mode == "rec" and L < 2:
            raise ValueError("RecGen needs L >= 2")
        out: list = []
        a_hat = None
        if L == 1:
            self._emit(1, st.o, force_tokens, out)
        else:
            a_hat = self.reconstruct(L, st.o)
            for row in a_hat:
                self._emit(L - 1, row, force_tokens, out)
        own = np.array([o for o, _, _ in out], dtype=np.int64)
        used = np.array([u for _, u, _ in out], dtype=np.int64)
        logits = np.stack([lg for _, _, lg in out])
        a = None
        if mode == "hier":
            s = self.w["embed"][used]
            for l in range(1, L):
                s, st.caches[l - 1] = self.encode(l, s, st.counts[l - 1], st.caches[l - 1])
                st.counts[l - 1] += s.shape[0]
            a = s if L >= 2 else None
            top_in = s
        else:
            top_in = a_hat if force_a is None else np.asarray(force_a, dtype=np.float64)
        u = chunker(top_in, self.w[f"chunker{L}"], cfg.chunks[L - 1])
        o, st.caches[L - 1] = stack(cfg, self.w, "top", cfg.enc_layers[L - 1], u,
                                    st.counts[L - 1] + np.arange(1), st.caches[L - 1])
        st.o = o[-1].copy()
        st.counts[L - 1] += 1
        st.top_inputs.append(u[0].copy())
        st.tokens.extend(int(t) for t in used)
        return HierStep(tokens=own, used=used, logits=logits, a_hat=a_hat, a=a)

    # -- teacher-forced scoring -------------------------------------------------
    def score(self, tokens):
        """Log-probability of every token after the first top chunk under
        teacher forcing (explainer, quality section).  The bottom-up pass
        encodes the true tokens.  Top output o_k conditions top chunk k + 1
        down every level, and each decoder reads the true tokens of its
        sub-chunk.  Returns (log-probabilities [T - C], logits [T - C, V])."""
        cfg = self.cfg
        tokens = np.asarray(tokens, dtype=np.int64)
        T = tokens.shape[0]
        if T <= cfg.C or T % cfg.C:
            raise ValueError("the prompt must be a multiple of C_1 * ... * C_L longer than one top chunk")
        s = self.w["embed"][tokens]
        for l in range(1, cfg.L + 1):
            s, _ = self.encode(l, s, 0, None)
        logits = []
        for k in range(1, T // cfg.C):
            force = tokens[k * cfg.C:(k + 1) * cfg.C]
            out: list = []
            if cfg.L == 1:
                self._emit(1, s[k - 1], force, out)
            else:
                for row in self.reconstruct(cfg.L, s[k - 1]):
                    self._emit(cfg.L - 1, row, force, out)
            logits.extend(lg for _, _, lg in out)
        logits = np.stack(logits)
        z = logits - logits.max(axis=1, keepdims=True)
        logp = z - np.log(np.exp(z).sum(axis=1, keepdims=True))
        return logp[np.arange(T - cfg.C), tokens[cfg.C:]], logits

    # -- full recomputation (pins the incremental paths) --------------------------
    def full_top(self, top_inputs):
        """Top encoder over a whole list of coarse inputs, from scratch."""
        cfg = self.cfg
        u = np.stack(top_inputs)
        return stack(cfg, self.w, "top", cfg.enc_layers[-1], u, np.arange(u.shape[0]), None)
