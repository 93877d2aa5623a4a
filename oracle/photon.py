"""Plain fp64 NumPy oracle of PHOTON's hierarchical prefill, HierGen and RecGen.

TEST INFRASTRUCTURE ONLY -- see oracle/__init__.py for who may use it.

Every function follows a passage of the PHOTON pages (ACL 2026 record and
the "PHOTON vertical scan" explainer).  Citations name the page and the
passage:

  [abstract]       PHOTON (ACL 2026), abstract: bottom-up encoder compresses
                   tokens into low-rate states; top-down decoders reconstruct
                   tokens; recursive generation updates only the coarsest
                   stream.
  [modules]        explainer, architecture section, module table: Context
                   Chunker / Encoder / Converter / Decoder.
  [setting]        explainer, architecture section: L = 2, C1 = C2 = 4 (and 2x2).
  [hiergen]        explainer, RecGen section: the three-stage HierGen loop.
  [recgen]         explainer, RecGen section: feed the bottleneck
                   reconstruction A-hat straight to the top encoder.
  [thm-a6]         explainer, RecGen section, quoting Appendix A Theorem A.6.
  [cache-discard]  explainer, RecGen section: only the top-level global KV
                   is kept; level-1..L-1 encoder caches are dropped after
                   prefill.
  [span]           explainer, 475x section: decoder attention confined to
                   the chunk (span R_l + C_l), independent of T.

Where the pages leave a step open the oracle takes one plain reading,
listed as R1..R18 in the project's design notes.  In short: pre-RMSNorm
Transformer blocks (eps 1e-6, gain 1), full multi-head attention with
rotate-half RoPE (theta 1e4, 0-based positions inside each stream), erf-GELU
4x MLP, no biases, untied head; the Chunker concatenates C states in time
order and applies one linear C*d -> d map (R1); the Converter is a
transposed 1-D convolution with kernel = stride = C on a length-1 input,
i.e. C independent d x d maps (R2); converter outputs are a prefix of the
decoder's chunk-local causal sequence (R3); Decoder_2 runs once over its C2
conditioning positions and its final-norm outputs are A-hat (R4); top output
o_k conditions chunk k+1 (R6); one decode call = one top-level chunk (R7).

The oracle processes one sequence at a time (sequences never interact) and
computes the token decoder by full recomputation over its short chunk-local
sequence, with no decoder cache at all.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np
from scipy.special import erf

from .sampling import sample as draw
from .weights import make_weights


@dataclass(frozen=True)
class Config:
    vocab: int
    d_model: int
    n_heads: int
    head_dim: int
    C1: int
    C2: int
    L1: int
    Ltop: int
    Ld1: int
    Ld2: int
    mlp_mult: int = 4
    dtype: str = "fp32"
    init_std: float = 0.02
    rope_theta: float = 10000.0
    norm_eps: float = 1e-6

    @property
    def C(self) -> int:
        return self.C1 * self.C2

    @classmethod
    def from_dict(cls, d: dict) -> "Config":
        names = cls.__dataclass_fields__.keys()
        return cls(**{k: d[k] for k in names if k in d})


# ----------------------------------------------------------------------------
# Transformer pieces ([modules]: encoder and decoder are Transformer stacks)
# ----------------------------------------------------------------------------

def rmsnorm(x: np.ndarray, g: np.ndarray, eps: float) -> np.ndarray:
    """x / sqrt(mean(x^2) + eps) * g over the last axis (R9)."""
    return x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps) * g


def rope(x: np.ndarray, pos: np.ndarray, theta: float) -> np.ndarray:
    """Rotate-half rotary embedding (R8).

    x: [n, H, dh]; pos: [n] integer positions.  Pair (i, i + dh/2) of each
    head is rotated by the angle pos * theta^(-2i/dh).
    """
    dh = x.shape[-1]
    half = dh // 2
    inv = theta ** (-2.0 * np.arange(half, dtype=np.float64) / dh)
    ang = np.asarray(pos, dtype=np.float64)[:, None] * inv[None, :]
    c = np.cos(ang)[:, None, :]
    s = np.sin(ang)[:, None, :]
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * c - x2 * s, x1 * s + x2 * c], axis=-1)


def gelu(x: np.ndarray) -> np.ndarray:
    """erf-GELU: x * Phi(x) (R10)."""
    return 0.5 * x * (1.0 + erf(x / math.sqrt(2.0)))


def attention(q: np.ndarray, k: np.ndarray, v: np.ndarray,
              q_pos: np.ndarray, k_pos: np.ndarray) -> np.ndarray:
    """Multi-head softmax attention with an additive -inf causal mask (R11).

    q: [nq, H, dh]; k, v: [nk, H, dh]; query at position p sees keys at
    positions <= p.  Returns [nq, H, dh].
    """
    dh = q.shape[-1]
    q_pos = np.asarray(q_pos)
    k_pos = np.asarray(k_pos)
    out = np.empty(q.shape[:1] + v.shape[1:])
    kt = k.transpose(1, 2, 0)            # [H, dh, nk]
    vt = v.transpose(1, 0, 2)            # [H, nk, dh]
    ascending = bool(np.all(np.diff(k_pos) > 0))
    # Query rows are independent (one softmax per row); they are processed
    # in groups only to bound the memory of the score matrix.  With keys in
    # ascending position order, keys after the group's last visible position
    # have weight exactly 0 and are left out of the group's products.
    step = max(1, (1 << 25) // max(1, q.shape[1] * k.shape[0]))
    for lo in range(0, q.shape[0], step):
        hi = min(q.shape[0], lo + step)
        nk = k.shape[0]
        if ascending:
            nk = int(np.searchsorted(k_pos, q_pos[lo:hi].max(), side="right"))
        s = np.matmul(q[lo:hi].transpose(1, 0, 2), kt[:, :, :nk])
        s *= 1.0 / math.sqrt(dh)
        allowed = k_pos[None, :nk] <= q_pos[lo:hi, None]
        np.copyto(s, -np.inf, where=~allowed[None])
        s -= s.max(axis=-1, keepdims=True)
        np.exp(s, out=s)
        s /= s.sum(axis=-1, keepdims=True)
        out[lo:hi] = np.matmul(s, vt[:, :nk]).transpose(1, 0, 2)
    return out


@dataclass
class LayerKV:
    """Keys/values of one layer for one sequence: [n, H, dh] each, post-RoPE keys."""
    k: np.ndarray
    v: np.ndarray


def block(cfg: Config, w: dict, prefix: str, x: np.ndarray, pos: np.ndarray,
          past: LayerKV | None) -> tuple[np.ndarray, LayerKV]:
    """One pre-norm block over rows x [n, d] at stream positions pos [n].

    `past` holds the keys/values of positions 0..pos[0]-1 of the same stream
    (None for an empty cache).  Returns the new rows and the extended cache.
    """
    n, d = x.shape
    H, dh, eps = cfg.n_heads, cfg.head_dim, cfg.norm_eps
    h = rmsnorm(x, w[prefix + "g_attn"], eps)
    q = (h @ w[prefix + "wq"].T).reshape(n, H, dh)
    k = (h @ w[prefix + "wk"].T).reshape(n, H, dh)
    v = (h @ w[prefix + "wv"].T).reshape(n, H, dh)
    q = rope(q, pos, cfg.rope_theta)
    k = rope(k, pos, cfg.rope_theta)
    if past is not None:
        k = np.concatenate([past.k, k], axis=0)
        v = np.concatenate([past.v, v], axis=0)
    kv = LayerKV(k, v)
    a = attention(q, k, v, pos, np.arange(k.shape[0]))
    x = x + a.reshape(n, d) @ w[prefix + "wo"].T
    h = rmsnorm(x, w[prefix + "g_mlp"], eps)
    x = x + gelu(h @ w[prefix + "w1"].T) @ w[prefix + "w2"].T
    return x, kv


def stack(cfg: Config, w: dict, name: str, n_layers: int, x: np.ndarray,
          pos: np.ndarray, past: list[LayerKV] | None
          ) -> tuple[np.ndarray, list[LayerKV]]:
    """A stack of blocks followed by its final RMSNorm; returns (normed, caches)."""
    caches = []
    for l in range(n_layers):
        x, kv = block(cfg, w, f"{name}.{l}.", x, pos, None if past is None else past[l])
        caches.append(kv)
    return rmsnorm(x, w[name + ".g_final"], cfg.norm_eps), caches


# ----------------------------------------------------------------------------
# PHOTON modules ([modules])
# ----------------------------------------------------------------------------

def chunker(x: np.ndarray, W: np.ndarray, C: int) -> np.ndarray:
    """Context Chunker (R1): concatenate each group of C consecutive rows
    in time order (element j*d + i is feature i of member j) and apply the
    linear map W [d, C*d].  [n*C, d] -> [n, d]."""
    n = x.shape[0] // C
    return x.reshape(n, C * x.shape[1]) @ W.T


def converter(o: np.ndarray, W: np.ndarray, C: int) -> np.ndarray:
    """Context Converter (R2): transposed conv1d, kernel = stride = C, on a
    length-1 input: vector j of the output is W[j*d:(j+1)*d] @ o.  [d] -> [C, d]."""
    d = o.shape[-1]
    return (W @ o).reshape(C, d)


# ----------------------------------------------------------------------------
# Sequence state and the three procedures
# ----------------------------------------------------------------------------

@dataclass
class SeqState:
    """Everything the oracle keeps for one sequence between calls."""
    mode: str                          # "hier" or "rec"
    top: list[LayerKV]                 # top-encoder KV, N entries per layer
    l1: list[LayerKV] | None           # level-1 encoder KV (None after RecGen prefill)
    o: np.ndarray                      # pending top output (after final norm), [d]
    N: int                             # top-level entries
    N1: int                            # level-1 entries (0 once discarded)
    tokens: list[int] = field(default_factory=list)   # prompt + generated ids
    top_inputs: list[np.ndarray] = field(default_factory=list)  # chunker-2 outputs fed to the top
    steps: int = 0                     # decode calls since the prefill (chunks generated)


@dataclass
class StepResult:
    tokens: np.ndarray      # [C] int: the oracle's own choices (j*C1 + i order)
    used: np.ndarray        # [C] int: tokens fed back (forced or own)
    logits: np.ndarray      # [C, V] fp64
    a_hat: np.ndarray       # [C2, d] Decoder_2 reconstruction
    a: np.ndarray | None    # [C2, d] level-1 encoder states of the chunk (HierGen only)
    near_tie: np.ndarray    # [C] bool: top-2 gap < 1e-5 * range of the compared values (R12)


class PhotonOracle:
    """fp64 reference of the whole hot path for a given (config, seed)."""

    def __init__(self, cfg: Config, seed: int, weights: dict | None = None):
        self.cfg = cfg
        self.w = make_weights(cfg, seed) if weights is None else weights

    # -- bottom-up ------------------------------------------------------------
    def encode_level1(self, tokens: np.ndarray, start: int,
                      past: list[LayerKV] | None):
        """Embedding -> Chunker_1 -> Encoder_1 over the level-1 positions that
        the tokens form ([modules], Chunker and Encoder rows).  Returns
        (s1 [n1, d] after the final norm, extended level-1 caches)."""
        cfg, w = self.cfg, self.w
        h0 = w["embed"][np.asarray(tokens)]
        z = chunker(h0, w["chunker1"], cfg.C1)
        pos = start + np.arange(z.shape[0])
        return stack(cfg, w, "enc1", cfg.L1, z, pos, past)

    def top_encode(self, u: np.ndarray, start: int, past: list[LayerKV] | None):
        """Top Context Encoder over coarse inputs u [n, d] at positions
        start..start+n-1; it owns the only global cache ([modules],
        [cache-discard]).  Returns (normed outputs [n, d], caches)."""
        cfg = self.cfg
        pos = start + np.arange(u.shape[0])
        return stack(cfg, self.w, "top", cfg.Ltop, u, pos, past)

    def prefill(self, tokens: np.ndarray, mode: str) -> SeqState:
        """Hierarchical prefill of one prompt ([abstract], [modules]).

        T must be a positive multiple of C = C1*C2 (R6).  In RecGen mode the
        level-1 caches are dropped afterwards ([cache-discard])."""
        cfg = self.cfg
        tokens = np.asarray(tokens, dtype=np.int64)
        T = tokens.shape[0]
        if T <= 0 or T % cfg.C:
            raise ValueError("prompt length must be a positive multiple of C1*C2")
        s1, l1 = self.encode_level1(tokens, 0, None)
        u = chunker(s1, self.w["chunker2"], cfg.C2)
        o_all, top = self.top_encode(u, 0, None)
        return SeqState(mode=mode, top=top, l1=(l1 if mode == "hier" else None),
                        o=o_all[-1].copy(), N=T // cfg.C,
                        N1=(T // cfg.C1 if mode == "hier" else 0),
                        tokens=[int(t) for t in tokens],
                        top_inputs=[r.copy() for r in u])

    def prefill_after(self, prefix: SeqState, tokens: np.ndarray, mode: str) -> SeqState:
        """Prefill of `tokens` continuing a HierGen-mode state `prefix` (a shared
        context that precedes them): the same Chunker/Encoder passes as
        `prefill`, with the prefix's level-1 and top caches as the past.
        Equal to prefill(prefix tokens + tokens), which the tests pin."""
        cfg = self.cfg
        if prefix.l1 is None:
            raise ValueError("the prefix must keep its level-1 cache (HierGen mode)")
        tokens = np.asarray(tokens, dtype=np.int64)
        T = tokens.shape[0]
        if T <= 0 or T % cfg.C:
            raise ValueError("prompt length must be a positive multiple of C1*C2")
        s1, l1 = self.encode_level1(tokens, prefix.N1, prefix.l1)
        u = chunker(s1, self.w["chunker2"], cfg.C2)
        o_all, top = self.top_encode(u, prefix.N, prefix.top)
        return SeqState(mode=mode, top=top, l1=(l1 if mode == "hier" else None),
                        o=o_all[-1].copy(), N=prefix.N + T // cfg.C,
                        N1=(prefix.N1 + T // cfg.C1 if mode == "hier" else 0),
                        tokens=list(prefix.tokens) + [int(t) for t in tokens],
                        top_inputs=list(prefix.top_inputs) + [r.copy() for r in u])

    # -- top-down -------------------------------------------------------------
    def decode_chunk2(self, o: np.ndarray) -> np.ndarray:
        """Converter_2 then Decoder_2 over its C2 conditioning positions
        (chunk-local causal, positions 0..C2-1); final-norm outputs are A-hat
        ([modules], [recgen], R3, R4)."""
        cfg = self.cfg
        c = converter(o, self.w["converter2"], cfg.C2)
        a_hat, _ = stack(cfg, self.w, "dec2", cfg.Ld2, c, np.arange(cfg.C2), None)
        return a_hat

    def token_decoder_logits(self, cond: np.ndarray, prev_tokens: list[int]) -> np.ndarray:
        """Logits for the next token of a level-1 chunk ([modules], [span]).

        The chunk-local sequence is the C1 conditioning vectors followed by
        the embeddings of the chunk's tokens so far; the decoder runs
        causally over it (positions 0..) and the head reads its last row."""
        cfg, w = self.cfg, self.w
        rows = [cond] + ([w["embed"][np.asarray(prev_tokens)]] if prev_tokens else [])
        x = np.concatenate(rows, axis=0)
        h, _ = stack(cfg, w, "dec1", cfg.Ld1, x, np.arange(x.shape[0]), None)
        return h[-1] @ w["head"].T

    def emit_tokens(self, a_hat: np.ndarray, force: np.ndarray | None, sample=None, first_t: int = 0):
        """Write the C tokens of the next top-level chunk from A-hat.

        Sub-chunk j uses Converter_1(A-hat_j) as its conditioning; its tokens
        depend on nothing else (R4).  Greedy argmax, lowest index on ties (R12);
        with `sample` = (temperature, seed, b[, top_p]) the token is drawn
        from softmax(logits / temperature), optionally restricted to its top-p
        nucleus (oracle/sampling.py), token index first_t + j*C1 + i.  `force` (teacher forcing, entries < 0 = not
        forced) replaces the token fed back, not the recorded choice."""
        cfg = self.cfg
        C1, C2, V = cfg.C1, cfg.C2, cfg.vocab
        own = np.zeros(C1 * C2, dtype=np.int64)
        used = np.zeros(C1 * C2, dtype=np.int64)
        logits = np.zeros((C1 * C2, V))
        tie = np.zeros(C1 * C2, dtype=bool)
        for j in range(C2):
            cond = converter(a_hat[j], self.w["converter1"], C1)
            prev: list[int] = []
            for i in range(C1):
                t = j * C1 + i
                lg = self.token_decoder_logits(cond, prev)
                logits[t] = lg
                if sample is None:
                    own[t], z = int(np.argmax(lg)), lg
                else:
                    temperature, seed, b = sample[:3]
                    top_p = sample[3] if len(sample) > 3 else 1.0
                    own[t], z = draw(lg, temperature, seed, b, first_t + t, top_p)
                    z = z[np.isfinite(z)]
                srt = np.sort(z)
                tie[t] = (srt[-1] - srt[-2]) < 1e-5 * (srt[-1] - srt[0])
                used[t] = own[t] if force is None or force[t] < 0 else int(force[t])
                prev.append(int(used[t]))
        return own, used, logits, tie

    def top_step(self, st: SeqState, u: np.ndarray) -> None:
        """Advance the top encoder by one coarse position with input u [d]."""
        o, top = self.top_encode(u[None, :], st.N, st.top)
        st.top = top
        st.o = o[-1].copy()
        st.N += 1
        st.top_inputs.append(u.copy())

    def decode_step(self, st: SeqState, mode: str, force_tokens=None,
                    force_a=None, sample=None) -> StepResult:
        """One top-level chunk of decoding (R7).

        HierGen ([hiergen]): write the chunk's tokens, re-encode them
        (Embedding -> Chunker_1 -> Encoder_1 with its cache), Chunker_2, one
        top step.  RecGen ([recgen]): write the tokens, then feed
        Chunker_2(A-hat) to the top encoder; no level-1 work at all.
        `force_a` (test hook for [thm-a6]) replaces A-hat as the RecGen top
        input.  `sample` = (temperature, seed, b): temperature sampling for
        the sequence in batch row b (oracle/sampling.py); None = greedy."""
        cfg = self.cfg
        if mode == "hier" and st.l1 is None:
            raise ValueError("HierGen needs the level-1 cache (discarded by a RecGen prefill)")
        a_hat = self.decode_chunk2(st.o)
        own, used, logits, tie = self.emit_tokens(a_hat, force_tokens, sample, st.steps * cfg.C)
        a = None
        if mode == "hier":
            a, st.l1 = self.encode_level1(used, st.N1, st.l1)
            st.N1 += cfg.C2
            top_in = a
        else:
            top_in = a_hat if force_a is None else np.asarray(force_a, dtype=np.float64)
        u = chunker(top_in, self.w["chunker2"], cfg.C2)[0]
        self.top_step(st, u)
        st.tokens.extend(int(t) for t in used)
        st.steps += 1
        return StepResult(tokens=own, used=used, logits=logits, a_hat=a_hat, a=a, near_tie=tie)

    # -- teacher-forced scoring -------------------------------------------------
    def score(self, tokens):
        """Log-probability of every token of chunks 1..N-1 of a prompt under
        teacher forcing (explainer, quality section: the reported quality is
        measured with teacher-forced HierGen).

        The bottom-up pass encodes the true tokens; the top output o_k of
        chunk k conditions chunk k+1 (R6); Decoder_2 and the token decoder
        then read chunk k+1's true tokens as their inputs (R3, R4), so every
        position's next-token distribution comes out at once.  The first
        chunk has no top output before it and is not scored.  Returns
        (log-probabilities [T - C], logits [T - C, V])."""
        cfg, w = self.cfg, self.w
        tokens = np.asarray(tokens, dtype=np.int64)
        T = tokens.shape[0]
        if T <= cfg.C or T % cfg.C:
            raise ValueError("the prompt must be a multiple of C1*C2 longer than one chunk")
        s1, _ = self.encode_level1(tokens, 0, None)
        o_all, _ = self.top_encode(chunker(s1, w["chunker2"], cfg.C2), 0, None)
        logits = []
        for k in range(1, T // cfg.C):
            a_hat = self.decode_chunk2(o_all[k - 1])
            for j in range(cfg.C2):
                cond = converter(a_hat[j], w["converter1"], cfg.C1)
                base = k * cfg.C + j * cfg.C1
                for i in range(cfg.C1):
                    logits.append(self.token_decoder_logits(cond, [int(t) for t in tokens[base:base + i]]))
        logits = np.stack(logits)
        z = logits - logits.max(axis=1, keepdims=True)
        logp = z - np.log(np.exp(z).sum(axis=1, keepdims=True))
        return logp[np.arange(T - cfg.C), tokens[cfg.C:]], logits

    # -- full recomputation (used to pin the incremental paths) ---------------
    def full_hier(self, tokens: np.ndarray) -> SeqState:
        """HierGen state after all of `tokens`, computed from scratch."""
        return self.prefill(np.asarray(tokens), "hier")

    def full_top(self, top_inputs: list[np.ndarray]):
        """Top encoder over a whole list of coarse inputs, from scratch."""
        return self.top_encode(np.stack(top_inputs), 0, None)


# ----------------------------------------------------------------------------
# Kernel-level references
# ----------------------------------------------------------------------------

def decode_attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, p0: int) -> np.ndarray:
    """Attention of q_len new queries at positions p0.. over one (sequence, head).

    q: [q_len, dh]; k, v: [n, dh] with n >= p0 + q_len.  Query i sees keys
    0..p0+i.  Returns [q_len, dh]."""
    ql = q.shape[0]
    out = attention(q[:, None, :], k[:, None, :], v[:, None, :],
                    p0 + np.arange(ql), np.arange(k.shape[0]))
    return out[:, 0, :]


def tpm(tok_per_s: float, gib: float) -> float:
    """Throughput per unit memory: tokens/s divided by GiB (explainer, memory-wall
    and 475x sections)."""
    return tok_per_s / gib
