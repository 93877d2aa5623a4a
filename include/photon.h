/*
 * photon.h -- C ABI of the B200 PHOTON inference library (libphoton.so).
 *
 * PHOTON (ACL 2026, "Hierarchical Autoregressive Modeling for Lightspeed and
 * Memory-Efficient Language Generation") keeps a hierarchy of latent
 * streams: a bottom-up Context Chunker + Context Encoder compress tokens into
 * coarse states, and top-down Context Converter + Context Decoder stacks
 * write tokens back chunk by chunk.  This library implements, for L = 2
 * levels, the hierarchical prefill and the two per-chunk decode procedures
 * described on the "PHOTON vertical scan" explainer page (RecGen section):
 * HierGen (re-encode the written tokens) and RecGen (feed the decoder's
 * bottleneck reconstruction A-hat straight to the top encoder).
 *
 * Conventions (all entry points):
 *  - Every call returns PHOTON_OK (0) or a negative PHOTON_ERR_* code and
 *    never exits or throws.  photon_last_error() returns a message for the
 *    last failing call on the calling thread.
 *  - Device pointers ("d_" prefix) are caller-owned CUDA device memory, for
 *    example torch tensors' data_ptr().  The library owns the model, the
 *    caches and all their device buffers.
 *  - `stream` is a cudaStream_t (NULL = legacy default stream).  Work is
 *    enqueued on it and the calls return before the GPU finishes, except
 *    where a call is documented as synchronising.
 *  - Storage: dtype 0 = fp32 everywhere; dtype 1 = bf16 weights, KV caches
 *    and inter-kernel activations with fp32 residual stream, accumulation,
 *    norms, softmax and GELU.
 *  - Token ids are int32.  Sequences in a batch never interact.
 */
#ifndef PHOTON_H_
#define PHOTON_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define PHOTON_API __attribute__((visibility("default")))
#else
#define PHOTON_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct photon_model photon_model; /* opaque, library-owned */
typedef struct photon_cache photon_cache; /* opaque, library-owned */

/* Model shape.  Explainer, architecture section (module table and the
 * hierarchy setting: L = 2, C1 = C2 = 4, or 2 x 2).  Readings taken where the
 * pages are silent: pre-RMSNorm blocks (gain 1), full multi-head attention
 * with rotate-half RoPE per stream, erf-GELU MLP of width mlp_mult*d_model,
 * no biases, untied head.  Constraints checked by photon_init_weights:
 * levels == 2; d_model == n_heads * head_dim; head_dim in {32, 64};
 * d_model % 64 == 0; 1 <= C1, C2 <= 4; conv_kernel == 0 or equal to both C1
 * and C2 (the converter is a transposed 1-D convolution with kernel = stride
 * = C); dtype in {0, 1}. */
typedef struct photon_config {
  int32_t vocab;
  int32_t d_model;
  int32_t n_heads;
  int32_t head_dim;
  int32_t levels;        /* must be 2 */
  int32_t chunk[2];      /* C1 (tokens per level-1 state), C2 (level-1 states per top state) */
  int32_t enc_layers[2]; /* L1 (level-1 encoder), Ltop (top encoder) */
  int32_t dec_layers[2]; /* Ld1 (token decoder), Ld2 (level-2 decoder) */
  int32_t mlp_mult;      /* MLP width multiple (4) */
  int32_t conv_kernel;   /* 0 = C_l; otherwise must equal C1 and C2 */
  int32_t dtype;         /* 0 fp32, 1 bf16 */
  float init_std;        /* 0.02 */
  float rope_theta;      /* 10000 */
  float norm_eps;        /* 1e-6 */
} photon_config;

enum {
  PHOTON_OK = 0,
  PHOTON_ERR_ARG = -1,          /* invalid argument or shape */
  PHOTON_ERR_OOM = -2,          /* device allocation failed */
  PHOTON_ERR_CUDA = -3,         /* a CUDA runtime call failed */
  PHOTON_ERR_CAPACITY = -4,     /* decoding past max_new_chunks */
  PHOTON_ERR_MODE = -5,         /* HierGen on a cache whose level-1 KV was discarded */
  PHOTON_ERR_DEVICE_CHECK = -6  /* a kernel reported an error word (bad token id, expired wait) */
};

enum { PHOTON_MODE_HIER = 0, PHOTON_MODE_REC = 1 };

/* Builds a model with weights drawn on the device by the counter-based
 * generator: tensor t (fixed order: embed, chunker1, level-1 encoder
 * blocks + final gain, chunker2, top blocks + final gain, converter2,
 * level-2 decoder blocks + gain, converter1, token decoder blocks + gain,
 * head; per block g_attn, wq, wk, wv, wo, g_mlp, w1, w2), element e: an
 * N(0, init_std^2) variable by Marsaglia's polar method from the SplitMix64
 * stream of key mix(mix(seed + gamma*(t+1)) + gamma*(e+1)) (attempt a takes
 * the stream's outputs 2a+1 and 2a+2 as 53-bit uniforms on [-1, 1); ln by its
 * atanh series; every fp64 step correctly rounded), rounded to fp32 then to
 * the storage type; RMSNorm gains are 1.  Linear maps are [out, in].
 * Synchronising.  Errors: ERR_ARG (bad config or out==NULL), ERR_OOM,
 * ERR_CUDA. */
PHOTON_API int photon_init_weights(const photon_config* cfg, uint64_t seed, photon_model** out);

/* Frees a model.  Every cache built on it must have been freed first
 * (ERR_ARG otherwise).  Synchronising. */
PHOTON_API int photon_free_model(photon_model* m);

/* Hierarchical prefill (explainer, module table: Chunker -> Encoder per
 * level; the top encoder's KV is the only global cache).
 *   d_tokens: device int32 [B, T] row-major prompt ids, 0 <= id < vocab.
 *   T must be a positive multiple of C1*C2 (partial chunks are undefined).
 *   mode: PHOTON_MODE_HIER keeps the level-1 encoder KV for HierGen;
 *         PHOTON_MODE_REC discards it after prefill (RecGen section: only the
 *         top-level global KV is kept) and, when no HierGen cache is alive,
 *         releases the level-1 encoder and chunker weights until the next
 *         prefill needs them.
 *   max_new_chunks: decode steps this cache can take (each step appends one
 *         top-level entry and, in HIER mode, C2 level-1 entries).
 *   prefix: NULL, or a cache prefilled in HIER mode with B = 1 whose context
 *         precedes every sequence of this batch (shared-prefix serving).  The
 *         new cache reads the prefix's top and level-1 KV in place; the
 *         prefix must outlive it.
 *   out: receives the new cache.  Invalid token ids set the device error
 *         word (see photon_cache_info).
 *   B * C2 must be at most 65535 (the attention kernels' grid limit).
 * Errors: ERR_ARG, ERR_OOM, ERR_CUDA. */
PHOTON_API int photon_prefill(photon_model* m, const photon_cache* prefix, const int32_t* d_tokens,
                   int32_t B, int32_t T, int32_t mode, int32_t max_new_chunks, void* stream,
                   photon_cache** out);

/* One HierGen decode step = one top-level chunk of C1*C2 tokens per sequence
 * (explainer, RecGen section, the three-stage loop): Converter_2 and the
 * level-2 decoder turn the pending top output into A-hat; Converter_1 and the
 * token decoder write the tokens greedily (lowest id on ties), the chunk's
 * sub-chunks in parallel; the tokens are re-encoded (Chunker_1, level-1
 * encoder with its cache, Chunker_2) and the top encoder advances one step.
 *   d_out_tokens: device int32 [B, C1*C2]; token t = j*C1 + i is position i
 *                 of level-1 sub-chunk j.
 *   d_out_logits: NULL or device fp32 [B, C1*C2, vocab] logits of each token.
 * Errors: ERR_ARG, ERR_MODE (cache prefilled in REC mode), ERR_CAPACITY. */
PHOTON_API int photon_decode_step_hier(photon_model* m, photon_cache* c, int32_t* d_out_tokens,
                            float* d_out_logits, void* stream);

/* One RecGen decode step (explainer, RecGen section): tokens as in HierGen,
 * then Chunker_2(A-hat) is fed straight to the top encoder; no level-1
 * encoder work and no level-1 cache.  Same buffers and errors as HierGen
 * except that it accepts caches of both modes. */
PHOTON_API int photon_decode_step_rec(photon_model* m, photon_cache* c, int32_t* d_out_tokens,
                           float* d_out_logits, void* stream);

/* The decode step with its test hooks.
 *   mode: PHOTON_MODE_HIER or PHOTON_MODE_REC.
 *   d_force_tokens: NULL or device int32 [B, C1*C2]; entries >= 0 replace the
 *     token fed back into the decoder (and, in HierGen, re-encoded), entries
 *     < 0 keep the greedy choice.  d_out_tokens always receives the greedy
 *     choice.  (Teacher forcing.)
 *   d_force_a: NULL or device [B*C2, d_model] of the storage type; in RecGen
 *     it replaces A-hat as the top encoder's input (the condition of
 *     Theorem A.6, explainer RecGen section).  Ignored in HierGen.
 * Errors as above. */
PHOTON_API int photon_decode_step_ex(photon_model* m, photon_cache* c, int32_t mode, int32_t* d_out_tokens,
                          float* d_out_logits, const int32_t* d_force_tokens,
                          const void* d_force_a, void* stream);

/* RecGen decode of n consecutive top-level chunks in one call (explainer,
 * RecGen section): the same tokens as n calls of photon_decode_step_rec,
 * written to d_out_tokens [B, n * C1 * C2] (device, row-major; chunk k in
 * columns k*C .. k*C + C - 1).  Because a RecGen chunk's top-encoder input
 * (Chunker_2 of A-hat) does not depend on its tokens, the token decoder of
 * chunk k runs on an internal stream while the main chain (Converter_2,
 * Decoder_2, Chunker_2, top-encoder step) of chunk k + 1 runs on `stream`;
 * all work is joined into `stream` before the call returns (asynchronous, as
 * the other decode calls).  Allocates its token-branch buffers on the first
 * call (counted in the cache's bytes).  Errors: ERR_ARG, ERR_CAPACITY (more
 * chunks than the cache has room for), ERR_OOM, ERR_CUDA. */
PHOTON_API int photon_decode_rec_chunks(photon_model* m, photon_cache* c, int32_t n_chunks,
                                        int32_t* d_out_tokens, void* stream);

/* Frees a cache and its device buffers.  A prefix cache can only be freed
 * after every cache built on it (ERR_ARG otherwise).  Stream-ordered: the
 * buffers return to the library's pool on the stream of the cache's last
 * call, after all of its pending work, and the call returns without waiting
 * (a cache built on a shared prefix waits for its own work).  The handle is
 * invalid afterwards. */
PHOTON_API int photon_free_cache(photon_cache* c);

/* Token choice of the cache's later decode steps (both modes).
 * temperature == 0: greedy (lowest id among the maxima), the default.
 * temperature > 0: each token is drawn from softmax(logits / temperature) by
 * the Gumbel-max rule: argmax_v(logit_v / T + G_v), ties to the lowest id,
 * with standard Gumbel noise G_v = -ln(-ln u_v) from a counter-based
 * generator (a pure function of seed, the sequence's batch row b, the
 * token's index t among the tokens this cache has generated, and v):
 *   K   = mix64(mix64(seed + g*(b+1)) + g*(t+1))
 *         (mix64: the SplitMix64 output function, g = 0x9E3779B97F4A7C15),
 *   h   = MurmurHash3_x86_32 with seed 0 of the 12-byte message K (8 bytes,
 *         little-endian) followed by v (4 bytes, little-endian),
 *   u_v = (floor(h / 256) + 1/2) / 2^24.
 * The explainer's quality section (several varied queries per prompt)
 * motivates sampling; the pages do not fix the sampler.  Tokens written by
 * photon_decode_step_ex's teacher forcing are unaffected; the own choices
 * are sampled.  Host-only (no device work); the next decode call re-captures
 * its graphs.  Errors: ERR_ARG (NULL cache, negative, NaN, infinite or
 * subnormal-reciprocal temperature). */
PHOTON_API int photon_cache_set_sampling(photon_cache* c, float temperature, uint64_t seed);

/* Nucleus (top-p) restriction of the cache's temperature sampling: each
 * draw runs over the smallest set of most probable tokens whose probability
 * under softmax(logits / T) reaches top_p (ties at its edge included), i.e.
 * {v : p_v >= theta} for the largest such theta, renormalised; the Gumbel
 * noise is photon_cache_set_sampling's.  top_p = 1 (the default) turns it
 * off; it has no effect while the temperature is 0.  Such heads write their
 * logits and draw in a separate kernel instead of the fused epilogue.
 * Host-only; the next decode call re-captures its graphs.  Errors: ERR_ARG
 * (NULL cache, top_p outside (0, 1]). */
PHOTON_API int photon_cache_set_top_p(photon_cache* c, float top_p);

/* Kernel-level draw (tests): row r of d_logits [rows, V] (fp32) is a head
 * row b*C2 + j emitting token j*C1 + i of chunk *d_chunk (device int32);
 * d_out[r] receives its draw under (temperature, top_p, seed) exactly as a
 * sampling decode step would.  Errors: ERR_ARG, ERR_CUDA. */
PHOTON_API int photon_sample_logits(const float* d_logits, int32_t rows, int32_t V, float temperature,
                                    float top_p, uint64_t seed, const int32_t* d_chunk, int32_t C1, int32_t C2,
                                    int32_t i, int32_t* d_out, void* stream);

typedef struct photon_cache_stats {
  int32_t B, T, mode;
  int32_t N;          /* top-level entries visible (prefix + own) */
  int32_t N1;         /* level-1 entries visible (0 once discarded) */
  int32_t n_prefix;   /* top entries read from the shared prefix */
  int32_t n1_prefix;  /* level-1 entries read from the shared prefix */
  int32_t capacity;   /* own top-level slots */
  int32_t steps;      /* decode steps taken */
  int32_t max_new_chunks;
  int32_t device_error; /* first error word reported by a kernel, 0 if none */
  int32_t l1_resident;  /* 1 while the level-1 KV is allocated */
  uint64_t kv_bytes;    /* top + level-1 KV allocated for this cache */
  uint64_t workspace_bytes;
  int32_t graph_steps;  /* decode steps replayed from a captured CUDA graph */
  int32_t graph_kernels; /* kernels in that graph (0 before the first capture) */
} photon_cache_stats;

/* Cache bookkeeping.  Synchronises the cache's last stream to read the
 * device error word.  Errors: ERR_ARG. */
PHOTON_API int photon_cache_info(photon_cache* c, photon_cache_stats* out);

typedef struct photon_model_stats {
  uint64_t param_count;       /* all parameters */
  uint64_t resident_bytes;    /* weight bytes currently on the device */
  uint64_t encoder_bytes;     /* level-1 encoder + chunker-1 weight bytes */
  int32_t encoder_resident;   /* 1 if those weights are on the device */
  int32_t n_tensors;
  int32_t live_caches;
  int32_t tcgen05_gemm;       /* 1 if the tcgen05/TMA GEMM path is available */
  uint64_t encoder_restores;  /* times released encoder weights came back by a host-to-device copy */
  uint64_t encoder_regenerations; /* ... by being drawn again (the first draw not counted) */
  int32_t kv_page_rows;       /* paged top KV: positions per page (0: no page pool) */
  int32_t kv_pool_pages;      /* pages in the pool */
  int32_t kv_free_pages;      /* pages no live cache holds (released ones included) */
  int32_t kv_paged_caches;    /* live caches built by photon_prefill_paged */
  uint64_t kv_pool_bytes;     /* device bytes of the pool (every top layer, K and V) */
} photon_model_stats;

PHOTON_API int photon_model_info(const photon_model* m, photon_model_stats* out);

/* Residency of the level-1 encoder and Chunker_1 weights (explainer, RecGen
 * section: only the decoders, and the top encoder that RecGen feeds, have to
 * stay on the device while decoding).  A RecGen prefill releases them when
 * no HierGen cache is alive; the next prefill or HierGen step needs them
 * back:
 *   PHOTON_ENC_RESTORE (default): host-to-device copy from a pinned host copy
 *     the library makes at the first release (a trained model's weights
 *     would come back this way);
 *   PHOTON_ENC_REGENERATE: drawn again on the device from the seed;
 *   PHOTON_ENC_KEEP: never released (more resident memory, no restore).
 * Affects later prefills.  Errors: ERR_ARG. */
enum { PHOTON_ENC_RESTORE = 0, PHOTON_ENC_REGENERATE = 1, PHOTON_ENC_KEEP = 2 };
PHOTON_API int photon_model_set_encoder_residency(photon_model* m, int32_t policy);

/* Copies parameter tensor `index` (generator order) into d_dst as stored:
 * the storage type for drawn tensors, fp32 for RMSNorm gains; out_bytes
 * receives the size.  Call with d_dst = NULL to query the size.  The level-1
 * encoder tensors are regenerated if they are not resident.
 * Errors: ERR_ARG (index, buffer too small). */
PHOTON_API int photon_export_weight(photon_model* m, int32_t index, void* d_dst, size_t dst_bytes,
                         size_t* out_bytes, void* stream);

enum {
  PHOTON_STATE_TOP_K = 0,   /* [B][H][N_own][head_dim] own top-level keys (post-RoPE), layer `layer` */
  PHOTON_STATE_TOP_V = 1,   /* same layout, values */
  PHOTON_STATE_L1_K = 2,    /* [B][H][N1_own][head_dim] level-1 keys */
  PHOTON_STATE_L1_V = 3,
  PHOTON_STATE_PENDING_O = 4, /* [B][d_model] top output after the final norm (conditions the next chunk) */
  PHOTON_STATE_A_HAT = 5,   /* [B*C2][d_model] last step's level-2 decoder reconstruction */
  PHOTON_STATE_A = 6        /* [B*C2][d_model] last HierGen step's level-1 encoder states */
};

/* Data-parallel serving of a shared prefix (multi-query serving over one
 * long context, the explainer's quality section): one rank prefills the
 * prefix, the others receive its state instead of recomputing it.
 *
 * photon_prefill_shell allocates and sets up a cache exactly as
 * photon_prefill(m, prefix, tokens, B, T, mode, max_new_chunks) would,
 * positions included, but runs no kernel on its state: the top and level-1
 * KV and the pending top output hold whatever the allocator returned until
 * the caller fills them (e.g. with a broadcast of another rank's prefilled
 * cache of the same model, B, T, mode and max_new_chunks).  Errors as
 * photon_prefill; ERR_ARG for a model of other than two levels.
 *
 * photon_cache_state_buffer returns the device address and size in bytes
 * of one whole state buffer a prefill writes, with every layer and the
 * unused capacity included: which = PHOTON_STATE_TOP_K / TOP_V ([Ltop][B]
 * [H][Ncap][head_dim]), L1_K / L1_V ([L1][B][H][N1cap][head_dim]; NULL and
 * 0 once a RecGen prefill discarded them) or PENDING_O ([B][d_model]); all
 * of the storage type.  Two caches built by the same calls on the same
 * model have buffers of equal sizes, so copying each buffer from one to
 * the other makes the second cache equal to the first.  The memory stays
 * owned by the cache; the caller must order its writes after the
 * cache's stream.  Errors: ERR_ARG (NULL pointers, another state). */
PHOTON_API int photon_prefill_shell(photon_model* m, const photon_cache* prefix, int32_t B, int32_t T,
                         int32_t mode, int32_t max_new_chunks, void* stream, photon_cache** out);
PHOTON_API int photon_cache_state_buffer(photon_cache* c, int32_t which, void** d_ptr, size_t* bytes);

/* Paged top KV (the top encoder's cache grows by one entry per generated
 * chunk, the explainer's RecGen and memory sections; many requests over one
 * shared context, its quality section).  A cache built by
 * photon_prefill_paged keeps its own top-level keys and values in pages of a
 * pool the model owns instead of a [B][H][Ncap][head_dim] block sized for
 * max_new_chunks up front: a page holds page_rows consecutive positions of
 * one sequence, for every head, in every top layer (K and V); pages are
 * taken when the prefill or a decode step first writes into them, and come
 * back to the pool when the cache is freed (reusable once the work queued
 * on the cache's stream before the free has finished).  The computation is
 * the contiguous cache's: same kernels, same tokens.
 *
 * photon_model_set_kv_pages allocates the pool: pool_pages pages of
 * page_rows positions, Ltop * 2 * pool_pages * n_heads * page_rows *
 * head_dim elements of the storage type; (0, 0) frees it.  Replaces an
 * existing pool; refused while a paged cache is live.  Errors: ERR_ARG
 * (model of other than two levels, sizes, paged caches live), ERR_OOM.
 *
 * photon_prefill_paged takes photon_prefill's arguments and errors, plus
 * ERR_ARG when the model has no pool and ERR_CAPACITY when the pool cannot
 * supply the prompt's pages.  A decode step that needs a page the pool
 * cannot supply fails with ERR_CAPACITY before running anything.  A paged
 * cache may read a contiguous shared prefix but cannot be one, and has no
 * single top-KV state buffer (photon_cache_state_buffer refuses TOP_K /
 * TOP_V); photon_export_state gathers its pages. */
PHOTON_API int photon_model_set_kv_pages(photon_model* m, int32_t page_rows, int32_t pool_pages);
PHOTON_API int photon_prefill_paged(photon_model* m, const photon_cache* prefix, const int32_t* d_tokens,
                                    int32_t B, int32_t T, int32_t mode, int32_t max_new_chunks, void* stream,
                                    photon_cache** out);

/* Copies a piece of cache state (storage type) into d_dst, compacted to
 * the entries in use.  Call with d_dst = NULL to query the size.
 * Errors: ERR_ARG (unknown state, layer out of range, discarded level-1 KV,
 * buffer too small). */
PHOTON_API int photon_export_state(photon_cache* c, int32_t which, int32_t layer, void* d_dst,
                        size_t dst_bytes, size_t* out_bytes, void* stream);

/* Kernel-level entry: C[M, N] (fp32, row stride ldc) = A[M, K] * W[N, K]^T
 * with A, W of the storage type (row strides lda, ldw in elements).
 * path: 0 = the library's choice, 1 = CUDA-core kernel, 2 = tcgen05 kernel
 * (bf16 only; K % 64 == 0, N % 64 == 0).  splits / swap (-1 = automatic)
 * steer the tcgen05 kernel's split-K count and operand swap.  Allocates its
 * split-K scratch internally.  Errors: ERR_ARG (unsupported shape or path). */
PHOTON_API int photon_gemm(int32_t dtype, const void* d_A, int64_t lda, const void* d_W, int64_t ldw,
                int32_t M, int32_t N, int32_t K, float* d_C, int64_t ldc, int32_t path,
                int32_t splits, int32_t swap, void* stream);

/* Kernel-level entry for the pre-norm projection of every encoder and
 * decoder block (each block normalises its residual stream before the
 * attention and MLP projections; RMSNorm is this library's reading of the
 * norm): C[M, N] (fp32, row stride ldc) = bf16(RMSNorm(x)) * W[N, K]^T with
 * RMSNorm(x)[r, k] = x[r, k] / sqrt(mean_k x[r, k]^2 + eps) * g[k].
 * x: fp32 [M, K] (row stride ldx elements, 16-byte aligned rows), g: fp32
 * [K], W: bf16 [N, K] (row stride ldw).  bf16 only.  Runs the few-token
 * tcgen05 kernel that normalises its own operand; where that kernel does not
 * take the shape (see gemm_tc_fuses_norm: M <= 256, K % 64 == 0, N % 64 == 0,
 * a cluster plan exists) the norm runs as a separate kernel before the
 * GEMM, with the same result up to the order of the sum of squares.
 * Allocates its scratch internally.  Errors: ERR_ARG (bad arguments). */
PHOTON_API int photon_gemm_rmsnorm(const float* d_x, int64_t ldx, const float* d_g, float eps,
                                   const void* d_W, int64_t ldw, int32_t M, int32_t N, int32_t K,
                                   float* d_C, int64_t ldc, void* stream);

/* Kernel-level entry: causal prefill attention (Encoder_1 over the level-1
 * positions of a prompt, the top encoder over its chunks).  For G groups x
 * H heads, q_len new queries at positions p0..p0+q_len-1 attend to keys
 * 0..p0+i: positions < n_pre from a shared prefix d_kp/d_vp [H][cap_pre]
 * [head_dim] (the same for every group; NULL when n_pre = 0), later ones
 * from d_k/d_v [G][H][cap][head_dim] at slot pos - n_pre (post-RoPE keys,
 * storage type).  Slots past p0 - n_pre + q_len and prefix rows past n_pre
 * are never read, whatever they hold.  d_q, d_o: [G*q_len][H*head_dim].
 * Scale 1/sqrt(head_dim).  path: 0 = the library's choice, 1 = CUDA-core
 * kernel, 2 = mma.sync tiles (bf16, head_dim 64), 3 = tcgen05 kernel (bf16,
 * head_dim 64, q_len >= 128, and with a prefix G*q_len >= 128).  d_err as
 * for photon_attn_decode.  Allocates the prefix pass's partials internally.
 * Errors: ERR_ARG (bad arguments, or a path that does not take the shape). */
PHOTON_API int photon_attn_prefill(int32_t dtype, const void* d_q, const void* d_k, const void* d_v,
                                   const void* d_kp, const void* d_vp, int32_t G, int32_t H,
                                   int32_t head_dim, int32_t cap, int32_t q_len, int32_t p0,
                                   int32_t cap_pre, int32_t n_pre, int32_t path, void* d_o,
                                   int32_t* d_err, void* stream);

/* Kernel-level entry: split-K decode attention (the top-encoder decode
 * kernel).  For G groups x H heads, q_len <= 4 new queries at positions
 * p0..p0+q_len-1 attend causally over keys 0..p0+i of a cache
 * d_k/d_v [G][H][cap][head_dim] (storage type, post-RoPE keys);
 * d_q and d_o are [G*q_len][H*head_dim].  Scale 1/sqrt(head_dim).
 * d_err (device int32, nullable): the kernels' error word.  A bounded wait
 * that runs out (about 2 s; the long-cache streamed kernel waits on its bulk
 * copies) leaves d_o unwritten and sets *d_err to a nonzero code, which the
 * caller reads after the stream has synchronised (zero it before the call).
 * With d_err NULL such a timeout goes unreported.
 * Allocates its split scratch internally.  Errors: ERR_ARG. */
PHOTON_API int photon_attn_decode(int32_t dtype, const void* d_q, const void* d_k, const void* d_v, int32_t G,
                       int32_t H, int32_t head_dim, int32_t cap, int32_t q_len, int32_t p0,
                       void* d_o, int32_t* d_err, void* stream);

/* Bytes of split scratch photon_attn_decode needs for this shape (0 when
 * every (group, head) pair is one chunk, or the long-cache streamed kernel
 * takes it); a host-side planning query that launches nothing.  Written to
 * *out_bytes.  Errors: ERR_ARG. */
PHOTON_API int photon_attn_decode_scratch_bytes(int32_t dtype, int32_t G, int32_t H, int32_t head_dim,
                                                int32_t cap, int32_t q_len, int32_t p0, uint64_t* out_bytes);

/* Allocation-free variant of photon_attn_decode (this entry point has no
 * counterpart in the PHOTON paper; it exists for callers that cannot let the
 * library allocate device memory: a host framework that owns all device
 * memory through its own pool, a latency-critical loop where an allocation
 * may synchronise the device, or a process close to its memory limit).
 * Same arguments, layouts and results as photon_attn_decode, but the split
 * scratch is a fixed 256 KiB array compiled into the library (held on every
 * GPU that loads the library until the process exits); the call allocates
 * and frees nothing.  The array's device address is looked up during the
 * first call on each device, so make that first call before any stream
 * capture.  A shape that needs no split scratch never looks it up.  All
 * calls share the array: calls whose GPU work may overlap race on it and
 * must be ordered by the caller.  d_err as for photon_attn_decode (a word
 * the caller owns; NULL leaves wait timeouts unreported).  Errors: ERR_ARG
 * (bad arguments), ERR_CAPACITY (the shape needs more than the 256 KiB of
 * scratch; the message says how much), ERR_CUDA. */
PHOTON_API int photon_attn_decode_noalloc(int32_t dtype, const void* d_q, const void* d_k,
                                          const void* d_v, int32_t G, int32_t H, int32_t head_dim,
                                          int32_t cap, int32_t q_len, int32_t p0, void* d_o,
                                          int32_t* d_err, void* stream);

/* Teacher-forced scoring (explainer, quality section: PHOTON's reported
 * quality is measured with teacher-forced HierGen).  For prompts d_tokens
 * [B, T] (device, row-major; T a multiple of C1*C2 and longer than one
 * chunk) writes d_out_logprob [B, T - C1*C2] (device fp32): the natural-log
 * probability of token t (t >= C1*C2) given the prompt before it.  The
 * bottom-up pass encodes the true tokens; the top output of chunk k
 * conditions chunk k + 1 through Converter_2, Decoder_2 and Converter_1, and
 * the token decoder reads the chunk's true tokens (one causal pass per
 * sub-chunk).  The first chunk has no conditioning and is not scored.
 * Synchronising (it reports device checks).  Allocates its temporaries from
 * the library's pool.  Long batches are scored a slice of whole sequences at
 * a time, so that the decoders' (sequence, chunk, sub-chunk) groups stay
 * within the attention kernels' grid limit.  One sequence may hold at most
 * 65535 / (C2 * min(2*C1 - 1, 4)) + 1 chunks.  Errors: ERR_ARG (including
 * a longer sequence), ERR_OOM, ERR_CUDA, ERR_DEVICE_CHECK (a token id
 * outside the vocabulary). */
PHOTON_API int photon_score(photon_model* m, const int32_t* d_tokens, int32_t B, int32_t T,
                            float* d_out_logprob, void* stream);

/* ------------------------------------------------------------------------
 * Any number of levels (explainer, architecture section: every module is
 * written for a general level l; RecGen section: Theorem A.6 needs A-hat = A
 * only at the L -> L-1 interface).  L = 1 is a single-level block model
 * (token blocks of C_1 merged by one linear map, a causal encoder over the
 * blocks, a block-local token decoder), the shape of the Block Transformer
 * the explainer compares PHOTON against; L = 3 adds a middle level.
 *
 * Level l = 1..L has chunk size chunk[l-1], encoder depth enc_layers[l-1]
 * (the last is the top encoder) and decoder depth dec_layers[l-1] (the first
 * is the token decoder).  Tensor order: embed; for l = 1..L chunker_l and
 * encoder_l (blocks + final gain); for l = L..1 converter_l and decoder_l
 * (blocks + final gain); head -- for L = 2 the same tensors and draws as
 * photon_init_weights.  A model made here runs through photon_prefill,
 * photon_decode_step_hier / _rec / _ex, photon_decode_rec_chunks,
 * photon_cache_info, photon_export_weight / _state and the free calls.
 * Prefill encodes bottom-up through every level; a decode step goes
 * top-down level by level (Converter_l, then Decoder_l over its C_l
 * conditioning positions for every group at once), then the token decoder
 * writes the chunk's C tokens; HierGen re-encodes them through levels
 * 1..L-1 (whose caches grow) and RecGen (L >= 2) feeds Chunker_L(A-hat_L)
 * to the top encoder, keeping only the top cache.  Every weight stays
 * resident.  The two-level optimisations (the forked and pipelined RecGen
 * branches, the persistent top step) are specific to photon_init_weights
 * models; steps here are captured once per mode into a graph and replayed.
 * Not supported on these models: shared prefixes, photon_score,
 * photon_multi_query. */
#define PHOTON_MAX_LEVELS 4
typedef struct {
  int32_t vocab, d_model, n_heads, head_dim;
  int32_t levels;                         /* L, 1..PHOTON_MAX_LEVELS */
  int32_t chunk[PHOTON_MAX_LEVELS];       /* C_1 .. C_L, each 1..4 */
  int32_t enc_layers[PHOTON_MAX_LEVELS];  /* encoder depth of levels 1..L */
  int32_t dec_layers[PHOTON_MAX_LEVELS];  /* decoder depth of levels 1..L */
  int32_t mlp_mult, dtype;
  float init_std, rope_theta, norm_eps;
} photon_level_config;

/* Errors: ERR_ARG (bad config), ERR_OOM, ERR_CUDA.  Synchronising. */
PHOTON_API int photon_init_weights_levels(const photon_level_config* cfg, uint64_t seed, photon_model** out);

/* ------------------------------------------------------------------------
 * Multi-query aggregation (explainer, quality section: the single-query
 * quality gap is closed by running several slightly varied queries, about
 * nine, and combining their outputs by majority vote or best-of-N).
 *
 * A query group is N consecutive rows of a batch.  The rows may hold
 * different prompts (the caller's variations), and each row draws its own
 * sampling noise (the generator is keyed by the row). */
enum {
  PHOTON_AGG_VOTE = 0, /* the row whose span equals the spans of the most rows */
  PHOTON_AGG_BEST = 1  /* the row with the largest sum of log-probabilities over its span */
};

/* Picks one row per group.  Group q holds rows q*N .. q*N + N - 1 of
 * d_cand [Q*N, L] (device int32, row-major; PHOTON_AGG_VOTE) or of
 * d_logprob [Q*N, L] (device fp32; PHOTON_AGG_BEST).  Only positions
 * [span_begin, span_begin + span_len) of a row take part.
 *   VOTE: count[n] = the number of rows of the group whose span is identical
 *         to row n's (row n included); the winner has the largest count.
 *   BEST: sum[n] = the fp64 sum of row n's span; the winner has the largest
 *         sum, and a NaN sum ranks below every number.
 * Ties go to the lower row.  d_choice [Q] (device int32) receives the
 * winner's index within its group (0 .. N-1).  d_score [Q*N] (device fp64,
 * may be NULL) receives count[n] or sum[n] for every row.  The buffers are
 * the caller's and must hold the sizes above.  Asynchronous on `stream`.
 * One CTA per group.  The vote costs O(N^2 * span_len) reads, so it suits
 * groups of a few dozen rows.  Q = 0 is a no-op.  Errors: ERR_ARG (unknown
 * mode, N <= 0, Q < 0, a span outside [0, L], a NULL buffer that the mode
 * reads or writes), ERR_CUDA. */
PHOTON_API int photon_aggregate(int32_t mode, const int32_t* d_cand, const float* d_logprob, int32_t Q,
                                int32_t N, int32_t L, int32_t span_begin, int32_t span_len,
                                int32_t* d_choice, double* d_score, void* stream);

/* The whole multi-query pass.  d_prompts [Q*N, T] (device int32; T a
 * positive multiple of C1*C2) are prefilled in RecGen mode, after `prefix`
 * if one is given.  Every row decodes n_chunks chunks with temperature /
 * top-p sampling (photon_cache_set_sampling, photon_cache_set_top_p; a
 * temperature of 0 is greedy).  Row r of d_cand [Q*N, n_chunks*C1*C2]
 * (device int32) receives its continuation.  Each group then picks its
 * winner over the whole continuation:
 *   PHOTON_AGG_VOTE: photon_aggregate's vote over the continuation tokens.
 *   PHOTON_AGG_BEST: photon_score over prompt + continuation.  The
 *                    log-probabilities of the continuation's tokens are
 *                    summed, i.e. each row's log-likelihood of its
 *                    continuation given its own prompt.  No prefix.
 * d_choice [Q] and d_score [Q*N] (may be NULL) are as in photon_aggregate.
 * The cache and all temporaries come from the library's pool and are
 * released before the call returns.  Synchronising (it reports device
 * checks).  Errors: ERR_ARG (NULL buffer, bad shapes, temperature or top_p
 * out of range, a prefix with PHOTON_AGG_BEST, a vanilla model), ERR_OOM,
 * ERR_CUDA, ERR_DEVICE_CHECK (a token id outside the vocabulary). */
PHOTON_API int photon_multi_query(photon_model* m, const photon_cache* prefix, const int32_t* d_prompts,
                                  int32_t Q, int32_t N, int32_t T, int32_t n_chunks, float temperature,
                                  float top_p, uint64_t seed, int32_t mode, int32_t* d_cand,
                                  int32_t* d_choice, double* d_score, void* stream);

/* ------------------------------------------------------------------------
 * Same-kernel baseline: a vanilla token-level Transformer.
 *
 * The explainer's decode-heavy table (475x section) compares PHOTON's
 * throughput per memory with a vanilla Transformer of similar size.  This is
 * that baseline built from the same kernels: one causal pre-norm stack over
 * the token stream (PHOTON's block: RMSNorm, rotate-half RoPE per token
 * position, full multi-head attention, erf-GELU MLP, no biases), a final
 * RMSNorm and an untied head, with a KV cache over every token.  Weights use
 * the same generator as photon_init_weights (tensor order: embed [V, d];
 * per layer g_attn, Wq, Wk, Wv, Wo, g_mlp, W1, W2; final gain; head [V, d]),
 * so photon_export_weight and photon_model_info work on it.  The PHOTON
 * entry points reject a vanilla model and vice versa. */
typedef struct photon_vanilla_cache photon_vanilla_cache; /* opaque, library-owned */

typedef struct photon_vanilla_config {
  int32_t vocab;
  int32_t d_model;
  int32_t n_heads;
  int32_t head_dim;
  int32_t layers;
  int32_t mlp_mult;
  int32_t dtype;   /* 0 fp32, 1 bf16 */
  float init_std;
  float rope_theta;
  float norm_eps;
} photon_vanilla_config;

/* Model with weights drawn on the device.  Constraints as photon_init_weights
 * (d_model == n_heads * head_dim, head_dim in {32, 64}, d_model % 64 == 0),
 * layers >= 1.  Synchronising.  Errors: ERR_ARG, ERR_OOM, ERR_CUDA. */
PHOTON_API int photon_vanilla_init(const photon_vanilla_config* cfg, uint64_t seed, photon_model** out);

/* Prefill of B prompts d_tokens [B, T] (device, row-major, T >= 2): the
 * first T-1 tokens of each prompt enter the KV cache; the last one is the
 * input of the first decode step.  Room for max_new_tokens decode steps.
 * B must be at most 65535 (the attention kernels' grid limit).
 * Errors: ERR_ARG, ERR_OOM, ERR_CUDA. */
PHOTON_API int photon_vanilla_prefill(photon_model* m, const int32_t* d_tokens, int32_t B, int32_t T,
                                      int32_t max_new_tokens, void* stream, photon_vanilla_cache** out);

/* One token per sequence: feeds the pending token (the last prompt token,
 * then the previous step's choice, or d_force_tokens[b] if given and >= 0)
 * at the next position and writes the greedy choice (lowest id on ties) to
 * d_out_tokens [B].  d_out_logits (nullable) receives fp32 logits [B, V].
 * Steps without logits or forcing replay a captured graph after the first.
 * Errors: ERR_ARG, ERR_CAPACITY (more than max_new_tokens steps), ERR_CUDA. */
PHOTON_API int photon_vanilla_decode_step(photon_model* m, photon_vanilla_cache* c, int32_t* d_out_tokens,
                                          float* d_out_logits, const int32_t* d_force_tokens,
                                          void* stream);

typedef struct photon_vanilla_stats {
  int32_t B, N;            /* sequences; positions in the KV cache */
  int32_t capacity, steps; /* KV capacity; decode steps taken */
  int32_t device_error;    /* device error word (0 = none) */
  int32_t graph_steps;     /* decode steps replayed from the captured graph */
  uint64_t kv_bytes;       /* KV cache bytes */
  uint64_t workspace_bytes;
} photon_vanilla_stats;

/* Synchronises the cache's stream, then reports.  Errors: ERR_ARG, ERR_CUDA. */
PHOTON_API int photon_vanilla_cache_info(photon_vanilla_cache* c, photon_vanilla_stats* out);

/* Stream-ordered release (as photon_free_cache).  Errors: ERR_ARG, ERR_CUDA. */
PHOTON_API int photon_vanilla_free_cache(photon_vanilla_cache* c);

/* Number of kernels this library has launched in this process so far
 * (every launch of every entry point; host-side counter, no GPU access). */
PHOTON_API uint64_t photon_launch_count(void);

/* Message describing the last error on this thread ("" if none). */
PHOTON_API const char* photon_last_error(void);

/* Test hook for the failure paths (no counterpart in the paper): the n-th
 * device allocation the library makes from now on (n = 1: the next one;
 * model weights, caches, workspaces) fails as if the device were out of
 * memory, so the call that makes it returns PHOTON_ERR_OOM and releases
 * what it had allocated.  n = 0 turns the hook off.  Process-wide.
 * Errors: ERR_ARG (n < 0). */
PHOTON_API int photon_debug_fail_alloc(int64_t n);

/* Self-test of the kernels' bounded waits (no counterpart in the paper):
 * launches one thread that waits on a barrier nothing ever arrives on,
 * through the same bounded wait the kernels use, with a budget of
 * limit_cycles clock cycles.  When the budget runs out the kernel writes a
 * nonzero code to d_err (device int32 the caller owns) and returns; the call
 * synchronises the stream and reports it.  The context stays usable.
 * Errors: ERR_DEVICE_CHECK (the wait ran out: the expected outcome),
 * ERR_ARG, ERR_CUDA. */
PHOTON_API int photon_selftest_wait_timeout(int64_t limit_cycles, int32_t* d_err, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* PHOTON_H_ */
