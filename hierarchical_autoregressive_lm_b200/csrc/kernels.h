// Internal launch API of the PHOTON kernels (host side).  Not part of the
// public C ABI; the runtime in runtime.cu is the only caller.
#pragma once

#include <cuda.h>  // CUtensorMap (type only)
#include <cuda_runtime.h>
#include <stdint.h>

namespace photon {

enum DType : int { DT_F32 = 0, DT_BF16 = 1 };
inline size_t dtype_size(int dt) { return dt == DT_F32 ? 4 : 2; }

// What a GEMM does with each accumulator value acc(row, col).
enum EpiKind : int {
  EPI_STORE_T = 0,    // out[row, col] = T(acc)
  EPI_STORE_F32 = 1,  // out[row, col] = acc (fp32)
  EPI_ADD_F32 = 2,    // out[row, col] += acc (fp32 residual stream)
  EPI_GELU_T = 3,     // out[row, col] = T(gelu(acc))
  EPI_QKV = 4,        // fused q/k/v split + RoPE + KV-cache write (see below)
  EPI_ARGMAX = 5,     // LM head: per-tile greedy partials (+ optional fp32 logits)
};

// Epilogue parameters.  For EPI_QKV the GEMM output has 3*d columns
// (q | k | v).  Row r belongs to group g = r / q_len (a sequence, or a
// decoder sub-chunk) and sits at stream position pos = p0 + r % q_len.
// Temperature sampling of the token decoder's head (csrc/sampling.cuh):
// with inv_t > 0 the row's maximum runs over logit * inv_t + Gumbel noise.
struct SampleArgs {
  float inv_t = 0.f;             // 1 / temperature; 0 = greedy
  unsigned long long seed = 0;
  const int* chunk = nullptr;    // device: chunks the cache has generated so far
  int C1 = 0, C2 = 0, i = 0;     // head row = b*C2 + j emits token j*C1 + i of the chunk
};

// q and k are rotated (rotate-half RoPE with the table `rope`, float2
// (cos, sin) per [pos][i], i < dh/2); q goes to q_out[r, :d]; k and v go to
// the caches laid out [G][H][cap][dh] at slot pos - kv_off.
struct Epilogue {
  int kind = EPI_STORE_T;
  void* out = nullptr;
  long long ldo = 0;
  void* q_out = nullptr;
  void* k_cache = nullptr;
  void* v_cache = nullptr;
  int d = 0, H = 0, dh = 0, cap = 0, q_len = 1, p0 = 0, kv_off = 0;
  // Paged KV (kv_table set): k_cache / v_cache are this layer's page arrays
  // [kv_pages][H][kv_page_rows][dh]; slot s of group g is row s % rows of
  // page kv_table[g * kv_tab_len + s / rows].  A slot outside the table or a
  // page outside the arrays is not written.
  const int* kv_table = nullptr;
  int kv_tab_len = 0, kv_page_rows = 0, kv_pages = 0;
  const float2* rope = nullptr;
  // If set, the position of a group's first row is *p0_dev + p0 (read on the
  // device, so a captured decode step can be replayed at later positions).
  const int* p0_dev = nullptr;
  // EPI_ARGMAX: argmax_part[row * argmax_tiles + tile] receives the packed
  // (value, lowest index) maximum of the row over the tile's columns; `out`
  // (if set) receives the fp32 logits.
  unsigned long long* argmax_part = nullptr;
  int argmax_tiles = 0;
  SampleArgs samp;  // EPI_ARGMAX: temperature sampling instead of greedy when samp.inv_t > 0
  // RMSNorm split across a producer / consumer pair of GEMMs (a pre-norm
  // block's residual update and the next projection).  RMSNorm(x)[r] =
  // rstd[r] * x[r] * g with a scalar rstd per row, so the next projection can
  // run on bf16(x * g) and scale its accumulator by rstd[r]:
  //  - producer (EPI_ADD_F32 of k_gemm_dec): also writes xs_out[r, c] =
  //    bf16(x_new[r, c] * g_next[c]) (row stride ldo) and this CTA's partial
  //    sum of x_new^2 over its columns into ssq_out[r * ssq_slots + slot];
  //  - consumer: rstd[r] = 1 / sqrt(sum of ssq_in[r * ssq_slots + 0..ssq_slots)
  //    in slot order / norm_d + norm_eps) multiplies the accumulator before
  //    the rest of the epilogue.
  void* xs_out = nullptr;  // bf16
  const float* g_next = nullptr;
  float* ssq_out = nullptr;
  const float* ssq_in = nullptr;
  int ssq_slots = 0;
  int norm_d = 0;
  float norm_eps = 0.f;
};

// C = A[M, K] * W[N, K]^T with A, W of the storage type, fp32 accumulation.
struct GemmArgs {
  const void* A = nullptr;
  long long lda = 0;
  const void* W = nullptr;
  long long ldw = 0;
  int M = 0, N = 0, K = 0;
  Epilogue ep;
  // Fused RMSNorm of the activation operand: when norm_x is set, A is not
  // read; the kernel uses bf16(norm_x[row] / sqrt(mean(norm_x[row]^2) +
  // norm_eps) * norm_g) instead (norm_x fp32 [M, K], row stride norm_ld).
  // Only the tcgen05 few-token path accepts it (gemm_tc_fuses_norm).
  const float* norm_x = nullptr;
  long long norm_ld = 0;
  const float* norm_g = nullptr;
  float norm_eps = 0.f;
};

// Scratch the GEMM may use for split-K: fp32 partial tiles, and one counter
// per output tile that must be zero before the first split launch (the
// kernel leaves every counter at zero again).
struct GemmWorkspace {
  float* part = nullptr;
  size_t bytes = 0;
  int* counters = nullptr;
  int n_counters = 0;
};
constexpr int kGemmTileCounters = 4096;

// Attention of q_len new queries per group over a key/value cache.
// Query i of group g sits at absolute position p0 + i and sees keys at
// positions 0..p0+i.  Keys at positions < n_pre come from a shared prefix
// cache Kp/Vp ([H][cap_pre][dh], the same for every group); keys at
// positions >= n_pre come from the group's own cache K/V ([G][H][cap][dh])
// at slot pos - n_pre.  Q rows are [G*q_len, q_ld] (head h at column h*dh),
// outputs O the same layout.
struct AttnArgs {
  const void* Q = nullptr;
  long long q_ld = 0;
  const void* K = nullptr;
  const void* V = nullptr;
  int cap = 0;
  const void* Kp = nullptr;
  const void* Vp = nullptr;
  int cap_pre = 0, n_pre = 0;
  int G = 0, H = 0, dh = 0, q_len = 1, p0 = 0;
  void* O = nullptr;
  long long o_ld = 0;
  float scale = 1.0f;
  // If set, the first query's position is *p0_dev + p0 (read on the device).
  const int* p0_dev = nullptr;
  // Largest key count the launch must cover (0: p0 + q_len).  The key
  // chunking is planned for this count; chunks past the live keys write
  // empty partials.
  int n_plan = 0;
  // Paged own keys (kv_table set): K / V are this layer's page arrays
  // [kv_pages][H][kv_page_rows][dh] and own slot s of group g is row
  // s % rows of page kv_table[g * kv_tab_len + s / rows]; a slot outside the
  // table or a page outside the arrays reads row 0 of page 0 instead.
  const int* kv_table = nullptr;
  int kv_tab_len = 0, kv_page_rows = 0, kv_pages = 0;
};

// Row index (in head-size units) of own slot s of (group g, head h) in a
// paged KV array, or -1 when the slot or its page is out of range.
__host__ __device__ inline long long paged_kv_row(const int* table, int tab_len, int rows, int pages, int H, int g,
                                                  int h, int s) {
  if (s < 0 || rows <= 0) return -1;
  const int lp = s / rows;
  if (lp >= tab_len) return -1;
  const int phys = table[(long long)g * tab_len + lp];
  if (phys < 0 || phys >= pages) return -1;
  return ((long long)phys * H + h) * rows + (s - lp * rows);
}

// ---- weights -----------------------------------------------------------
// N(0, sigma^2) draw of tensor `tensor_index` (definition in k_misc.cu).
void launch_init_normal(int dt, void* dst, long long numel, uint64_t seed, int tensor_index,
                        double sigma, cudaStream_t s);
void launch_fill_f32(float* dst, long long n, float v, cudaStream_t s);
void launch_to_f32(int dt, const void* src, float* dst, long long n, cudaStream_t s);

// ---- elementwise / rows -------------------------------------------------
// out[r, :] = E[ids[r], :] (storage type).  Invalid ids set *err.
void launch_embed(int dt, const int32_t* ids, const void* E, void* out, int rows, int d, int vocab,
                  int* err, cudaStream_t s);
// x[r, :] = fp32(E[ids[r], :]).
void launch_embed_f32(int dt, const int32_t* ids, const void* E, float* x, int rows, int d,
                      int vocab, int* err, cudaStream_t s);
// out[r, :] = T(rmsnorm(x[r*in_step + in_off, :]) * g).
void launch_rmsnorm(int dt, const float* x, const float* g, void* out, int rows, int d,
                    int in_step, int in_off, float eps, cudaStream_t s);
// Greedy token for row g of logits (lowest index among maxima), or with
// samp.inv_t > 0 the token drawn from softmax(logits * inv_t) (Gumbel-max,
// sampling.cuh).  Writes the own choice to own[g*C1 + i]; the token fed back
// (force[g*C1+i] if >= 0, else the own choice) to used[g*C1 + i] and
// next_ids[g].
void launch_argmax(const float* logits, long long ld, int rows, int V, int i, int C1,
                   const int32_t* force, int32_t* own, int32_t* used, int32_t* next_ids, int* err,
                   const SampleArgs& samp, cudaStream_t s);
// Greedy token per row from the head GEMM's per-tile partials (EPI_ARGMAX);
// same outputs as launch_argmax.
// argmax from tile partials + embedding of the chosen token into x + its
// RMSNorm into xn (d % 4 == 0)
void launch_argmax_embed_norm(int dt, const unsigned long long* part, int tiles, int rows, int V, int i,
                              int C1, const int32_t* force, int32_t* own, int32_t* used,
                              int32_t* next_ids, int* err, const void* E, float* x, const float* g,
                              void* xn, int d, float eps, cudaStream_t s);
// Nucleus (top-p) draw per row of logits (Gumbel-max over the smallest set
// of most probable tokens reaching top_p); outputs as launch_argmax.
void launch_sample_topp(const float* logits, long long ld, int rows, int V, int i, int C1, const SampleArgs& sa,
                        float top_p, const int32_t* force, int32_t* own, int32_t* used, int32_t* next_ids,
                        int* err, cudaStream_t s);
// out[r] = log softmax(logits[r, :V])[target[r]] (teacher-forced scoring).
void launch_logprob(const float* logits, int V, const int32_t* target, float* out, int rows, int* err,
                    cudaStream_t s);
// chunk_ctr (nullable): incremented once, after the reduction (the chunk count
// the sampling heads read).
void launch_argmax_partials(const unsigned long long* part, int tiles, int rows, int V, int i,
                            int C1, const int32_t* force, int32_t* own, int32_t* used,
                            int32_t* next_ids, int* err, int* chunk_ctr, cudaStream_t s);
// One thread waits on an mbarrier nothing arrives on, with a budget of
// `limit` cycles, through the kernels' bounded wait; sets *err on expiry.
void launch_wait_selftest(long long limit, int* err, cudaStream_t s);
// pos[0] += dN; pos[1] += dN1 (device-side decode positions).
void launch_advance(int* pos, int dN, int dN1, cudaStream_t s);

// ---- persistent single-row step of a chunk-local decoder stack ------------
// All L pre-norm blocks of one token-decoder step in one cooperative launch
// (see k_stack.cu).  rows = groups (one new row each), local caches
// [G][H][cap][64] per layer, the new row at position p0 (< 16).  part /
// tile_cnt: split scratch (stack_local_scratch_bytes; counters zero, left
// zero); bar: one zero-initialised word the launch resets itself.
struct StackLocalLaunch {
  const void* wqkv[8];
  const void* wo[8];
  const void* w1[8];
  const void* w2[8];
  const float* g_attn[8];
  const float* g_mlp[8];
  float* x;
  void* xn;
  void* q;
  void* att;
  void* hid;
  void* kc;
  void* vc;
  long long layer_elems;
  const float2* rope;
  float* part;
  int* tile_cnt;
  int cnt_len;
  unsigned int* bar;
  int* err;
  int rows, d, H, f, L, cap, p0;
  float eps, scale;
  int skip_first_norm;
};
size_t stack_local_scratch_bytes(int rows, int d);
bool stack_local_supported(int rows, int d, int H, int dh, int f, int L, int p0, int cap);
bool launch_stack_local(const StackLocalLaunch& s, cudaStream_t stream);

// ---- persistent top-encoder decode step (k_top_step.cu) -------------------
// Chunker_2 + all top-encoder blocks at one new position + the final norm, in
// one launch.  ch_in: [B, C2*d] bf16 input rows (A-hat or A), row stride
// ch_ld.  Buffers: x fp32 [B, d]; xs, q, att bf16 [B, d]; hid bf16 [B, f];
// ssq fp32 [B, top_step_ssq_slots(d)]; part top_step_part_bytes; cnt
// top_step_counters ints and bar 3 words, zero before the first launch (each
// launch leaves them zero).  kc / vc: the top cache [L][B][H][cap][64]
// (layer stride layer_elems elements), the new key at slot pos[0] - kv_off.
// The launch advances pos[0] by 1 and pos[1] by dN1.
constexpr int kTopMaxLayers = 16;
struct TopStepLaunch {
  const void* ch_in;
  long long ch_ld;
  const void* w_ch;
  const void* wqkv[kTopMaxLayers];
  const void* wo[kTopMaxLayers];
  const void* w1[kTopMaxLayers];
  const void* w2[kTopMaxLayers];
  const float* g_attn[kTopMaxLayers];
  const float* g_mlp[kTopMaxLayers];
  const float* g_final;
  float* x;
  void* xs;
  float* ssq;
  void* q;
  void* att;
  void* hid;
  void* kc;
  void* vc;
  long long layer_elems;
  int cap, kv_off;
  const float2* rope;
  int* pos;
  int dN1;
  void* o_out;
  float* part;
  size_t part_bytes;
  int* cnt;
  unsigned* bar;
  int* err;
  int B, d, H, f, L, C2;
  float eps, scale;
};
struct TopStepPlan;
bool top_step_supported(int B, int d, int H, int dh, int f, int L, int C2, int cap);
size_t top_step_part_bytes(int d, int f, int C2);
int top_step_counters(int d);
int top_step_ssq_slots(int d);
// Builds the launch (tensor maps, work split) once; nullptr if the shape or
// buffers are not supported.
TopStepPlan* top_step_plan(const TopStepLaunch& s);
void top_step_free(TopStepPlan* p);
bool launch_top_step(const TopStepPlan* p, cudaStream_t stream);

// ---- GEMM ----------------------------------------------------------------
void launch_gemm(int dt, const GemmArgs& a, const GemmWorkspace& ws, int* err, cudaStream_t s);
void launch_gemm_simt(int dt, const GemmArgs& a, cudaStream_t s);
// tcgen05 path (bf16): returns false if the shape is not supported.
bool launch_gemm_tc(const GemmArgs& a, const GemmWorkspace& ws, int* err, cudaStream_t s,
                    int force_splits = 0, int force_swap = -1);
size_t gemm_tc_workspace_bytes(int M, int N, int K, int force_splits = 0, int force_swap = -1);
// True when launch_gemm_tc takes GemmArgs with norm_x set for this shape.
bool gemm_tc_fuses_norm(int M, int N, int K);
// Split RMSNorm (Epilogue::xs_out / ssq_in): the number of ssq slots the
// producer GEMM of this shape writes (its CTAs per token tile), or 0 if the
// shape does not run on a kernel that produces them; and whether the
// consumer of this shape applies ssq_in.
int gemm_tc_ssq_slots(int M, int N, int K);
bool gemm_tc_takes_ssq(int M, int N, int K);
// Column tiles of the tcgen05 plan for an EPI_ARGMAX GEMM (0: not supported).
int gemm_tc_argmax_tiles(int M, int N, int K);
void launch_splitk_reduce(int dt, const float* part, int splits, int M, int N, const Epilogue& ep,
                          cudaStream_t s);

// ---- attention ------------------------------------------------------------
// Decode attention (q_len <= 4).  `part` is fp32 scratch for the partials of
// (group, head) pairs whose keys are split across CTAs;
// attn_decode_workspace_bytes gives its size (0 when nothing is split).
size_t attn_decode_workspace_bytes(int dt, const AttnArgs& a);
// Returns false (nothing launched) for unsupported shapes or too little scratch.
bool launch_attn_decode(int dt, const AttnArgs& a, float* part, size_t part_bytes, int* err,
                        cudaStream_t s);
// Causal attention for many new queries per group (prefill).
void launch_attn_prefill(int dt, const AttnArgs& a, int* err, cudaStream_t s);
// Attention with a shared prefix as two passes (bf16, dh = 64): all query
// rows against the prefix rows, then each group's own causal keys merged
// with that partial.  part holds attn_prefix_split_bytes(a).  Returns false
// (nothing launched) when the shape or the scratch does not fit.
size_t attn_prefix_split_bytes(const AttnArgs& a);
bool launch_attn_prefix_split(int dt, const AttnArgs& a, float* part, size_t part_bytes, int* err,
                              cudaStream_t s);
// The CUDA-core prefill kernel (any storage type, head size 32 or 64).
bool launch_attn_prefill_simt(int dt, const AttnArgs& a, cudaStream_t s);
// Prefill attention on a chosen kernel (0 the library's choice, 1 CUDA
// cores, 2 mma.sync, 3 tcgen05); with a prefix (n_pre > 0) paths 2 and 3
// take the two-pass split and need attn_prefix_split_bytes(a) of part.
// Returns false (possibly after launching a first pass) when the path does
// not take the shape.
bool launch_attn_prefill_path(int dt, const AttnArgs& a, int path, float* part, size_t part_bytes, int* err,
                              cudaStream_t s);

// ---- error message of the calling thread (read by photon_last_error) ----
void set_error_message(const char* msg);

// ---- launch accounting ------------------------------------------------------
// Process-wide count of kernels this library has launched.
void note_launch(long long n = 1);
unsigned long long launch_total();

// ---- TMA descriptors -----------------------------------------------------
bool tma_available();
// 2-D bf16 tensor map over a row-major [rows, K] matrix (leading dimension ld
// elements): box 64 (K) x box_rows, 128-byte swizzle, zero fill.
bool tma_map_bf16(CUtensorMap* m, const void* ptr, long long rows, int K, long long ld, int box_rows);
bool tma_map_bf16_3d(CUtensorMap* m, const void* ptr, long long d0, long long d1, long long d2,
                     long long stride1, long long stride2, int box0, int box1);
// Tensor-core (tcgen05) prefill attention, k_attn_prefill_tc.cu: bf16, head
// size 64, at least 128 query rows; false when the shape is not supported.
// ALL: own keys only (no prefix).  PREFIX: every query row against the
// shared prefix, fp32 partials into part; OWN: own keys merged with them.
bool launch_attn_prefill_tc(const AttnArgs& a, int* err, cudaStream_t s);
bool launch_attn_prefix_tc(const AttnArgs& a, float* part, int* err, cudaStream_t s);
bool launch_attn_own_tc(const AttnArgs& a, float* part, int* err, cudaStream_t s);

}  // namespace photon
