// Host runtime of the PHOTON library: model weights and their residency,
// KV caches and workspaces, and the launch sequences of prefill, HierGen and
// RecGen.  Implements the C ABI declared in include/photon.h.
//
// Procedure sources (PHOTON pages): module table of the explainer's
// architecture section (Chunker, Encoder, Converter, Decoder), the RecGen
// section (HierGen's three stages, RecGen's direct A-hat feed, top-only cache
// retention, decoder-only weight residency) and the 475x section (decoder
// attention confined to the chunk).
#include <cmath>
#include <cstdarg>
#include <cstdlib>
#include <cstdio>
#include <cstring>
#include <atomic>
#include <mutex>
#include <string>
#include <vector>

#include "kernels.h"
#include "photon.h"

using namespace photon;

// ============================================================== errors
static thread_local std::string g_err;

static int fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_err = buf;
  return code;
}

namespace photon {
void set_error_message(const char* msg) { g_err = msg; }
}  // namespace photon

#define CK(call)                                                                   \
  do {                                                                             \
    cudaError_t e_ = (call);                                                       \
    if (e_ != cudaSuccess) {                                                       \
      if (e_ == cudaErrorMemoryAllocation) {                                       \
        cudaGetLastError();                                                        \
        return fail(PHOTON_ERR_OOM, "%s: out of device memory", #call);            \
      }                                                                            \
      return fail(PHOTON_ERR_CUDA, "%s: %s", #call, cudaGetErrorString(e_));       \
    }                                                                              \
  } while (0)

#define RET(x)                     \
  do {                             \
    int r_ = (x);                  \
    if (r_ != PHOTON_OK) return r_; \
  } while (0)

// ============================================================== model
enum Group { G_EMB = 0, G_ENC1 = 1, G_TOP = 2, G_DEC = 3, G_COUNT = 4 };

struct TensorRec {
  std::string name;
  int group;
  size_t offset;  // bytes inside the group buffer
  long long numel;
  bool gain;      // RMSNorm gain: fp32, value 1
};

struct BlockW {
  const float* g_attn;
  const void* wqkv;  // [3d, d]: wq, wk, wv stored back to back
  const void* wo;
  const float* g_mlp;
  const void* w1;
  const void* w2;
};

struct photon_model {
  photon_config cfg;
  int dt;
  size_t es;
  uint64_t seed;
  int d, H, dh, V, C1, C2, C, f, L1, Ltop, Ld1, Ld2;
  // same-kernel baseline: a vanilla token-level Transformer (embed, L_van
  // blocks from i_van, final gain i_van_g, head i_head) instead of PHOTON
  bool vanilla = false;
  int i_van = 0, L_van = 0, i_van_g = 0;
  bool graph_failed_van = false;  // the vanilla step could not be captured
  // RoPE tables (cos, sin per position and frequency), made once per model and
  // grown when a cache needs more positions; caches point at the latest one,
  // so every table stays until the model is freed
  std::vector<float2*> rope_tables;
  int rope_positions = 0;
  // paged top KV (photon_model_set_kv_pages): page arrays
  // [Ltop][K, V][kv_pool_pages][H][kv_page_rows][dh]; a page id names the
  // same slot in every array, so one table entry maps a run of positions of
  // one sequence in every layer.  Pages released by a cache become reusable
  // once the work queued before the release has finished (its event).
  int kv_page_rows = 0, kv_pool_pages = 0, kv_paged_caches = 0;
  char* kv_pool = nullptr;
  std::vector<int> kv_free;
  std::vector<std::pair<cudaEvent_t, std::vector<int>>> kv_pending;
  std::vector<TensorRec> t;
  size_t group_bytes[G_COUNT] = {0, 0, 0, 0};
  char* group_ptr[G_COUNT] = {nullptr, nullptr, nullptr, nullptr};
  // first tensor index of each piece
  int i_embed, i_ch1, i_enc1, i_enc1_g, i_ch2, i_top, i_top_g, i_cv2, i_dec2, i_dec2_g, i_cv1,
      i_dec1, i_dec1_g, i_head;
  int live_caches = 0;
  int hier_caches = 0;
  bool use_tc = false;
  // Decode-step graph executables, one per mode, reused across caches: a new
  // cache's captured step updates the executable instead of instantiating.
  cudaGraphExec_t graph[2] = {nullptr, nullptr};
  const void* graph_owner[2] = {nullptr, nullptr};
  long long graph_kernels[2] = {0, 0};  // kernel launches captured in graph[mode]
  // pipelined RecGen graphs [main/token part][A-hat parity], reused across
  // caches through executable updates; pg_owner = the cache captured last
  cudaGraphExec_t pg[2][2] = {{nullptr, nullptr}, {nullptr, nullptr}};
  const void* pg_owner = nullptr;
  long long pg_kernels[2] = {0, 0};
  // one event per stream that has enqueued work reading the level-1 encoder
  // weights since they were generated; their release waits on all of them
  std::vector<std::pair<cudaStream_t, cudaEvent_t>> enc_users;
  int enc_policy = PHOTON_ENC_RESTORE;  // how released encoder weights come back
  void* enc_host = nullptr;             // their pinned host copy (PHOTON_ENC_RESTORE)
  uint64_t enc_restores = 0, enc_regenerations = 0;  // how often they came back, by which route

  // any-L models (photon_init_weights_levels): per level l (index l - 1)
  // chunk size, encoder and decoder depth, and first tensor of each piece
  bool general = false;
  int NL = 2;
  int Cl[PHOTON_MAX_LEVELS] = {}, El[PHOTON_MAX_LEVELS] = {}, Dl[PHOTON_MAX_LEVELS] = {};
  int i_chl[PHOTON_MAX_LEVELS] = {}, i_encl[PHOTON_MAX_LEVELS] = {}, i_encl_g[PHOTON_MAX_LEVELS] = {};
  int i_cvl[PHOTON_MAX_LEVELS] = {}, i_decl[PHOTON_MAX_LEVELS] = {}, i_decl_g[PHOTON_MAX_LEVELS] = {};
  cudaGraphExec_t ggraph[2] = {nullptr, nullptr};  // captured any-L decode step per mode
  const void* ggraph_owner[2] = {nullptr, nullptr};
  long long ggraph_kernels[2] = {0, 0};

  const void* ptr(int idx) const { return group_ptr[t[idx].group] + t[idx].offset; }
  BlockW block(int first, int l) const {
    const int b = first + 8 * l;
    return BlockW{(const float*)ptr(b), ptr(b + 1), ptr(b + 4), (const float*)ptr(b + 5),
                  ptr(b + 6), ptr(b + 7)};
  }
};

// any-L models (defined with their prefill and decode further down)
static int gen_check(const photon_level_config* c);
static void build_specs_levels(photon_model* m);
struct GenCache;
static int gen_prefill(photon_model* m, const int32_t* d_tokens, int B, int T, int mode, int max_new,
                       cudaStream_t s, photon_cache** out);
static int gen_decode_step(photon_model* m, photon_cache* c, int mode, int32_t* d_out_tokens, float* d_out_logits,
                           const int32_t* d_force_tokens, const void* d_force_a, cudaStream_t s);

static int check_config(const photon_config* c) {
  if (!c) return fail(PHOTON_ERR_ARG, "config is NULL");
  if (c->levels != 2) return fail(PHOTON_ERR_ARG, "only L = 2 levels are supported");
  if (c->vocab <= 0 || c->d_model <= 0 || c->n_heads <= 0 || c->head_dim <= 0)
    return fail(PHOTON_ERR_ARG, "non-positive model dimension");
  if (c->d_model != c->n_heads * c->head_dim)
    return fail(PHOTON_ERR_ARG, "d_model must equal n_heads * head_dim");
  if (c->head_dim != 32 && c->head_dim != 64) return fail(PHOTON_ERR_ARG, "head_dim must be 32 or 64");
  if (c->d_model % 64) return fail(PHOTON_ERR_ARG, "d_model must be a multiple of 64");
  for (int l = 0; l < 2; ++l) {
    if (c->chunk[l] < 1 || c->chunk[l] > 4) return fail(PHOTON_ERR_ARG, "chunk sizes must be 1..4");
    if (c->enc_layers[l] < 1 || c->dec_layers[l] < 1) return fail(PHOTON_ERR_ARG, "layer counts must be >= 1");
  }
  if (c->conv_kernel != 0 && (c->conv_kernel != c->chunk[0] || c->conv_kernel != c->chunk[1]))
    return fail(PHOTON_ERR_ARG, "conv_kernel must equal C1 and C2 (kernel = stride = C)");
  if (c->mlp_mult < 1) return fail(PHOTON_ERR_ARG, "mlp_mult must be >= 1");
  if (c->dtype != 0 && c->dtype != 1) return fail(PHOTON_ERR_ARG, "dtype must be 0 (fp32) or 1 (bf16)");
  if (!(c->norm_eps > 0.f) || !(c->rope_theta > 0.f) || !(c->init_std > 0.f))
    return fail(PHOTON_ERR_ARG, "eps, theta and init_std must be positive");
  return PHOTON_OK;
}

static void build_specs(photon_model* m) {
  const long long d = m->d, V = m->V, f = m->f;
  auto add = [&](const std::string& n, int g, long long numel, bool gain) {
    m->t.push_back(TensorRec{n, g, 0, numel, gain});
  };
  auto blocks = [&](const char* p, int n, int g) {
    for (int l = 0; l < n; ++l) {
      const std::string s = std::string(p) + "." + std::to_string(l) + ".";
      add(s + "g_attn", g, d, true);
      add(s + "wq", g, d * d, false);
      add(s + "wk", g, d * d, false);
      add(s + "wv", g, d * d, false);
      add(s + "wo", g, d * d, false);
      add(s + "g_mlp", g, d, true);
      add(s + "w1", g, f * d, false);
      add(s + "w2", g, d * f, false);
    }
  };
  m->i_embed = (int)m->t.size();
  add("embed", G_EMB, V * d, false);
  m->i_ch1 = (int)m->t.size();
  add("chunker1", G_ENC1, d * m->C1 * d, false);
  m->i_enc1 = (int)m->t.size();
  blocks("enc1", m->L1, G_ENC1);
  m->i_enc1_g = (int)m->t.size();
  add("enc1.g_final", G_ENC1, d, true);
  m->i_ch2 = (int)m->t.size();
  add("chunker2", G_TOP, d * m->C2 * d, false);
  m->i_top = (int)m->t.size();
  blocks("top", m->Ltop, G_TOP);
  m->i_top_g = (int)m->t.size();
  add("top.g_final", G_TOP, d, true);
  m->i_cv2 = (int)m->t.size();
  add("converter2", G_DEC, m->C2 * d * d, false);
  m->i_dec2 = (int)m->t.size();
  blocks("dec2", m->Ld2, G_DEC);
  m->i_dec2_g = (int)m->t.size();
  add("dec2.g_final", G_DEC, d, true);
  m->i_cv1 = (int)m->t.size();
  add("converter1", G_DEC, m->C1 * d * d, false);
  m->i_dec1 = (int)m->t.size();
  blocks("dec1", m->Ld1, G_DEC);
  m->i_dec1_g = (int)m->t.size();
  add("dec1.g_final", G_DEC, d, true);
  m->i_head = (int)m->t.size();
  add("head", G_DEC, V * d, false);
  for (auto& r : m->t) {
    const size_t bytes = (size_t)r.numel * (r.gain ? 4 : m->es);
    r.offset = m->group_bytes[r.group];
    m->group_bytes[r.group] += (bytes + 255) & ~size_t(255);
  }
}

// Stream-ordered pool owned by the library, one per device.  Its release
// threshold is unbounded: memory that a freed cache returns stays mapped and
// is handed to the next cache, instead of being unmapped at the next
// synchronisation and mapped again by the next prefill.  photon_free_model
// trims it back to nothing.
static std::mutex g_pool_mu;
static cudaMemPool_t g_pool[64];

static cudaError_t library_pool(cudaMemPool_t* out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(g_pool_mu);
  if (!g_pool[dev]) {
    cudaMemPoolProps p;
    memset(&p, 0, sizeof(p));
    p.allocType = cudaMemAllocationTypePinned;
    p.handleTypes = cudaMemHandleTypeNone;
    p.location.type = cudaMemLocationTypeDevice;
    p.location.id = dev;
    cudaMemPool_t pool = nullptr;
    e = cudaMemPoolCreate(&pool, &p);
    if (e != cudaSuccess) return e;
    uint64_t keep = ~0ull;
    e = cudaMemPoolSetAttribute(pool, cudaMemPoolAttrReleaseThreshold, &keep);
    if (e != cudaSuccess) {
      cudaMemPoolDestroy(pool);
      return e;
    }
    g_pool[dev] = pool;
  }
  *out = g_pool[dev];
  return cudaSuccess;
}

// Test hook (photon_debug_fail_alloc): the n-th device allocation from now
// on fails as if the device were out of memory; 0 = off.
static std::atomic<long long> g_fail_alloc{0};
static bool injected_alloc_failure() {
  long long v = g_fail_alloc.load();
  while (v > 0) {
    if (g_fail_alloc.compare_exchange_weak(v, v - 1)) return v == 1;
  }
  return false;
}

static cudaError_t pool_malloc(void** p, size_t bytes, cudaStream_t s) {
  if (injected_alloc_failure()) {
    *p = nullptr;
    return cudaErrorMemoryAllocation;
  }
  cudaMemPool_t pool = nullptr;
  cudaError_t e = library_pool(&pool);
  if (e != cudaSuccess) return e;
  return cudaMallocFromPoolAsync(p, bytes, pool, s);
}

// Draws (or fills) every tensor of one group into its buffer.
static void generate_group(photon_model* m, int g, cudaStream_t s) {
  const double K = (double)m->cfg.init_std;  // sigma of the normal draw (fp32 value)
  for (size_t i = 0; i < m->t.size(); ++i) {
    const TensorRec& r = m->t[i];
    if (r.group != g) continue;
    void* p = m->group_ptr[g] + r.offset;
    if (r.gain)
      launch_fill_f32((float*)p, r.numel, 1.0f, s);
    else
      launch_init_normal(m->dt, p, r.numel, m->seed, (int)i, K, s);
  }
}

// Level-1 encoder + chunker-1 weights are needed only by prefill and HierGen
// (RecGen section: during RecGen decode the encoder hierarchy is never
// called).  They are released after a RecGen prefill when no HierGen cache
// is alive, and regenerated from the seed when needed again.
// Residency of the level-1 encoder and Chunker_1 weights (explainer, RecGen
// section: during RecGen decoding only the decoders (and, by R15, the top
// encoder) need to stay on the device).  After a RecGen prefill they are
// released unless a HierGen cache needs them; the next prefill brings them
// back: by a host-to-device copy from a pinned host copy made at the first
// release (PHOTON_ENC_RESTORE, the default, what a trained model would do),
// by drawing them again from the seed (PHOTON_ENC_REGENERATE), or they are
// never released (PHOTON_ENC_KEEP).
static int ensure_encoder(photon_model* m, cudaStream_t s) {
  if (m->group_ptr[G_ENC1]) return PHOTON_OK;
  CK(pool_malloc((void**)&m->group_ptr[G_ENC1], m->group_bytes[G_ENC1], s));
  if (m->enc_policy == PHOTON_ENC_RESTORE && m->enc_host) {
    CK(cudaMemcpyAsync(m->group_ptr[G_ENC1], m->enc_host, m->group_bytes[G_ENC1], cudaMemcpyHostToDevice, s));
    ++m->enc_restores;
  } else {
    generate_group(m, G_ENC1, s);
    ++m->enc_regenerations;
  }
  CK(cudaGetLastError());
  return PHOTON_OK;
}
// Marks the end of the work just enqueued on `s` that reads the encoder.
static int note_encoder_use(photon_model* m, cudaStream_t s) {
  for (auto& u : m->enc_users)
    if (u.first == s) {
      CK(cudaEventRecord(u.second, s));
      return PHOTON_OK;
    }
  cudaEvent_t e = nullptr;
  CK(cudaEventCreateWithFlags(&e, cudaEventDisableTiming));
  m->enc_users.emplace_back(s, e);
  CK(cudaEventRecord(e, s));
  return PHOTON_OK;
}
// Stream-ordered release on `s`, after every user stream's last recorded use.
static int release_encoder(photon_model* m, cudaStream_t s) {
  if (!m->group_ptr[G_ENC1] || m->enc_policy == PHOTON_ENC_KEEP) return PHOTON_OK;
  if (m->enc_policy == PHOTON_ENC_RESTORE && !m->enc_host) {
    // the pinned host copy, made once (the weights never change)
    if (cudaMallocHost(&m->enc_host, m->group_bytes[G_ENC1]) != cudaSuccess) {
      cudaGetLastError();
      m->enc_host = nullptr;
      return fail(PHOTON_ERR_OOM, "pinned host memory for the encoder weights");
    }
    CK(cudaMemcpyAsync(m->enc_host, m->group_ptr[G_ENC1], m->group_bytes[G_ENC1], cudaMemcpyDeviceToHost, s));
    CK(cudaStreamSynchronize(s));
  }
  for (auto& u : m->enc_users) {
    CK(cudaStreamWaitEvent(s, u.second, 0));
    cudaEventDestroy(u.second);
  }
  m->enc_users.clear();
  CK(cudaFreeAsync(m->group_ptr[G_ENC1], s));
  m->group_ptr[G_ENC1] = nullptr;
  return PHOTON_OK;
}

// ============================================================== cache
constexpr int kSsqCap = 256;  // split-RMSNorm partial-sum slots per row (>= CTAs per token tile)
static int stream_priority_high() {
  int least = 0, greatest = 0;
  if (cudaDeviceGetStreamPriorityRange(&least, &greatest) != cudaSuccess) return 0;
  return greatest;
}
struct Bufs {
  void* xn;
  void* q;
  void* att;
  void* hid;
  const float2* rope;
  float* gemm_ws;
  size_t gemm_ws_bytes;
  int* gemm_cnt;  // split-K tile counters (zeroed; one array per concurrent stream)
  float* attn_ws;
  size_t attn_ws_bytes;
  int* err;
  void* sn_x = nullptr;    // split RMSNorm: bf16(x * g) for the next projection
  float* sn_ss = nullptr;  // ... and its per-row partial sums of squares
  int sn_cap = 0;          // floats per row in sn_ss
  float* pre_ws = nullptr;  // shared-prefix attention: the prefix pass's partials
  size_t pre_ws_bytes = 0;
};

struct photon_cache {
  photon_model* m = nullptr;
  const photon_cache* prefix = nullptr;
  mutable int dependents = 0;
  int B = 0, T = 0, mode = 0, max_new = 0;
  int N = 0, N1 = 0, n_pre = 0, n1_pre = 0;
  int Ncap = 0, N1cap = 0;
  int steps = 0;
  cudaStream_t stream = nullptr;
  char *top_k = nullptr, *top_v = nullptr;
  size_t top_layer = 0;
  // paged top KV: top_k / top_v are the model's layer-0 page arrays and
  // top_layer the stride between layers; kv_table [B][kv_tab_len] maps a
  // sequence's runs of kv_page_rows positions to pages (host mirror beside)
  bool paged = false;
  int* kv_table = nullptr;
  std::vector<int> kv_table_host;
  int kv_tab_len = 0, kv_mapped = 0;  // table length; runs mapped per sequence so far
  std::vector<int> kv_held;
  char *l1_k = nullptr, *l1_v = nullptr;
  size_t l1_layer = 0;
  void* o = nullptr;
  float2* rope = nullptr;
  // decode workspace
  float *xd = nullptr, *xs = nullptr, *xt = nullptr, *x1 = nullptr, *logits = nullptr;
  void *xn = nullptr, *q = nullptr, *att = nullptr, *hid = nullptr;
  void *a_hat = nullptr, *a = nullptr, *embd = nullptr, *hn = nullptr;
  char *d2k = nullptr, *d2v = nullptr, *d1k = nullptr, *d1v = nullptr;
  size_t d2_layer = 0, d1_layer = 0;
  int32_t *next_ids = nullptr, *used = nullptr;
  float* gemm_ws = nullptr;
  size_t gemm_ws_bytes = 0;
  int* gemm_cnt = nullptr;
  int* gemm_cnt_t = nullptr;
  void* sn_x = nullptr;              // split RMSNorm buffers (main chain / top branch)
  float* sn_ss = nullptr;
  void* sn_x_t = nullptr;
  float* sn_ss_t = nullptr;
  int sn_rows = 0;                   // rows sn_x / sn_ss hold (sn_x_t / sn_ss_t hold B)
  // pipelined RecGen (photon_decode_rec_chunks): the token branch of a chunk
  // overlaps the next chunk's main chain, so it gets its own buffers, A-hat
  // is double-buffered, and both halves are captured as separate graphs
  bool pipe_ready = false;
  void* ahat_p[2] = {nullptr, nullptr};
  const void* ahat_latest = nullptr;  // the A-hat of the last decode step
  float* xd_k = nullptr;
  void *xn_k = nullptr, *q_k = nullptr, *att_k = nullptr, *hid_k = nullptr, *sn_x_k = nullptr;
  float *gemm_ws_k = nullptr, *attn_ws_k = nullptr, *sn_ss_k = nullptr;
  int* gemm_cnt_k = nullptr;
  cudaStream_t tstream = nullptr;
  cudaEvent_t ev_main[2] = {nullptr, nullptr}, ev_tok[2] = {nullptr, nullptr};
  float* stk_part = nullptr;         // persistent token-step kernel: split partials
  int* stk_cnt = nullptr;            // ... its tile counters (zeroed)
  unsigned int* stk_bar = nullptr;   // ... its grid-barrier word
  int stk_cnt_len = 0;
  float* attn_ws = nullptr;
  size_t attn_ws_bytes = 0;
  float* pre_ws = nullptr;       // shared-prefix attention partials (caches built on a prefix)
  size_t pre_ws_bytes = 0;
  int* d_err = nullptr;
  int* d_pos = nullptr;          // device {N, N1, chunks generated, 0} read by the decode kernels
  float samp_inv_t = 0.f;        // token sampling: 1 / temperature (0: greedy)
  unsigned long long samp_seed = 0;
  float samp_top_p = 1.f;        // nucleus mass (1: the whole vocabulary)
  unsigned long long* amax_part = nullptr;  // [B*C2][amax_cap] head partials
  int amax_cap = 0;
  int32_t* tok_out = nullptr;    // [B, C] greedy tokens of the last graph-replayed step
  // persistent top-step kernel (k_top_step.cu): scratch shared by the top
  // chains of this cache (at most one runs at a time) and the launch plans,
  // one per (input rows, buffer set, mode)
  bool tk_ok = false;
  float* tk_part = nullptr;
  size_t tk_part_bytes = 0;
  int* tk_cnt = nullptr;
  unsigned* tk_bar = nullptr;
  struct TopPlanKey {
    const void* src;
    const void* xs;
    int mode;
    TopStepPlan* plan;
  };
  std::vector<TopPlanKey> tk_plans;
  // RecGen's top-encoder branch runs on its own stream with its own buffers
  cudaStream_t side = nullptr;
  cudaStream_t cap = nullptr;  // the decode step is captured here (any caller stream can replay it)
  cudaStream_t hi = nullptr;   // high-priority stream for the RecGen token branch
  cudaEvent_t ev_fork = nullptr, ev_join = nullptr, ev_join_hi = nullptr;
  void *xn_t = nullptr, *q_t = nullptr, *att_t = nullptr, *hid_t = nullptr;
  float* gemm_ws_t = nullptr;
  float* attn_ws_t = nullptr;
  bool graph_failed[2] = {false, false};
  int graph_steps = 0;
  std::vector<void*> allocs;
  size_t kv_bytes = 0, ws_bytes = 0;
  bool has_a_hat = false, has_a = false;
  struct GenCache* gen = nullptr;  // any-L models: their per-level state
  int32_t* gen_tok_out() const { return tok_out; }
};

struct Allocator {
  cudaStream_t s;
  std::vector<void*>* list;
  size_t* counter;
  cudaError_t err = cudaSuccess;
  template <typename P>
  P* get(size_t bytes) {
    if (bytes == 0 || err != cudaSuccess) return nullptr;
    void* p = nullptr;
    err = pool_malloc(&p, (bytes + 255) & ~size_t(255), s);
    if (err != cudaSuccess) return nullptr;
    list->push_back(p);
    if (counter) *counter += bytes;
    return reinterpret_cast<P*>(p);
  }
};

static void free_list(std::vector<void*>& l, cudaStream_t s) {
  for (void* p : l) cudaFreeAsync(p, s);
  l.clear();
}

// One stack invocation: group/position layout and the caches it writes/reads.
struct StackRun {
  int G = 0, q_len = 1, p0 = 0, kv_off = 0;
  char* kc = nullptr;
  char* vc = nullptr;
  size_t layer_bytes = 0;
  int cap = 0;
  const char* kp = nullptr;
  const char* vp = nullptr;
  size_t pre_layer_bytes = 0;
  int cap_pre = 0, n_pre = 0;
  const int* p0_dev = nullptr;  // device position of the first row (added to p0)
  int n_plan = 0;               // key count the decode attention is planned for
  // paged own KV: kc / vc are the page arrays of layer 0, layer_bytes the
  // stride between layers, and slot s of group g lives in page
  // kv_table[g * kv_tab_len + s / kv_page_rows]
  const int* kv_table = nullptr;
  int kv_tab_len = 0, kv_page_rows = 0, kv_pages = 0;
  bool xn_ready = false;        // the first block's attention norm is already in b.xn
  int sn_rows = 0;              // rows the split-RMSNorm buffers of the Bufs hold (0: none)
};

static void gemm(photon_model* m, const Bufs& b, const void* A, long long lda, const void* W,
                 long long ldw, int M, int N, int K, const Epilogue& ep, cudaStream_t s);

// Shared-prefix attention in two passes (PHOTON_PREFIX_SPLIT=0: one pass per
// (group, head) over prefix and own keys together).
static bool prefix_split_enabled() {
  static const bool on = [] {
    const char* e = getenv("PHOTON_PREFIX_SPLIT");
    return !(e && e[0] == '0');
  }();
  return on;
}

static bool split_norm_enabled() {
  static const bool on = [] {
    const char* e = getenv("PHOTON_SPLIT_NORM");
    return !(e && e[0] == '0');
  }();
  return on;
}

// Persistent top-step kernel for the top encoder's decode step
// (PHOTON_TOP_MEGA=1; otherwise one kernel per projection).
static bool top_mega_enabled() {
  static const bool on = [] {
    const char* e = getenv("PHOTON_TOP_MEGA");
    return e && e[0] == '1';
  }();
  return on;
}

// Whether a block over `rows` rows can split its two RMSNorms across the
// neighbouring GEMMs (O and W2 produce, QKV and W1 consume); false keeps the
// norm kernels.
static bool split_norm_ok(const photon_model* m, const Bufs& b, int rows, int cap_rows) {
  if (!m->use_tc || !b.sn_x || !b.sn_ss || !split_norm_enabled() || rows > cap_rows) return false;
  const int d = m->d, f = m->f;
  const int so = gemm_tc_ssq_slots(rows, d, d), s2 = gemm_tc_ssq_slots(rows, d, f);
  return so > 0 && so <= b.sn_cap && s2 > 0 && s2 <= b.sn_cap && gemm_tc_takes_ssq(rows, 3 * d, d) &&
         gemm_tc_takes_ssq(rows, f, d);
}

static void gemm(photon_model* m, const Bufs& b, const void* A, long long lda, const void* W,
                 long long ldw, int M, int N, int K, const Epilogue& ep, cudaStream_t s) {
  GemmArgs g;
  g.A = A;
  g.lda = lda;
  g.W = W;
  g.ldw = ldw;
  g.M = M;
  g.N = N;
  g.K = K;
  g.ep = ep;
  GemmWorkspace ws{b.gemm_ws, b.gemm_ws_bytes, b.gemm_cnt, b.gemm_cnt ? kGemmTileCounters : 0};
  if (ep.ssq_in != nullptr || ep.xs_out != nullptr) {
    // split-RMSNorm roles exist only on the tcgen05 paths the planner chose;
    // a refusal here is a planning bug: flag it on the device error word
    if (!launch_gemm_tc(g, ws, b.err, s)) cudaMemsetAsync(b.err, 0x7f, sizeof(int), s);
    return;
  }
  if (m->use_tc)
    launch_gemm(m->dt, g, ws, b.err, s);
  else
    launch_gemm_simt(m->dt, g, s);
}

// GEMM of a pre-norm projection: RMSNorm(x; g) * W^T.  The norm runs first
// into b.xn; with PHOTON_FUSE_NORM=1 the few-token tcgen05 kernel
// normalises its own operand instead.
// Off by default: every weight-tile cluster of a wide projection would
// normalise the same rows again (fp32 reads, twice), which measured slower
// than one norm kernel writing a bf16 copy that the GEMM reads with TMA.
static bool fuse_norm_enabled() {
  static const bool on = [] {
    const char* e = getenv("PHOTON_FUSE_NORM");
    return e && e[0] == '1';
  }();
  return on;
}

static void gemm_normed(photon_model* m, const Bufs& b, const float* x, const float* g,
                        const void* W, long long ldw, int M, int N, int K, const Epilogue& ep,
                        cudaStream_t s, bool xn_ready = false) {
  if (xn_ready) {  // a fused row kernel already wrote RMSNorm(x) into b.xn
    gemm(m, b, b.xn, K, W, ldw, M, N, K, ep, s);
    return;
  }
  if (m->use_tc && fuse_norm_enabled() && gemm_tc_fuses_norm(M, N, K)) {
    GemmArgs a;
    a.W = W;
    a.ldw = ldw;
    a.M = M;
    a.N = N;
    a.K = K;
    a.ep = ep;
    a.norm_x = x;
    a.norm_ld = K;
    a.norm_g = g;
    a.norm_eps = m->cfg.norm_eps;
    GemmWorkspace ws{b.gemm_ws, b.gemm_ws_bytes, b.gemm_cnt, b.gemm_cnt ? kGemmTileCounters : 0};
    if (launch_gemm_tc(a, ws, b.err, s)) return;
  }
  launch_rmsnorm(m->dt, x, g, b.xn, M, K, 1, 0, m->cfg.norm_eps, s);
  gemm(m, b, b.xn, K, W, ldw, M, N, K, ep, s);
}

static Epilogue epi(int kind, void* out, long long ldo) {
  Epilogue e;
  e.kind = kind;
  e.out = out;
  e.ldo = ldo;
  return e;
}

// Pre-norm block (reading R8-R11): x += Attn(RMSNorm(x)); x += MLP(RMSNorm(x)).
// One pre-norm block.  sn_slots: on entry, > 0 when the previous block's W2
// already produced bf16(x * g_attn) and its row sums of squares (split
// RMSNorm, slots of that GEMM); on return, the same for the next block
// (g_next = its attention gain, null for the last block of the stack).
static void run_block(photon_model* m, const BlockW& w, float* x, const StackRun& r, int layer,
                      const Bufs& b, cudaStream_t s, int& sn_slots, const float* g_next) {
  const int d = m->d, rows = r.G * r.q_len;
  const float eps = m->cfg.norm_eps;
  const bool sn = split_norm_ok(m, b, rows, r.sn_rows);
  Epilogue e;
  e.kind = EPI_QKV;
  e.q_out = b.q;
  e.k_cache = r.kc + layer * r.layer_bytes;
  e.v_cache = r.vc + layer * r.layer_bytes;
  e.d = d;
  e.H = m->H;
  e.dh = m->dh;
  e.cap = r.cap;
  e.q_len = r.q_len;
  e.p0 = r.p0;
  e.kv_off = r.kv_off;
  e.rope = b.rope;
  e.p0_dev = r.p0_dev;
  e.kv_table = r.kv_table;
  e.kv_tab_len = r.kv_tab_len;
  e.kv_page_rows = r.kv_page_rows;
  e.kv_pages = r.kv_pages;
  if (sn && sn_slots > 0) {
    e.ssq_in = b.sn_ss;
    e.ssq_slots = sn_slots;
    e.norm_d = d;
    e.norm_eps = eps;
    gemm(m, b, b.sn_x, d, w.wqkv, d, rows, 3 * d, d, e, s);
  } else {
    gemm_normed(m, b, x, w.g_attn, w.wqkv, d, rows, 3 * d, d, e, s, r.xn_ready && layer == 0);
  }

  AttnArgs a;
  a.Q = b.q;
  a.q_ld = d;
  a.K = e.k_cache;
  a.V = e.v_cache;
  a.cap = r.cap;
  if (r.kp) {
    a.Kp = r.kp + layer * r.pre_layer_bytes;
    a.Vp = r.vp + layer * r.pre_layer_bytes;
    a.cap_pre = r.cap_pre;
    a.n_pre = r.n_pre;
  }
  a.G = r.G;
  a.H = m->H;
  a.dh = m->dh;
  a.q_len = r.q_len;
  a.p0 = r.p0;
  a.O = b.att;
  a.o_ld = d;
  a.scale = 1.0f / sqrtf((float)m->dh);
  a.p0_dev = r.p0_dev;
  a.n_plan = r.n_plan;
  a.kv_table = r.kv_table;
  a.kv_tab_len = r.kv_tab_len;
  a.kv_page_rows = r.kv_page_rows;
  a.kv_pages = r.kv_pages;
  bool done = false;
  // with a shared prefix: the prefix once for all queries, then each group's own keys
  if (r.kp && b.pre_ws && prefix_split_enabled())
    done = launch_attn_prefix_split(m->dt, a, b.pre_ws, b.pre_ws_bytes, b.err, s);
  if (!done && r.q_len <= 4) done = launch_attn_decode(m->dt, a, b.attn_ws, b.attn_ws_bytes, b.err, s);
  if (!done) launch_attn_prefill(m->dt, a, b.err, s);

  Epilogue eo = epi(EPI_ADD_F32, x, d);
  int slots_o = 0;
  if (sn) {  // O projection also produces the MLP norm's operand
    slots_o = gemm_tc_ssq_slots(rows, d, d);
    eo.xs_out = b.sn_x;
    eo.g_next = w.g_mlp;
    eo.ssq_out = b.sn_ss;
    eo.ssq_slots = slots_o;
  }
  gemm(m, b, b.att, d, w.wo, d, rows, d, d, eo, s);
  if (sn) {
    Epilogue e1 = epi(EPI_GELU_T, b.hid, m->f);
    e1.ssq_in = b.sn_ss;
    e1.ssq_slots = slots_o;
    e1.norm_d = d;
    e1.norm_eps = eps;
    gemm(m, b, b.sn_x, d, w.w1, d, rows, m->f, d, e1, s);
  } else {
    gemm_normed(m, b, x, w.g_mlp, w.w1, d, rows, m->f, d, epi(EPI_GELU_T, b.hid, m->f), s);
  }
  Epilogue e2 = epi(EPI_ADD_F32, x, d);
  sn_slots = 0;
  if (sn && g_next) {  // W2 also produces the next block's attention-norm operand
    const int sl = gemm_tc_ssq_slots(rows, d, m->f);
    e2.xs_out = b.sn_x;
    e2.g_next = g_next;
    e2.ssq_out = b.sn_ss;
    e2.ssq_slots = sl;
    sn_slots = sl;
  }
  gemm(m, b, b.hid, m->f, w.w2, m->f, rows, d, m->f, e2, s);
}

static void run_stack(photon_model* m, int first, int n_layers, float* x, const StackRun& r,
                      const Bufs& b, cudaStream_t s) {
  int sn_slots = 0;
  for (int l = 0; l < n_layers; ++l)
    run_block(m, m->block(first, l), x, r, l, b, s, sn_slots,
              l + 1 < n_layers ? m->block(first, l + 1).g_attn : nullptr);
}

static size_t gemm_ws_need(const photon_model* m, int M, int N, int K) {
  if (!m->use_tc) return 0;
  return gemm_tc_workspace_bytes(M, N, K);
}
static size_t block_ws_need(const photon_model* m, int rows) {
  size_t w = 0;
  w = std::max(w, gemm_ws_need(m, rows, 3 * m->d, m->d));
  w = std::max(w, gemm_ws_need(m, rows, m->d, m->d));
  w = std::max(w, gemm_ws_need(m, rows, m->f, m->d));
  w = std::max(w, gemm_ws_need(m, rows, m->d, m->f));
  return w;
}
// Scratch of a decode-attention launch planned for n_plan keys per pair.
static size_t attn_ws_need(int dt, int G, int H, int dh, int q_len, int n_plan) {
  AttnArgs a;
  a.G = G;
  a.H = H;
  a.dh = dh;
  a.q_len = q_len;
  a.p0 = n_plan - q_len;
  a.n_plan = n_plan;
  return attn_decode_workspace_bytes(dt, a);
}

// cos/sin table: entry [pos][i] = (cos, sin)(pos * theta^(-2i/dh)), computed in fp64.
// The model's RoPE table for at least `positions` positions: (cos, sin) of
// p * theta^(-2i/dh), evaluated in fp64 on the host and rounded to fp32.  It
// is computed when a cache first needs more positions than the model's table
// has (then for twice as many, so growth is rare), not once per prefill.
static int upload_rope(photon_model* m, float2** out, int positions) {
  if (positions > m->rope_positions) {
    const int n = std::max(positions, 2 * m->rope_positions);
    const int half = m->dh / 2;
    std::vector<float2> host((size_t)n * half);
    for (int p = 0; p < n; ++p)
      for (int i = 0; i < half; ++i) {
        const double inv = std::pow((double)m->cfg.rope_theta, -2.0 * i / m->dh);
        const double ang = (double)p * inv;
        host[(size_t)p * half + i] = make_float2((float)std::cos(ang), (float)std::sin(ang));
      }
    float2* d = nullptr;
    const size_t bytes = host.size() * sizeof(float2);
    if (injected_alloc_failure() || cudaMalloc((void**)&d, bytes) != cudaSuccess) {
      cudaGetLastError();
      return PHOTON_ERR_OOM;
    }
    if (cudaMemcpy(d, host.data(), bytes, cudaMemcpyHostToDevice) != cudaSuccess) {
      cudaGetLastError();
      cudaFree(d);
      return fail(PHOTON_ERR_CUDA, "RoPE table upload failed");
    }
    m->rope_tables.push_back(d);
    m->rope_positions = n;
  }
  *out = m->rope_tables.back();
  return PHOTON_OK;
}

static Bufs decode_bufs(photon_cache* c) {
  Bufs b;
  b.xn = c->xn;
  b.q = c->q;
  b.att = c->att;
  b.hid = c->hid;
  b.rope = c->rope;
  b.gemm_ws = c->gemm_ws;
  b.gemm_ws_bytes = c->gemm_ws_bytes;
  b.gemm_cnt = c->gemm_cnt;
  b.attn_ws = c->attn_ws;
  b.attn_ws_bytes = c->attn_ws_bytes;
  b.err = c->d_err;
  b.sn_x = c->sn_x;
  b.sn_ss = c->sn_ss;
  b.sn_cap = c->sn_x ? kSsqCap : 0;
  b.pre_ws = c->pre_ws;
  b.pre_ws_bytes = c->pre_ws_bytes;
  return b;
}

// Allocates the model's weight groups and draws every tensor (synchronising);
// on failure releases them and the model.
static int alloc_and_generate(photon_model* m) {
  cudaStream_t s = nullptr;
  for (int g = 0; g < G_COUNT; ++g) {
    if (m->group_bytes[g] == 0) continue;
    cudaError_t e = injected_alloc_failure() ? cudaErrorMemoryAllocation
                                             : cudaMalloc((void**)&m->group_ptr[g], m->group_bytes[g]);
    if (e != cudaSuccess) {
      cudaGetLastError();
      for (int k = 0; k < g; ++k) cudaFree(m->group_ptr[k]);
      delete m;
      return e == cudaErrorMemoryAllocation ? fail(PHOTON_ERR_OOM, "out of device memory for the weights")
                                            : fail(PHOTON_ERR_CUDA, "weight allocation: %s", cudaGetErrorString(e));
    }
    generate_group(m, g, s);
  }
  cudaError_t e = cudaStreamSynchronize(s);
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e != cudaSuccess) {
    for (int g = 0; g < G_COUNT; ++g) cudaFree(m->group_ptr[g]);
    delete m;
    return fail(PHOTON_ERR_CUDA, "weight generation failed: %s", cudaGetErrorString(e));
  }
  return PHOTON_OK;
}

// ============================================================== C ABI
extern "C" {

const char* photon_last_error(void) { return g_err.c_str(); }

int photon_debug_fail_alloc(int64_t n) {
  g_err.clear();
  if (n < 0) return fail(PHOTON_ERR_ARG, "n must be >= 0");
  g_fail_alloc.store(n);
  return PHOTON_OK;
}

int photon_selftest_wait_timeout(int64_t limit_cycles, int32_t* d_err, void* stream) {
  g_err.clear();
  if (!d_err || limit_cycles < 0) return fail(PHOTON_ERR_ARG, "bad arguments");
  cudaStream_t s = (cudaStream_t)stream;
  CK(cudaMemsetAsync(d_err, 0, sizeof(int32_t), s));
  launch_wait_selftest((long long)limit_cycles, d_err, s);
  CK(cudaGetLastError());
  int32_t h = 0;
  CK(cudaMemcpyAsync(&h, d_err, sizeof(int32_t), cudaMemcpyDeviceToHost, s));
  CK(cudaStreamSynchronize(s));
  if (h != 0) return fail(PHOTON_ERR_DEVICE_CHECK, "device wait timed out (code %d)", h);
  return PHOTON_OK;
}

uint64_t photon_launch_count(void) { return (uint64_t)launch_total(); }

int photon_init_weights(const photon_config* cfg, uint64_t seed, photon_model** out) {
  g_err.clear();
  if (!out) return fail(PHOTON_ERR_ARG, "out is NULL");
  *out = nullptr;
  RET(check_config(cfg));
  int dev = 0;
  CK(cudaGetDevice(&dev));
  photon_model* m = new photon_model();
  m->cfg = *cfg;
  m->dt = cfg->dtype;
  m->es = dtype_size(m->dt);
  m->seed = seed;
  m->d = cfg->d_model;
  m->H = cfg->n_heads;
  m->dh = cfg->head_dim;
  m->V = cfg->vocab;
  m->C1 = cfg->chunk[0];
  m->C2 = cfg->chunk[1];
  m->C = m->C1 * m->C2;
  m->f = cfg->mlp_mult * cfg->d_model;
  m->L1 = cfg->enc_layers[0];
  m->Ltop = cfg->enc_layers[1];
  m->Ld1 = cfg->dec_layers[0];
  m->Ld2 = cfg->dec_layers[1];
  m->use_tc = (m->dt == DT_BF16) && tma_available();
  build_specs(m);
  RET(alloc_and_generate(m));
  *out = m;
  return PHOTON_OK;
}

int photon_init_weights_levels(const photon_level_config* cfg, uint64_t seed, photon_model** out) {
  g_err.clear();
  if (!out) return fail(PHOTON_ERR_ARG, "out is NULL");
  *out = nullptr;
  RET(gen_check(cfg));
  int dev = 0;
  CK(cudaGetDevice(&dev));
  photon_model* m = new photon_model();
  // the two-level config fields describe the bottom and the top of the hierarchy
  memset(&m->cfg, 0, sizeof(m->cfg));
  m->cfg.vocab = cfg->vocab;
  m->cfg.d_model = cfg->d_model;
  m->cfg.n_heads = cfg->n_heads;
  m->cfg.head_dim = cfg->head_dim;
  m->cfg.levels = cfg->levels;
  m->cfg.mlp_mult = cfg->mlp_mult;
  m->cfg.dtype = cfg->dtype;
  m->cfg.init_std = cfg->init_std;
  m->cfg.rope_theta = cfg->rope_theta;
  m->cfg.norm_eps = cfg->norm_eps;
  m->general = true;
  m->NL = cfg->levels;
  m->dt = cfg->dtype;
  m->es = dtype_size(m->dt);
  m->seed = seed;
  m->d = cfg->d_model;
  m->H = cfg->n_heads;
  m->dh = cfg->head_dim;
  m->V = cfg->vocab;
  m->f = cfg->mlp_mult * cfg->d_model;
  m->C = 1;
  for (int l = 0; l < m->NL; ++l) {
    m->Cl[l] = cfg->chunk[l];
    m->El[l] = cfg->enc_layers[l];
    m->Dl[l] = cfg->dec_layers[l];
    m->C *= m->Cl[l];
  }
  const int L = m->NL;
  m->C1 = m->Cl[0];
  m->C2 = m->Cl[L - 1];
  m->L1 = m->El[0];
  m->Ltop = m->El[L - 1];
  m->Ld1 = m->Dl[0];
  m->Ld2 = m->Dl[L - 1];
  m->use_tc = (m->dt == DT_BF16) && tma_available();
  build_specs_levels(m);
  // the top-level pieces under their two-level names (export, info)
  m->i_top = m->i_encl[L - 1];
  m->i_top_g = m->i_encl_g[L - 1];
  m->i_ch2 = m->i_chl[L - 1];
  m->i_cv1 = m->i_cvl[0];
  m->i_dec1 = m->i_decl[0];
  m->i_dec1_g = m->i_decl_g[0];
  RET(alloc_and_generate(m));
  *out = m;
  return PHOTON_OK;
}

int photon_free_model(photon_model* m) {
  g_err.clear();
  if (!m) return fail(PHOTON_ERR_ARG, "model is NULL");
  if (m->live_caches) return fail(PHOTON_ERR_ARG, "%d caches still use this model", m->live_caches);
  CK(cudaDeviceSynchronize());
  for (auto& u : m->enc_users) cudaEventDestroy(u.second);
  m->enc_users.clear();
  for (int k = 0; k < 2; ++k) {
    if (m->graph[k]) cudaGraphExecDestroy(m->graph[k]);
    if (m->ggraph[k]) cudaGraphExecDestroy(m->ggraph[k]);
    for (int p = 0; p < 2; ++p)
      if (m->pg[k][p]) cudaGraphExecDestroy(m->pg[k][p]);
  }
  for (int g = 0; g < G_COUNT; ++g)
    if (m->group_ptr[g]) cudaFree(m->group_ptr[g]);
  for (float2* r : m->rope_tables) cudaFree(r);
  for (auto& p : m->kv_pending) cudaEventDestroy(p.first);
  if (m->kv_pool) cudaFree(m->kv_pool);
  if (m->enc_host) cudaFreeHost(m->enc_host);
  delete m;
  cudaMemPool_t pool = nullptr;
  if (library_pool(&pool) == cudaSuccess) cudaMemPoolTrimTo(pool, 0);
  return PHOTON_OK;
}

int photon_model_set_encoder_residency(photon_model* m, int32_t policy) {
  g_err.clear();
  if (!m) return fail(PHOTON_ERR_ARG, "model is NULL");
  if (policy != PHOTON_ENC_RESTORE && policy != PHOTON_ENC_REGENERATE && policy != PHOTON_ENC_KEEP)
    return fail(PHOTON_ERR_ARG, "unknown residency policy %d", policy);
  m->enc_policy = policy;
  return PHOTON_OK;
}

int photon_model_info(const photon_model* m, photon_model_stats* out) {
  g_err.clear();
  if (!m || !out) return fail(PHOTON_ERR_ARG, "NULL argument");
  memset(out, 0, sizeof(*out));
  for (const auto& r : m->t) out->param_count += (uint64_t)r.numel;
  for (int g = 0; g < G_COUNT; ++g) {
    uint64_t bytes = 0;
    for (const auto& r : m->t)
      if (r.group == g) bytes += (uint64_t)r.numel * (r.gain ? 4 : m->es);
    if (g == G_ENC1) out->encoder_bytes = bytes;
    if (m->group_ptr[g]) out->resident_bytes += bytes;
  }
  out->encoder_resident = m->group_ptr[G_ENC1] != nullptr;
  out->n_tensors = (int32_t)m->t.size();
  out->live_caches = m->live_caches;
  out->tcgen05_gemm = m->use_tc ? 1 : 0;
  out->encoder_restores = m->enc_restores;
  out->encoder_regenerations = m->enc_regenerations;
  out->kv_page_rows = m->kv_page_rows;
  out->kv_pool_pages = m->kv_pool_pages;
  size_t held_back = 0;
  for (const auto& p : m->kv_pending) held_back += p.second.size();
  out->kv_free_pages = (int32_t)(m->kv_free.size() + held_back);
  out->kv_paged_caches = m->kv_paged_caches;
  out->kv_pool_bytes =
      m->kv_pool ? (uint64_t)m->Ltop * 2 * m->kv_pool_pages * m->H * m->kv_page_rows * m->dh * m->es : 0;
  return PHOTON_OK;
}

int photon_export_weight(photon_model* m, int32_t index, void* d_dst, size_t dst_bytes,
                         size_t* out_bytes, void* stream) {
  g_err.clear();
  if (!m) return fail(PHOTON_ERR_ARG, "model is NULL");
  if (index < 0 || index >= (int)m->t.size()) return fail(PHOTON_ERR_ARG, "tensor index out of range");
  const TensorRec& r = m->t[index];
  const size_t bytes = (size_t)r.numel * (r.gain ? 4 : m->es);
  if (out_bytes) *out_bytes = bytes;
  if (!d_dst) return PHOTON_OK;
  if (dst_bytes < bytes) return fail(PHOTON_ERR_ARG, "destination holds %zu bytes, need %zu", dst_bytes, bytes);
  cudaStream_t s = (cudaStream_t)stream;
  if (r.group == G_ENC1) RET(ensure_encoder(m, s));
  CK(cudaMemcpyAsync(d_dst, m->ptr(index), bytes, cudaMemcpyDeviceToDevice, s));
  if (r.group == G_ENC1) RET(note_encoder_use(m, s));
  return PHOTON_OK;
}

// ============================================================== paged top KV
static size_t kv_page_bytes(const photon_model* m) {
  return (size_t)m->H * m->kv_page_rows * m->dh * m->es;
}

// n pages from the pool: released pages whose work has finished come back
// first; if that is not enough, the oldest release is waited for.  False
// when the pool cannot supply them.
static bool kv_take(photon_model* m, int n, std::vector<int>& out) {
  auto reclaim = [&](size_t i) {
    m->kv_free.insert(m->kv_free.end(), m->kv_pending[i].second.begin(), m->kv_pending[i].second.end());
    cudaEventDestroy(m->kv_pending[i].first);
    m->kv_pending.erase(m->kv_pending.begin() + (long)i);
  };
  for (size_t i = 0; i < m->kv_pending.size();) {
    if (cudaEventQuery(m->kv_pending[i].first) == cudaSuccess) {
      reclaim(i);
    } else {
      cudaGetLastError();
      ++i;
    }
  }
  while ((int)m->kv_free.size() < n && !m->kv_pending.empty()) {
    cudaEventSynchronize(m->kv_pending[0].first);
    cudaGetLastError();
    reclaim(0);
  }
  if ((int)m->kv_free.size() < n) return false;
  out.assign(m->kv_free.end() - n, m->kv_free.end());
  m->kv_free.resize(m->kv_free.size() - n);
  return true;
}

// Releases a paged cache's pages: reusable once the work queued on s so far
// has finished.
static void kv_release(photon_model* m, photon_cache* c, cudaStream_t s) {
  if (c->kv_held.empty()) return;
  cudaEvent_t e = nullptr;
  if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) == cudaSuccess && cudaEventRecord(e, s) == cudaSuccess) {
    m->kv_pending.emplace_back(e, std::move(c->kv_held));
  } else {  // cannot order the reuse after the pending work: wait for it
    cudaGetLastError();
    if (e) cudaEventDestroy(e);
    cudaStreamSynchronize(s);
    m->kv_free.insert(m->kv_free.end(), c->kv_held.begin(), c->kv_held.end());
  }
  c->kv_held.clear();
}

// Maps pages until own slot `slot` of every sequence has one (a new run of
// kv_page_rows positions per sequence at a time).  The new table entries
// reach the device on s, before the work that writes those slots; entries
// are written once and never change while the cache lives.
static int kv_map_through(photon_cache* c, int slot, cudaStream_t s) {
  photon_model* m = c->m;
  const int P = m->kv_page_rows;
  const int need = slot / P + 1;
  if (need <= c->kv_mapped) return PHOTON_OK;
  if (need > c->kv_tab_len) return fail(PHOTON_ERR_CAPACITY, "paged cache is full (%d positions)", c->kv_tab_len * P);
  const int add = need - c->kv_mapped;
  std::vector<int> pages;
  if (!kv_take(m, add * c->B, pages))
    return fail(PHOTON_ERR_CAPACITY, "the KV page pool (%d pages) has no %d free pages", m->kv_pool_pages,
                add * c->B);
  size_t k = 0;
  for (int lp = c->kv_mapped; lp < need; ++lp)
    for (int b = 0; b < c->B; ++b) c->kv_table_host[(size_t)b * c->kv_tab_len + lp] = pages[k++];
  c->kv_held.insert(c->kv_held.end(), pages.begin(), pages.end());
  // columns kv_mapped .. need-1 of every row (pageable source: staged before the call returns)
  const size_t pitch = (size_t)c->kv_tab_len * sizeof(int);
  CK(cudaMemcpy2DAsync(c->kv_table + c->kv_mapped, pitch, c->kv_table_host.data() + c->kv_mapped, pitch,
                       (size_t)add * sizeof(int), c->B, cudaMemcpyHostToDevice, s));
  c->kv_mapped = need;
  c->kv_bytes += (size_t)add * c->B * m->Ltop * 2 * kv_page_bytes(m);
  return PHOTON_OK;
}

static void set_paged(StackRun& r, const photon_cache* c) {
  if (!c->paged) return;
  r.kv_table = c->kv_table;
  r.kv_tab_len = c->kv_tab_len;
  r.kv_page_rows = c->m->kv_page_rows;
  r.kv_pages = c->m->kv_pool_pages;
}

// o_all (nullable): also the final-normed top output of every own position,
// [B * T/C, d] in the storage type (teacher-forced scoring reads them all).
// shell: allocate and set up the cache as a prefill of T tokens would, but
// compute nothing (its state is then filled by the caller, e.g. a broadcast
// of another rank's prefilled cache).
static int prefill_impl(photon_model* m, const photon_cache* prefix, const int32_t* d_tokens, int32_t B,
                        int32_t T, int32_t mode, int32_t max_new_chunks, void* stream, photon_cache** out,
                        void* o_all, bool shell = false, bool paged = false) {
  g_err.clear();
  if (!m || !out) return fail(PHOTON_ERR_ARG, "NULL model or out");
  *out = nullptr;
  if (m->vanilla) return fail(PHOTON_ERR_ARG, "a vanilla baseline model takes the photon_vanilla_* calls");
  if (!d_tokens && !shell) return fail(PHOTON_ERR_ARG, "tokens pointer is NULL");
  if (B <= 0) return fail(PHOTON_ERR_ARG, "batch must be positive");
  // the attention kernels index (sequence, sub-chunk) groups in a grid
  // dimension of at most 65535
  if ((long long)B * m->C2 > 65535)
    return fail(PHOTON_ERR_ARG, "batch %d too large: B * C2 must be at most 65535", B);
  if (T <= 0 || T % m->C) return fail(PHOTON_ERR_ARG, "T = %d is not a positive multiple of C1*C2 = %d", T, m->C);
  if (mode != PHOTON_MODE_HIER && mode != PHOTON_MODE_REC) return fail(PHOTON_ERR_ARG, "unknown mode %d", mode);
  if (max_new_chunks < 0) return fail(PHOTON_ERR_ARG, "max_new_chunks must be >= 0");
  if (prefix) {
    if (prefix->m != m) return fail(PHOTON_ERR_ARG, "prefix belongs to another model");
    if (prefix->mode != PHOTON_MODE_HIER || !prefix->l1_k)
      return fail(PHOTON_ERR_ARG, "prefix must be prefilled in HIER mode");
    if (prefix->B != 1) return fail(PHOTON_ERR_ARG, "prefix batch must be 1");
    if (prefix->prefix) return fail(PHOTON_ERR_ARG, "nested prefixes are not supported");
    if (prefix->paged) return fail(PHOTON_ERR_ARG, "a paged cache cannot be a shared prefix");
  }
  const long long rows0 = (long long)B * T;
  if (rows0 > (1ll << 31) / 4) return fail(PHOTON_ERR_ARG, "B*T too large");
  cudaStream_t s = (cudaStream_t)stream;
  const int d = m->d, C1 = m->C1, C2 = m->C2, C = m->C;

  photon_cache* c = new photon_cache();
  c->m = m;
  c->prefix = prefix;
  c->B = B;
  c->T = T;
  c->mode = mode;
  c->max_new = max_new_chunks;
  c->stream = s;
  c->n_pre = prefix ? prefix->N : 0;
  c->n1_pre = prefix ? prefix->N1 : 0;
  const int N_own = T / C, N1_own = T / C1;
  c->Ncap = N_own + max_new_chunks;
  c->N1cap = N1_own + (mode == PHOTON_MODE_HIER ? C2 * max_new_chunks : 0);

  Allocator al{s, &c->allocs, &c->kv_bytes};
  auto bail = [&](int code) {
    cudaGetLastError();
    kv_release(m, c, s);
    if (c->side) cudaStreamDestroy(c->side);
    if (c->cap) cudaStreamDestroy(c->cap);
    if (c->hi) cudaStreamDestroy(c->hi);
    if (c->ev_fork) cudaEventDestroy(c->ev_fork);
    if (c->ev_join_hi) cudaEventDestroy(c->ev_join_hi);
    if (c->ev_join) cudaEventDestroy(c->ev_join);
    free_list(c->allocs, s);
    cudaStreamSynchronize(s);
    delete c;
    return code == PHOTON_ERR_OOM ? fail(code, "device allocation failed during prefill") : code;
  };
  int rc = ensure_encoder(m, s);
  if (rc) return bail(rc);

  const size_t hd = (size_t)m->H * m->dh;
  if (paged) {
    // top K / V in the model's pages, mapped run by run as positions arrive
    c->paged = true;
    c->kv_tab_len = (c->Ncap + m->kv_page_rows - 1) / m->kv_page_rows;
    c->kv_table = al.get<int>((size_t)B * c->kv_tab_len * sizeof(int));
    c->kv_table_host.assign((size_t)B * c->kv_tab_len, -1);
    c->top_k = m->kv_pool;
    c->top_v = m->kv_pool + (size_t)m->kv_pool_pages * kv_page_bytes(m);
    c->top_layer = 2 * (size_t)m->kv_pool_pages * kv_page_bytes(m);
  } else {
    c->top_layer = (size_t)B * hd * c->Ncap * m->es;
    c->top_k = al.get<char>(c->top_layer * m->Ltop);
    c->top_v = al.get<char>(c->top_layer * m->Ltop);
  }
  c->l1_layer = (size_t)B * hd * c->N1cap * m->es;
  c->l1_k = al.get<char>(c->l1_layer * m->L1);
  c->l1_v = al.get<char>(c->l1_layer * m->L1);
  if (al.err != cudaSuccess) return bail(PHOTON_ERR_OOM);
  if (paged) {  // the table (unmapped runs: -1), then pages for the prompt's positions
    if (cudaMemcpyAsync(c->kv_table, c->kv_table_host.data(), c->kv_table_host.size() * sizeof(int),
                        cudaMemcpyHostToDevice, s) != cudaSuccess)
      return bail(fail(PHOTON_ERR_CUDA, "page table upload failed"));
    const int rc_map = kv_map_through(c, N_own - 1, s);
    if (rc_map) return bail(rc_map);
  }

  // decode workspace (kept for the cache's lifetime)
  al.counter = &c->ws_bytes;
  const int rows_c = B * C, rows_g = B * C2;
  const size_t es = m->es;
  c->xd = al.get<float>((size_t)rows_c * d * 4);
  c->xs = al.get<float>((size_t)rows_g * d * 4);
  c->xt = al.get<float>((size_t)B * d * 4);
  c->x1 = al.get<float>((size_t)rows_g * d * 4);
  c->xn = al.get<void>((size_t)rows_c * d * es);
  c->q = al.get<void>((size_t)rows_c * d * es);
  c->att = al.get<void>((size_t)rows_c * d * es);
  c->hid = al.get<void>((size_t)rows_c * m->f * es);
  c->a_hat = al.get<void>((size_t)rows_g * d * es);
  c->a = al.get<void>((size_t)rows_g * d * es);
  c->embd = al.get<void>((size_t)rows_c * d * es);
  c->hn = al.get<void>((size_t)rows_g * d * es);
  c->o = al.get<void>((size_t)B * d * es);
  c->logits = al.get<float>((size_t)rows_g * m->V * 4);
  c->d2_layer = (size_t)B * hd * C2 * es;
  c->d2k = al.get<char>(c->d2_layer * m->Ld2);
  c->d2v = al.get<char>(c->d2_layer * m->Ld2);
  c->d1_layer = (size_t)rows_g * hd * (2 * C1) * es;
  c->d1k = al.get<char>(c->d1_layer * m->Ld1);
  c->d1v = al.get<char>(c->d1_layer * m->Ld1);
  c->next_ids = al.get<int32_t>((size_t)rows_g * 4);
  c->used = al.get<int32_t>((size_t)rows_c * 4);
  c->d_err = al.get<int>(16);
  c->d_pos = al.get<int>(16);
  c->amax_cap = (m->V + 127) / 128;
  c->amax_part = al.get<unsigned long long>((size_t)rows_g * c->amax_cap * 8);
  c->tok_out = al.get<int32_t>((size_t)rows_c * 4);
  size_t gw = 0;
  gw = std::max(gw, block_ws_need(m, B));
  gw = std::max(gw, block_ws_need(m, rows_g));
  gw = std::max(gw, block_ws_need(m, rows_c));
  gw = std::max(gw, gemm_ws_need(m, B, C2 * d, d));
  gw = std::max(gw, gemm_ws_need(m, rows_g, C1 * d, d));
  gw = std::max(gw, gemm_ws_need(m, B, d, C2 * d));
  gw = std::max(gw, gemm_ws_need(m, rows_g, d, C1 * d));
  gw = std::max(gw, gemm_ws_need(m, rows_g, m->V, d));
  c->gemm_ws_bytes = gw;
  c->gemm_ws = al.get<float>(gw);
  size_t aw = attn_ws_need(m->dt, B, m->H, m->dh, 1, c->n_pre + c->Ncap);
  if (mode == PHOTON_MODE_HIER)
    aw = std::max(aw, attn_ws_need(m->dt, B, m->H, m->dh, C2, c->n1_pre + c->N1cap));
  aw = std::max(aw, attn_ws_need(m->dt, B, m->H, m->dh, C2, C2));
  for (int i = 0; i < C1; ++i)
    aw = std::max(aw, attn_ws_need(m->dt, rows_g, m->H, m->dh, i == 0 ? C1 : 1, C1 + i));
  c->attn_ws_bytes = aw;
  c->attn_ws = al.get<float>(aw);
  if (prefix) {  // top step (1 query) and HierGen's level-1 re-encode (C2 queries) per sequence
    AttnArgs pa;
    pa.G = B;
    pa.q_len = C2;
    pa.H = m->H;
    pa.dh = m->dh;
    c->pre_ws_bytes = attn_prefix_split_bytes(pa);
    c->pre_ws = al.get<float>(c->pre_ws_bytes);
  }
  // top-encoder branch (B rows) of RecGen, run concurrently with the token decoder
  c->xn_t = al.get<void>((size_t)B * d * es);
  c->q_t = al.get<void>((size_t)B * d * es);
  c->att_t = al.get<void>((size_t)B * d * es);
  c->hid_t = al.get<void>((size_t)B * m->f * es);
  c->gemm_ws_t = al.get<float>(gw);
  c->gemm_cnt = al.get<int>(kGemmTileCounters * sizeof(int));
  c->gemm_cnt_t = al.get<int>(kGemmTileCounters * sizeof(int));
  if (m->use_tc) {
    const size_t srows = (size_t)std::max(rows_g * C1, std::max(rows_g, B));
    c->sn_rows = (int)srows;
    c->sn_x = al.get<void>(srows * d * es);
    c->sn_ss = al.get<float>(srows * kSsqCap * sizeof(float));
    c->sn_x_t = al.get<void>((size_t)B * d * es);
    c->sn_ss_t = al.get<float>((size_t)B * kSsqCap * sizeof(float));
    c->stk_cnt_len = (d / 128) * ((B * C2 + 63) / 64);
    c->stk_part = al.get<float>(stack_local_scratch_bytes(B * C2, d));
    c->stk_cnt = al.get<int>((size_t)c->stk_cnt_len * sizeof(int));
    c->stk_bar = al.get<unsigned int>(256);
    if (top_mega_enabled() && !prefix && !paged &&
        top_step_supported(B, d, m->H, m->dh, m->f, m->Ltop, C2, c->Ncap) &&
        top_step_ssq_slots(d) <= kSsqCap) {
      c->tk_part_bytes = top_step_part_bytes(d, m->f, C2);
      c->tk_part = al.get<float>(c->tk_part_bytes);
      c->tk_cnt = al.get<int>((size_t)top_step_counters(d) * sizeof(int));
      c->tk_bar = al.get<unsigned>(64);
      c->tk_ok = true;
    }
  }
  c->attn_ws_t = al.get<float>(aw);
  if (cudaStreamCreateWithFlags(&c->side, cudaStreamNonBlocking) != cudaSuccess ||
      cudaStreamCreateWithFlags(&c->cap, cudaStreamNonBlocking) != cudaSuccess ||
      cudaStreamCreateWithPriority(&c->hi, cudaStreamNonBlocking, stream_priority_high()) != cudaSuccess ||
      cudaEventCreateWithFlags(&c->ev_fork, cudaEventDisableTiming) != cudaSuccess ||
      cudaEventCreateWithFlags(&c->ev_join_hi, cudaEventDisableTiming) != cudaSuccess ||
      cudaEventCreateWithFlags(&c->ev_join, cudaEventDisableTiming) != cudaSuccess)
    return bail(fail(PHOTON_ERR_CUDA, "stream/event creation failed"));
  const int positions =
      std::max(std::max(c->n_pre + c->Ncap, c->n1_pre + N1_own + C2 * max_new_chunks), 2 * C1 + C2) + 1;
  rc = upload_rope(m, &c->rope, positions);
  if (al.err != cudaSuccess || rc) return bail(rc ? rc : PHOTON_ERR_OOM);
  if (cudaMemsetAsync(c->d_err, 0, 16, s) != cudaSuccess ||
      cudaMemsetAsync(c->gemm_cnt, 0, kGemmTileCounters * sizeof(int), s) != cudaSuccess ||
      cudaMemsetAsync(c->gemm_cnt_t, 0, kGemmTileCounters * sizeof(int), s) != cudaSuccess ||
      (c->stk_cnt && cudaMemsetAsync(c->stk_cnt, 0, (size_t)c->stk_cnt_len * sizeof(int), s) != cudaSuccess) ||
      (c->tk_cnt && cudaMemsetAsync(c->tk_cnt, 0, (size_t)top_step_counters(d) * sizeof(int), s) != cudaSuccess) ||
      (c->tk_bar && cudaMemsetAsync(c->tk_bar, 0, 64, s) != cudaSuccess))
    return bail(PHOTON_ERR_CUDA);

  if (!shell) {
    // prefill workspace (released at the end of this call)
    std::vector<void*> tmp;
    size_t tmp_bytes = 0;
    Allocator at{s, &tmp, &tmp_bytes};
    const long long rows1 = rows0 / C1, rows2 = rows0 / C;
    void* emb = at.get<void>((size_t)rows0 * d * es);
    float* x = at.get<float>((size_t)rows1 * d * 4);
    void* xn = at.get<void>((size_t)rows1 * d * es);
    void* q = at.get<void>((size_t)rows1 * d * es);
    void* att = at.get<void>((size_t)rows1 * d * es);
    void* hid = at.get<void>((size_t)rows1 * m->f * es);
    size_t pgw = std::max(block_ws_need(m, (int)rows1), block_ws_need(m, (int)rows2));
    pgw = std::max(pgw, gemm_ws_need(m, (int)rows1, d, C1 * d));
    pgw = std::max(pgw, gemm_ws_need(m, (int)rows2, d, C2 * d));
    float* pws = at.get<float>(pgw);
    size_t ppb = 0;
    float* ppw = nullptr;
    if (prefix) {  // the level-1 stack has the most query rows
      AttnArgs pa;
      pa.G = B;
      pa.q_len = N1_own;
      pa.H = m->H;
      pa.dh = m->dh;
      ppb = attn_prefix_split_bytes(pa);
      ppw = at.get<float>(ppb);
    }
    if (at.err != cudaSuccess) {
      free_list(tmp, s);
      return bail(PHOTON_ERR_OOM);
    }
    Bufs pb{xn, q, att, hid, c->rope, pws, pgw, c->gemm_cnt, nullptr, 0, c->d_err};
    pb.pre_ws = ppw;
    pb.pre_ws_bytes = ppb;

    // a1: embedding; a2: Chunker_1 (concatenate C1 states, linear C1*d -> d)
    launch_embed(m->dt, d_tokens, m->ptr(m->i_embed), emb, (int)rows0, d, m->V, c->d_err, s);
    gemm(m, pb, emb, (long long)C1 * d, m->ptr(m->i_ch1), (long long)C1 * d, (int)rows1, d, C1 * d,
         epi(EPI_STORE_F32, x, d), s);
    // a3: level-1 encoder over T/C1 positions per sequence, writing the level-1 KV
    StackRun r1;
    r1.G = B;
    r1.q_len = N1_own;
    r1.p0 = c->n1_pre;
    r1.kv_off = c->n1_pre;
    r1.kc = c->l1_k;
    r1.vc = c->l1_v;
    r1.layer_bytes = c->l1_layer;
    r1.cap = c->N1cap;
    if (prefix) {
      r1.kp = prefix->l1_k;
      r1.vp = prefix->l1_v;
      r1.pre_layer_bytes = prefix->l1_layer;
      r1.cap_pre = prefix->N1cap;
      r1.n_pre = c->n1_pre;
    }
    run_stack(m, m->i_enc1, m->L1, x, r1, pb, s);
    launch_rmsnorm(m->dt, x, (const float*)m->ptr(m->i_enc1_g), xn, (int)rows1, d, 1, 0,
                   m->cfg.norm_eps, s);
    // a4: Chunker_2 on the level-1 states (x is reused for the top stream)
    gemm(m, pb, xn, (long long)C2 * d, m->ptr(m->i_ch2), (long long)C2 * d, (int)rows2, d, C2 * d,
         epi(EPI_STORE_F32, x, d), s);
    // a5: top encoder over T/C positions, writing the top KV
    StackRun rt;
    rt.G = B;
    rt.q_len = N_own;
    rt.p0 = c->n_pre;
    rt.kv_off = c->n_pre;
    rt.kc = c->top_k;
    rt.vc = c->top_v;
    rt.layer_bytes = c->top_layer;
    rt.cap = c->Ncap;
    set_paged(rt, c);
    if (prefix) {
      rt.kp = prefix->top_k;
      rt.vp = prefix->top_v;
      rt.pre_layer_bytes = prefix->top_layer;
      rt.cap_pre = prefix->Ncap;
      rt.n_pre = c->n_pre;
    }
    run_stack(m, m->i_top, m->Ltop, x, rt, pb, s);
    // pending output: final norm of the last top position of each sequence
    launch_rmsnorm(m->dt, x, (const float*)m->ptr(m->i_top_g), c->o, B, d, N_own, N_own - 1,
                   m->cfg.norm_eps, s);
    if (o_all)
      launch_rmsnorm(m->dt, x, (const float*)m->ptr(m->i_top_g), o_all, B * N_own, d, 1, 0, m->cfg.norm_eps, s);
    cudaError_t le = cudaGetLastError();
    free_list(tmp, s);
    if (le != cudaSuccess) {
      return bail(fail(PHOTON_ERR_CUDA, "prefill launch failed: %s", cudaGetErrorString(le)));
    }

  }
  c->N = c->n_pre + N_own;
  c->N1 = c->n1_pre + N1_own;
  // a6: RecGen keeps only the top-level KV (RecGen section)
  if (mode == PHOTON_MODE_REC) {
    cudaFreeAsync(c->l1_k, s);
    cudaFreeAsync(c->l1_v, s);
    for (auto it = c->allocs.begin(); it != c->allocs.end();) {
      if (*it == c->l1_k || *it == c->l1_v)
        it = c->allocs.erase(it);
      else
        ++it;
    }
    c->kv_bytes -= 2 * c->l1_layer * m->L1;
    c->l1_k = c->l1_v = nullptr;
    c->N1 = 0;
  }
  {
    const int pos[4] = {c->N, c->N1, 0, 0};  // pageable source: staged before the call returns
    if (cudaMemcpyAsync(c->d_pos, pos, sizeof(pos), cudaMemcpyHostToDevice, s) != cudaSuccess)
      return bail(fail(PHOTON_ERR_CUDA, "position upload failed"));
  }
  // RecGen never reads the encoder again: drop it unless a HierGen cache does
  if (note_encoder_use(m, s) != PHOTON_OK ||
      (mode != PHOTON_MODE_HIER && m->hier_caches == 0 && release_encoder(m, s) != PHOTON_OK))
    return bail(PHOTON_ERR_CUDA);
  m->live_caches++;
  if (mode == PHOTON_MODE_HIER) m->hier_caches++;
  if (paged) m->kv_paged_caches++;
  if (prefix) prefix->dependents++;
  *out = c;
  return PHOTON_OK;
}

}  // extern "C"

// Enqueues one decode step (a7..a13) on s.  Every per-step varying value is
// read on the device (positions from c->d_pos), so the same launches can be
// captured once into a CUDA graph and replayed for later steps.
static bool recgen_fork_enabled() {
  static const bool on = [] {
    const char* e = getenv("PHOTON_RECGEN_FORK");
    return !(e && e[0] == '0');
  }();
  return on;
}
static bool token_priority_enabled() {
  static const bool on = [] {
    const char* e = getenv("PHOTON_TOKEN_PRIORITY");
    return e && e[0] == '1';
  }();
  return on;
}

static bool stack_mega_enabled() {
  static const bool on = [] {
    const char* e = getenv("PHOTON_STACK_MEGA");
    return e && e[0] == '1';
  }();
  return on;
}

// One single-row token-decoder step (all Ld1 blocks) as one persistent
// cooperative kernel; false when it does not apply (then run_stack does it).
static bool token_step_persistent(photon_model* m, photon_cache* c, const Bufs& b, float* x,
                                  const StackRun& r, cudaStream_t s) {
  if (!m->use_tc || !stack_mega_enabled() || !c->stk_part || r.q_len != 1 || m->Ld1 > 8) return false;
  if (!stack_local_supported(r.G, m->d, m->H, m->dh, m->f, m->Ld1, r.p0, r.cap)) return false;
  StackLocalLaunch k;
  memset(&k, 0, sizeof(k));
  for (int l = 0; l < m->Ld1; ++l) {
    const BlockW w = m->block(m->i_dec1, l);
    k.wqkv[l] = w.wqkv;
    k.wo[l] = w.wo;
    k.w1[l] = w.w1;
    k.w2[l] = w.w2;
    k.g_attn[l] = w.g_attn;
    k.g_mlp[l] = w.g_mlp;
  }
  k.x = x;
  k.xn = b.xn;
  k.q = b.q;
  k.att = b.att;
  k.hid = b.hid;
  k.kc = r.kc;
  k.vc = r.vc;
  k.layer_elems = (long long)(r.layer_bytes / 2);
  k.rope = b.rope;
  k.part = c->stk_part;
  k.tile_cnt = c->stk_cnt;
  k.cnt_len = c->stk_cnt_len;
  k.bar = c->stk_bar;
  k.err = b.err;
  k.rows = r.G;
  k.d = m->d;
  k.H = m->H;
  k.f = m->f;
  k.L = m->Ld1;
  k.cap = r.cap;
  k.p0 = r.p0;
  k.eps = m->cfg.norm_eps;
  k.scale = 1.0f / sqrtf((float)m->dh);
  k.skip_first_norm = r.xn_ready ? 1 : 0;
  return launch_stack_local(k, s);
}

// Which part of a decode step to enqueue: the whole step, or (pipelined
// RecGen) only the main chain (Converter_2, Decoder_2, Chunker_2, top step)
// or only the token branch (Converter_1, token decoder, heads) of A-hat
// buffer `parity`.
enum DecodePart { DEC_ALL = 0, DEC_MAIN = 1, DEC_TOK = 2 };

static Bufs tok_bufs(photon_cache* c) {
  Bufs b = decode_bufs(c);
  b.xn = c->xn_k;
  b.q = c->q_k;
  b.att = c->att_k;
  b.hid = c->hid_k;
  b.gemm_ws = c->gemm_ws_k;
  b.gemm_cnt = c->gemm_cnt_k;
  b.attn_ws = c->attn_ws_k;
  b.sn_x = c->sn_x_k;
  b.sn_ss = c->sn_ss_k;
  return b;
}

static void enqueue_decode(photon_model* m, photon_cache* c, int mode, int32_t* own_tokens,
                           float* d_out_logits, const int32_t* d_force_tokens,
                           const void* d_force_a, cudaStream_t s, int part = DEC_ALL,
                           int parity = 0) {
  int32_t* d_out_tokens = own_tokens;
  const int B = c->B, C1 = m->C1, C2 = m->C2, C = m->C, d = m->d, V = m->V, G = B * C2;
  const float eps = m->cfg.norm_eps;
  const Bufs b = decode_bufs(c);
  // A-hat of this step; the token branch's buffers and residual stream
  void* const ahat = part == DEC_ALL ? c->a_hat : c->ahat_p[parity];
  const Bufs bk = part == DEC_TOK ? tok_bufs(c) : b;
  float* const xdk = part == DEC_TOK ? c->xd_k : c->xd;
  auto top_step = [&](float* x, const Bufs& bb, cudaStream_t st) {
    StackRun rt;
    rt.G = B;
    rt.q_len = 1;
    rt.p0 = 0;
    rt.p0_dev = c->d_pos;
    rt.n_plan = c->n_pre + c->Ncap;
    rt.sn_rows = c->sn_x_t ? B : 0;
    rt.kv_off = c->n_pre;
    rt.kc = c->top_k;
    rt.vc = c->top_v;
    rt.layer_bytes = c->top_layer;
    rt.cap = c->Ncap;
    set_paged(rt, c);
    if (c->prefix) {
      rt.kp = c->prefix->top_k;
      rt.vp = c->prefix->top_v;
      rt.pre_layer_bytes = c->prefix->top_layer;
      rt.cap_pre = c->prefix->Ncap;
      rt.n_pre = c->n_pre;
    }
    run_stack(m, m->i_top, m->Ltop, x, rt, bb, st);
    launch_rmsnorm(m->dt, x, (const float*)m->ptr(m->i_top_g), c->o, B, d, 1, 0, eps, st);
    launch_advance(c->d_pos, 1, mode == PHOTON_MODE_HIER ? C2 : 0, st);
  };

  // a12 + a13: Chunker_2 of `src` ([B, C2*d] rows), the top step, its final
  // norm into the pending output, and the position advance -- in one
  // persistent launch when the cache has one planned, else kernel by kernel
  auto top_chain = [&](const void* src, const Bufs& bb, cudaStream_t st) {
    if (c->tk_ok) {
      TopStepPlan* plan = nullptr;
      for (auto& e : c->tk_plans)
        if (e.src == src && e.xs == bb.sn_x && e.mode == mode) plan = e.plan;
      if (!plan) {
        TopStepLaunch t;
        memset(&t, 0, sizeof(t));
        t.ch_in = src;
        t.ch_ld = (long long)C2 * d;
        t.w_ch = m->ptr(m->i_ch2);
        for (int l = 0; l < m->Ltop; ++l) {
          const BlockW w = m->block(m->i_top, l);
          t.wqkv[l] = w.wqkv;
          t.wo[l] = w.wo;
          t.w1[l] = w.w1;
          t.w2[l] = w.w2;
          t.g_attn[l] = w.g_attn;
          t.g_mlp[l] = w.g_mlp;
        }
        t.g_final = (const float*)m->ptr(m->i_top_g);
        t.x = c->xt;
        t.xs = bb.sn_x;
        t.ssq = bb.sn_ss;
        t.q = bb.q;
        t.att = bb.att;
        t.hid = bb.hid;
        t.kc = c->top_k;
        t.vc = c->top_v;
        t.layer_elems = (long long)(c->top_layer / m->es);
        t.cap = c->Ncap;
        t.kv_off = c->n_pre;
        t.rope = c->rope;
        t.pos = c->d_pos;
        t.dN1 = mode == PHOTON_MODE_HIER ? C2 : 0;
        t.o_out = c->o;
        t.part = c->tk_part;
        t.part_bytes = c->tk_part_bytes;
        t.cnt = c->tk_cnt;
        t.bar = c->tk_bar;
        t.err = c->d_err;
        t.B = B;
        t.d = d;
        t.H = m->H;
        t.f = m->f;
        t.L = m->Ltop;
        t.C2 = C2;
        t.eps = eps;
        t.scale = 1.0f / sqrtf((float)m->dh);
        plan = top_step_plan(t);
        if (plan) c->tk_plans.push_back({src, bb.sn_x, mode, plan});
      }
      if (plan && launch_top_step(plan, st)) return;
    }
    gemm(m, bb, src, (long long)C2 * d, m->ptr(m->i_ch2), (long long)C2 * d, B, d, C2 * d,
         epi(EPI_STORE_F32, c->xt, d), st);
    top_step(c->xt, bb, st);
  };

  if (part != DEC_TOK) {
  // a7: Converter_2 -- o [B, d] -> C2 conditioning vectors per sequence
  gemm(m, b, c->o, d, m->ptr(m->i_cv2), d, B, C2 * d, d, epi(EPI_STORE_F32, c->xd, (long long)C2 * d), s);
  // a8: level-2 decoder over its C2 positions (chunk-local causal) -> A-hat
  StackRun r2;
  r2.G = B;
  r2.q_len = C2;
  r2.kc = c->d2k;
  r2.vc = c->d2v;
  r2.layer_bytes = c->d2_layer;
  r2.cap = C2;
  r2.sn_rows = c->sn_rows;
  run_stack(m, m->i_dec2, m->Ld2, c->xd, r2, b, s);
  launch_rmsnorm(m->dt, c->xd, (const float*)m->ptr(m->i_dec2_g), ahat, G, d, 1, 0, eps, s);
  if (part == DEC_MAIN) {
    // pipelined RecGen: the top encoder's next input follows at once; the
    // token branch of this A-hat runs as its own graph
    top_chain(ahat, b, s);
    return;
  }
  }
  // RecGen: the top encoder's next input is Chunker_2(A-hat) and does not
  // depend on the tokens, so the top-encoder branch (a12-R, a13) runs on the
  // side stream, with its own buffers, while the token decoder (a9-a11)
  // runs here; the two chains join at the end of the step.
  const bool fork = part == DEC_ALL && mode == PHOTON_MODE_REC && c->side != nullptr && recgen_fork_enabled();
  if (fork) {
    cudaEventRecord(c->ev_fork, s);
    cudaStreamWaitEvent(c->side, c->ev_fork, 0);
    Bufs bt = b;
    bt.xn = c->xn_t;
    bt.q = c->q_t;
    bt.att = c->att_t;
    bt.hid = c->hid_t;
    bt.gemm_ws = c->gemm_ws_t;
    bt.gemm_cnt = c->gemm_cnt_t;
    bt.attn_ws = c->attn_ws_t;
    bt.sn_x = c->sn_x_t;
    bt.sn_ss = c->sn_ss_t;
    const void* src = d_force_a ? d_force_a : ahat;
    top_chain(src, bt, c->side);
    cudaEventRecord(c->ev_join, c->side);
  }
  // the token branch: the caller's stream, or (optionally) a high-priority
  // internal stream so its kernels win the scheduler against the top branch
  cudaStream_t ts = s;
  if (fork && token_priority_enabled() && c->hi) {
    cudaStreamWaitEvent(c->hi, c->ev_fork, 0);
    ts = c->hi;
  }
  // a9: Converter_1 -- each A-hat row -> C1 conditioning vectors (rows g*C1 + i)
  gemm(m, bk, ahat, d, m->ptr(m->i_cv1), d, G, C1 * d, d, epi(EPI_STORE_F32, xdk, (long long)C1 * d), ts);
  // a10/a11: token decoder, prefix pass over the C1 conditioning positions,
  // then C1-1 single-row steps; head + greedy argmax after each
  StackRun r1;
  r1.G = G;
  r1.q_len = C1;
  r1.kc = c->d1k;
  r1.vc = c->d1v;
  r1.layer_bytes = c->d1_layer;
  r1.cap = 2 * C1;
  r1.sn_rows = c->sn_rows;
  run_stack(m, m->i_dec1, m->Ld1, xdk, r1, bk, ts);
  const int amax_tiles = m->use_tc ? gemm_tc_argmax_tiles(G, V, d) : 0;
  bool fused_embed = false;  // the last head also embedded and normalised the next step's input
  int* chunk_ctr = c->d_pos + 2;  // chunks this cache has generated (sampling keys)
  auto head = [&](const float* x, int in_step, int in_off, int i) {
    launch_rmsnorm(m->dt, x, (const float*)m->ptr(m->i_dec1_g), c->hn, G, d, in_step, in_off, eps, ts);
    const long long ld = d_out_logits ? (long long)C1 * V : V;
    SampleArgs sa;
    sa.inv_t = c->samp_inv_t;
    sa.seed = c->samp_seed;
    sa.chunk = chunk_ctr;
    sa.C1 = C1;
    sa.C2 = C2;
    sa.i = i;
    const bool topp = c->samp_inv_t > 0.f && c->samp_top_p < 1.f;  // nucleus draws need the whole row
    if (amax_tiles > 0 && amax_tiles <= c->amax_cap && !topp) {
      // tensor-core head with the greedy choice fused into its epilogue;
      // logits are written only when the caller asks for them
      Epilogue e = epi(EPI_ARGMAX, d_out_logits ? d_out_logits + (size_t)i * V : nullptr, ld);
      e.argmax_part = c->amax_part;
      e.argmax_tiles = amax_tiles;
      e.samp = sa;
      gemm(m, bk, c->hn, d, m->ptr(m->i_head), d, G, V, d, e, ts);
      if (i + 1 < C1) {
        // greedy choice + the next step's embedding and first attention norm
        launch_argmax_embed_norm(m->dt, c->amax_part, amax_tiles, G, V, i, C1, d_force_tokens,
                                 d_out_tokens, c->used, c->next_ids, c->d_err, m->ptr(m->i_embed),
                                 c->xs, m->block(m->i_dec1, 0).g_attn, bk.xn, d, eps, ts);
        fused_embed = true;
      } else {
        launch_argmax_partials(c->amax_part, amax_tiles, G, V, i, C1, d_force_tokens, d_out_tokens,
                               c->used, c->next_ids, c->d_err, chunk_ctr, ts);
      }
    } else {
      float* lg = d_out_logits ? d_out_logits + (size_t)i * V : c->logits;
      gemm(m, bk, c->hn, d, m->ptr(m->i_head), d, G, V, d, epi(EPI_STORE_F32, lg, ld), ts);
      if (topp)
        launch_sample_topp(lg, ld, G, V, i, C1, sa, c->samp_top_p, d_force_tokens, d_out_tokens, c->used,
                           c->next_ids, c->d_err, ts);
      else
        launch_argmax(lg, ld, G, V, i, C1, d_force_tokens, d_out_tokens, c->used, c->next_ids,
                      c->d_err, sa, ts);
      if (i + 1 == C1) launch_advance(chunk_ctr, 1, 0, ts);  // count the chunk
    }
  };
  head(xdk, C1, C1 - 1, 0);
  for (int i = 1; i < C1; ++i) {
    if (!fused_embed)
      launch_embed_f32(m->dt, c->next_ids, m->ptr(m->i_embed), c->xs, G, d, V, c->d_err, ts);
    StackRun rs = r1;
    rs.q_len = 1;
    rs.p0 = C1 + i - 1;
    rs.xn_ready = fused_embed;
    fused_embed = false;
    if (!token_step_persistent(m, c, bk, c->xs, rs, ts)) run_stack(m, m->i_dec1, m->Ld1, c->xs, rs, bk, ts);
    head(c->xs, 1, 0, i);
  }
  if (part == DEC_TOK) return;
  // a12: input of the top encoder's next position
  if (fork) {
    if (ts != s) {
      cudaEventRecord(c->ev_join_hi, ts);
      cudaStreamWaitEvent(s, c->ev_join_hi, 0);
    }
    cudaStreamWaitEvent(s, c->ev_join, 0);  // join the top-encoder branch
    return;
  }
  if (mode == PHOTON_MODE_REC) {
    // RecGen without a side stream: Chunker_2(A-hat), no re-encoding
    top_chain(d_force_a ? d_force_a : c->a_hat, b, s);
    return;
  } else {
    // HierGen: embed the written tokens, Chunker_1, level-1 encoder with its cache, Chunker_2
    launch_embed(m->dt, c->used, m->ptr(m->i_embed), c->embd, B * C, d, V, c->d_err, s);
    gemm(m, b, c->embd, (long long)C1 * d, m->ptr(m->i_ch1), (long long)C1 * d, G, d, C1 * d,
         epi(EPI_STORE_F32, c->x1, d), s);
    StackRun re;
    re.G = B;
    re.q_len = C2;
    re.p0 = 0;
    re.p0_dev = c->d_pos + 1;
    re.n_plan = c->n1_pre + c->N1cap;
    re.kv_off = c->n1_pre;
    re.kc = c->l1_k;
    re.vc = c->l1_v;
    re.layer_bytes = c->l1_layer;
    re.cap = c->N1cap;
    re.sn_rows = c->sn_rows;
    if (c->prefix) {
      re.kp = c->prefix->l1_k;
      re.vp = c->prefix->l1_v;
      re.pre_layer_bytes = c->prefix->l1_layer;
      re.cap_pre = c->prefix->N1cap;
      re.n_pre = c->n1_pre;
    }
    run_stack(m, m->i_enc1, m->L1, c->x1, re, b, s);
    launch_rmsnorm(m->dt, c->x1, (const float*)m->ptr(m->i_enc1_g), c->a, G, d, 1, 0, eps, s);
    // a13: one top-encoder step at position N (KV append + decode attention)
    top_chain(c->a, b, s);
  }
}

static bool graphs_enabled() {
  static const bool on = [] {
    const char* e = getenv("PHOTON_DECODE_GRAPH");
    return !(e && e[0] == '0');
  }();
  return on;
}

// ============================================================== any number of levels
// The general hierarchy (photon_init_weights_levels): L levels, each with a
// chunker and an encoder going up and a converter and a decoder coming
// down (explainer, architecture section, module table written for a
// general level l).  Runs on the same kernels as the two-level path;
// eager launches, with the plain decode step captured into a graph per mode.
struct GenCache {
  int L = 0;
  // encoder caches of levels 1..L ([E_l][B][H][cap][dh] per K and V); the
  // lower ones only in HierGen mode
  char* kc[PHOTON_MAX_LEVELS] = {};
  char* vc[PHOTON_MAX_LEVELS] = {};
  size_t layer[PHOTON_MAX_LEVELS] = {};
  int cap[PHOTON_MAX_LEVELS] = {};
  int n[PHOTON_MAX_LEVELS] = {};   // host copy of the entries per level
  int* d_n = nullptr;               // device: entries per level, then the chunk counter at [PHOTON_MAX_LEVELS]
  // top-down: per level l residual stream [G_l * C_l, d], reconstruction
  // (l >= 2) and chunk-local decoder KV
  float* xdec[PHOTON_MAX_LEVELS] = {};
  void* ahat[PHOTON_MAX_LEVELS] = {};
  char* dk[PHOTON_MAX_LEVELS] = {};
  char* dv[PHOTON_MAX_LEVELS] = {};
  size_t dlayer[PHOTON_MAX_LEVELS] = {};
  int G[PHOTON_MAX_LEVELS] = {};    // groups of level l's decoder
  // token decoder single-row steps and the head
  float* xs = nullptr;
  void* hn = nullptr;
  float* logits = nullptr;
  int32_t* next_ids = nullptr;
  int32_t* used = nullptr;
  int32_t* tok_out = nullptr;
  // HierGen re-encode and the top input
  void* emb = nullptr;
  float* xre[PHOTON_MAX_LEVELS] = {};
  void* sre[PHOTON_MAX_LEVELS] = {};
  float* xt = nullptr;
  Bufs b;
  bool graph_failed[2] = {false, false};
};

static int gen_check(const photon_level_config* c) {
  if (!c) return fail(PHOTON_ERR_ARG, "config is NULL");
  if (c->levels < 1 || c->levels > PHOTON_MAX_LEVELS)
    return fail(PHOTON_ERR_ARG, "levels must be 1..%d", PHOTON_MAX_LEVELS);
  if (c->vocab <= 0 || c->d_model <= 0 || c->n_heads <= 0 || c->head_dim <= 0)
    return fail(PHOTON_ERR_ARG, "non-positive model dimension");
  if (c->d_model != c->n_heads * c->head_dim) return fail(PHOTON_ERR_ARG, "d_model must equal n_heads * head_dim");
  if (c->head_dim != 32 && c->head_dim != 64) return fail(PHOTON_ERR_ARG, "head_dim must be 32 or 64");
  if (c->d_model % 64) return fail(PHOTON_ERR_ARG, "d_model must be a multiple of 64");
  for (int l = 0; l < c->levels; ++l) {
    if (c->chunk[l] < 1 || c->chunk[l] > 4) return fail(PHOTON_ERR_ARG, "chunk sizes must be 1..4");
    if (c->enc_layers[l] < 1 || c->dec_layers[l] < 1) return fail(PHOTON_ERR_ARG, "layer counts must be >= 1");
  }
  if (c->mlp_mult < 1) return fail(PHOTON_ERR_ARG, "mlp_mult must be >= 1");
  if (c->dtype != 0 && c->dtype != 1) return fail(PHOTON_ERR_ARG, "dtype must be 0 (fp32) or 1 (bf16)");
  if (!(c->norm_eps > 0.f) || !(c->rope_theta > 0.f) || !(c->init_std > 0.f))
    return fail(PHOTON_ERR_ARG, "eps, theta and init_std must be positive");
  return PHOTON_OK;
}

// Tensor list of an L-level model: embed; chunker_l and encoder_l for
// l = 1..L (the last encoder is the top encoder); converter_l and decoder_l
// for l = L..1; head.  For L = 2 this is the two-level list.
static void build_specs_levels(photon_model* m) {
  const long long d = m->d, V = m->V, f = m->f;
  const int L = m->NL;
  auto add = [&](const std::string& n, int g, long long numel, bool gain) {
    m->t.push_back(TensorRec{n, g, 0, numel, gain});
  };
  auto blocks = [&](const std::string& p, int n, int g) {
    for (int l = 0; l < n; ++l) {
      const std::string s = p + "." + std::to_string(l) + ".";
      add(s + "g_attn", g, d, true);
      add(s + "wq", g, d * d, false);
      add(s + "wk", g, d * d, false);
      add(s + "wv", g, d * d, false);
      add(s + "wo", g, d * d, false);
      add(s + "g_mlp", g, d, true);
      add(s + "w1", g, f * d, false);
      add(s + "w2", g, d * f, false);
    }
  };
  m->i_embed = (int)m->t.size();
  add("embed", G_EMB, V * d, false);
  for (int l = 1; l <= L; ++l) {
    const int g = l == L ? G_TOP : G_ENC1;
    const std::string name = l == L ? "top" : "enc" + std::to_string(l);
    m->i_chl[l - 1] = (int)m->t.size();
    add("chunker" + std::to_string(l), g, d * m->Cl[l - 1] * d, false);
    m->i_encl[l - 1] = (int)m->t.size();
    blocks(name, m->El[l - 1], g);
    m->i_encl_g[l - 1] = (int)m->t.size();
    add(name + ".g_final", g, d, true);
  }
  for (int l = L; l >= 1; --l) {
    m->i_cvl[l - 1] = (int)m->t.size();
    add("converter" + std::to_string(l), G_DEC, m->Cl[l - 1] * d * d, false);
    m->i_decl[l - 1] = (int)m->t.size();
    blocks("dec" + std::to_string(l), m->Dl[l - 1], G_DEC);
    m->i_decl_g[l - 1] = (int)m->t.size();
    add("dec" + std::to_string(l) + ".g_final", G_DEC, d, true);
  }
  m->i_head = (int)m->t.size();
  add("head", G_DEC, V * d, false);
  for (auto& r : m->t) {
    const size_t bytes = (size_t)r.numel * (r.gain ? 4 : m->es);
    r.offset = m->group_bytes[r.group];
    m->group_bytes[r.group] += (bytes + 255) & ~size_t(255);
  }
}

// Product C_1 * ... * C_l (P(0) = 1).
static int gen_prod(const photon_model* m, int l) {
  int p = 1;
  for (int j = 0; j < l; ++j) p *= m->Cl[j];
  return p;
}

static int gen_prefill(photon_model* m, const int32_t* d_tokens, int B, int T, int mode, int max_new,
                       cudaStream_t s, photon_cache** out) {
  const int L = m->NL, d = m->d, C = m->C, C1 = m->Cl[0], H = m->H, dh = m->dh;
  const size_t es = m->es, hd = (size_t)H * dh;
  const float eps = m->cfg.norm_eps;
  if (mode == PHOTON_MODE_REC && L < 2) return fail(PHOTON_ERR_ARG, "RecGen needs at least two levels");
  photon_cache* c = new photon_cache();
  GenCache* g = new GenCache();
  c->gen = g;
  g->L = L;
  c->m = m;
  c->B = B;
  c->T = T;
  c->mode = mode;
  c->max_new = max_new;
  c->stream = s;
  Allocator al{s, &c->allocs, &c->kv_bytes};
  auto bail = [&](int code) {
    cudaGetLastError();
    if (c->cap) cudaStreamDestroy(c->cap);
    free_list(c->allocs, s);
    cudaStreamSynchronize(s);
    delete g;
    delete c;
    return code == PHOTON_ERR_OOM ? fail(code, "device allocation failed during prefill") : code;
  };
  // encoder caches: level l holds T / P(l) entries after prefill and grows by
  // C / P(l) per HierGen step (the top by one per step in both modes)
  std::vector<void*> tmp;
  size_t tmp_bytes = 0;
  Allocator at{s, &tmp, &tmp_bytes};
  for (int l = 1; l <= L; ++l) {
    const int Tl = T / gen_prod(m, l);
    const bool keep = l == L || mode == PHOTON_MODE_HIER;
    const int grow = l == L ? 1 : C / gen_prod(m, l);
    g->cap[l - 1] = Tl + (keep ? grow * max_new : 0);
    g->layer[l - 1] = (size_t)B * hd * g->cap[l - 1] * es;
    Allocator& A = keep ? al : at;
    g->kc[l - 1] = A.get<char>(g->layer[l - 1] * m->El[l - 1]);
    g->vc[l - 1] = A.get<char>(g->layer[l - 1] * m->El[l - 1]);
    g->n[l - 1] = keep ? Tl : 0;
  }
  c->top_k = g->kc[L - 1];
  c->top_v = g->vc[L - 1];
  c->top_layer = g->layer[L - 1];
  c->Ncap = g->cap[L - 1];
  c->N = g->n[L - 1];
  c->N1 = (L >= 2 && mode == PHOTON_MODE_HIER) ? g->n[0] : 0;
  c->N1cap = L >= 2 ? g->cap[0] : 0;
  if (L >= 2 && mode == PHOTON_MODE_HIER) {
    c->l1_k = g->kc[0];
    c->l1_v = g->vc[0];
    c->l1_layer = g->layer[0];
  }
  // decode workspace
  al.counter = &c->ws_bytes;
  c->o = al.get<void>((size_t)B * d * es);
  c->d_err = al.get<int>(16);
  g->d_n = al.get<int>(64);
  int rows_max = B * C;
  int groups = B;
  for (int l = L; l >= 1; --l) {
    const int Cl = m->Cl[l - 1];
    g->G[l - 1] = groups;
    const int rows = groups * Cl;
    g->xdec[l - 1] = al.get<float>((size_t)rows * d * 4);
    if (l >= 2) g->ahat[l - 1] = al.get<void>((size_t)rows * d * es);
    const int kv = l == 1 ? 2 * C1 : Cl;
    g->dlayer[l - 1] = (size_t)groups * hd * kv * es;
    g->dk[l - 1] = al.get<char>(g->dlayer[l - 1] * m->Dl[l - 1]);
    g->dv[l - 1] = al.get<char>(g->dlayer[l - 1] * m->Dl[l - 1]);
    groups = rows;
  }
  const int G1 = g->G[0];
  g->xs = al.get<float>((size_t)G1 * d * 4);
  g->hn = al.get<void>((size_t)G1 * d * es);
  g->logits = al.get<float>((size_t)G1 * m->V * 4);
  g->next_ids = al.get<int32_t>((size_t)G1 * 4);
  g->used = al.get<int32_t>((size_t)B * C * 4);
  g->tok_out = al.get<int32_t>((size_t)B * C * 4);
  c->tok_out = g->tok_out;
  g->emb = al.get<void>((size_t)B * C * d * es);
  for (int l = 1; l < L; ++l) {
    const int rows = B * (C / gen_prod(m, l));
    g->xre[l - 1] = al.get<float>((size_t)rows * d * 4);
    g->sre[l - 1] = al.get<void>((size_t)rows * d * es);
  }
  g->xt = al.get<float>((size_t)B * d * 4);
  // workspaces of every GEMM and attention shape of a decode step
  size_t gw = 0, aw = 0;
  auto gneed = [&](int M, int N, int K) { gw = std::max(gw, gemm_ws_need(m, M, N, K)); };
  auto aneed = [&](int G, int q, int n) { aw = std::max(aw, attn_ws_need(m->dt, G, H, dh, q, n)); };
  gw = std::max(gw, block_ws_need(m, B));
  gw = std::max(gw, block_ws_need(m, rows_max));
  gneed(B, m->Cl[L - 1] * d, d);
  gneed(B, d, m->Cl[L - 1] * d);
  for (int l = L; l >= 1; --l) {
    const int Gl = g->G[l - 1], Cl = m->Cl[l - 1];
    gw = std::max(gw, block_ws_need(m, Gl * Cl));
    gw = std::max(gw, block_ws_need(m, Gl));
    gneed(Gl, Cl * d, d);
    aneed(Gl, std::min(Cl, 4), l == 1 ? 2 * C1 : Cl);
  }
  gneed(G1, m->V, d);
  for (int i = 0; i < C1; ++i) aneed(G1, i == 0 ? std::min(C1, 4) : 1, C1 + i);
  aneed(B, 1, g->cap[L - 1]);
  for (int l = 1; l < L; ++l) {
    const int q = C / gen_prod(m, l), rows = B * q;
    gw = std::max(gw, block_ws_need(m, rows));
    gneed(rows, d, m->Cl[l - 1] * d);
    if (q <= 4) aneed(B, q, g->cap[l - 1]);
  }
  Bufs& b = g->b;
  b.xn = al.get<void>((size_t)rows_max * d * es);
  b.q = al.get<void>((size_t)rows_max * d * es);
  b.att = al.get<void>((size_t)rows_max * d * es);
  b.hid = al.get<void>((size_t)rows_max * m->f * es);
  b.gemm_ws_bytes = gw;
  b.gemm_ws = al.get<float>(gw);
  b.gemm_cnt = al.get<int>(kGemmTileCounters * sizeof(int));
  b.attn_ws_bytes = aw;
  b.attn_ws = al.get<float>(aw);
  b.err = c->d_err;
  int positions = 2 * C1 + 1;
  for (int l = 0; l < L; ++l) positions = std::max(positions, std::max(g->cap[l], m->Cl[l]) + 1);
  int rc = upload_rope(m, &c->rope, positions);
  b.rope = c->rope;
  if (al.err != cudaSuccess || rc) return bail(rc ? rc : PHOTON_ERR_OOM);
  if (cudaStreamCreateWithFlags(&c->cap, cudaStreamNonBlocking) != cudaSuccess)
    return bail(fail(PHOTON_ERR_CUDA, "stream creation failed"));
  std::vector<int> hn(PHOTON_MAX_LEVELS + 1, 0);
  for (int l = 0; l < L; ++l) hn[l] = g->n[l];
  if (cudaMemsetAsync(c->d_err, 0, 16, s) != cudaSuccess ||
      cudaMemsetAsync(b.gemm_cnt, 0, kGemmTileCounters * sizeof(int), s) != cudaSuccess ||
      cudaMemcpyAsync(g->d_n, hn.data(), hn.size() * sizeof(int), cudaMemcpyHostToDevice, s) != cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess)  // the host copy of hn leaves scope
    return bail(PHOTON_ERR_CUDA);

  // prefill: bottom-up through every level
  const long long rows0 = (long long)B * T, rows1 = rows0 / m->Cl[0];
  void* emb = at.get<void>((size_t)rows0 * d * es);
  float* x = at.get<float>((size_t)rows1 * d * 4);
  void* sb = at.get<void>((size_t)rows1 * d * es);
  size_t pgw = 0, paw = 0;
  for (int l = 1; l <= L; ++l) {
    const int rows = (int)(rows0 / gen_prod(m, l)), Tl = T / gen_prod(m, l);
    pgw = std::max(pgw, block_ws_need(m, rows));
    pgw = std::max(pgw, gemm_ws_need(m, rows, d, m->Cl[l - 1] * d));
    if (Tl <= 4) paw = std::max(paw, attn_ws_need(m->dt, B, H, dh, Tl, Tl));
  }
  Bufs pb;
  pb.xn = at.get<void>((size_t)rows1 * d * es);
  pb.q = at.get<void>((size_t)rows1 * d * es);
  pb.att = at.get<void>((size_t)rows1 * d * es);
  pb.hid = at.get<void>((size_t)rows1 * m->f * es);
  pb.rope = c->rope;
  pb.gemm_ws = at.get<float>(pgw);
  pb.gemm_ws_bytes = pgw;
  pb.gemm_cnt = b.gemm_cnt;
  pb.attn_ws = at.get<float>(paw);
  pb.attn_ws_bytes = paw;
  pb.err = c->d_err;
  if (at.err != cudaSuccess) {
    free_list(tmp, s);
    return bail(PHOTON_ERR_OOM);
  }
  launch_embed(m->dt, d_tokens, m->ptr(m->i_embed), emb, (int)rows0, d, m->V, c->d_err, s);
  const void* prev = emb;
  for (int l = 1; l <= L; ++l) {
    const int Cl = m->Cl[l - 1], Tl = T / gen_prod(m, l), rows = B * Tl;
    gemm(m, pb, prev, (long long)Cl * d, m->ptr(m->i_chl[l - 1]), (long long)Cl * d, rows, d, Cl * d,
         epi(EPI_STORE_F32, x, d), s);
    StackRun r;
    r.G = B;
    r.q_len = Tl;
    r.kc = g->kc[l - 1];
    r.vc = g->vc[l - 1];
    r.layer_bytes = g->layer[l - 1];
    r.cap = g->cap[l - 1];
    r.n_plan = Tl;
    run_stack(m, m->i_encl[l - 1], m->El[l - 1], x, r, pb, s);
    if (l < L) {
      launch_rmsnorm(m->dt, x, (const float*)m->ptr(m->i_encl_g[l - 1]), sb, rows, d, 1, 0, eps, s);
      prev = sb;
    } else {
      launch_rmsnorm(m->dt, x, (const float*)m->ptr(m->i_encl_g[l - 1]), c->o, B, d, Tl, Tl - 1, eps, s);
    }
  }
  const cudaError_t e = cudaGetLastError();
  free_list(tmp, s);
  if (e != cudaSuccess) return bail(fail(PHOTON_ERR_CUDA, "prefill launch: %s", cudaGetErrorString(e)));
  m->live_caches++;
  if (mode == PHOTON_MODE_HIER) m->hier_caches++;
  *out = c;
  return PHOTON_OK;
}

// One decode step of an L-level model: top-down through every level (all
// groups of a level at once), the token decoder and head, then the top
// encoder's next input and its step.
static void gen_enqueue(photon_model* m, photon_cache* c, int mode, int32_t* out_tokens, float* out_logits,
                        const int32_t* force, const void* force_a, cudaStream_t s) {
  GenCache* g = c->gen;
  const int L = m->NL, B = c->B, d = m->d, C = m->C, C1 = m->Cl[0], V = m->V;
  const float eps = m->cfg.norm_eps;
  const Bufs& b = g->b;
  const void* src = c->o;
  for (int l = L; l >= 2; --l) {
    const int Gl = g->G[l - 1], Cl = m->Cl[l - 1];
    gemm(m, b, src, d, m->ptr(m->i_cvl[l - 1]), d, Gl, Cl * d, d, epi(EPI_STORE_F32, g->xdec[l - 1], (long long)Cl * d), s);
    StackRun r;
    r.G = Gl;
    r.q_len = Cl;
    r.kc = g->dk[l - 1];
    r.vc = g->dv[l - 1];
    r.layer_bytes = g->dlayer[l - 1];
    r.cap = Cl;
    run_stack(m, m->i_decl[l - 1], m->Dl[l - 1], g->xdec[l - 1], r, b, s);
    launch_rmsnorm(m->dt, g->xdec[l - 1], (const float*)m->ptr(m->i_decl_g[l - 1]), g->ahat[l - 1], Gl * Cl, d, 1, 0,
                   eps, s);
    src = g->ahat[l - 1];
  }
  // token decoder over each group's C_1 conditioning vectors, then one row per token
  const int G1 = g->G[0];
  gemm(m, b, src, d, m->ptr(m->i_cvl[0]), d, G1, C1 * d, d, epi(EPI_STORE_F32, g->xdec[0], (long long)C1 * d), s);
  StackRun r1;
  r1.G = G1;
  r1.q_len = C1;
  r1.kc = g->dk[0];
  r1.vc = g->dv[0];
  r1.layer_bytes = g->dlayer[0];
  r1.cap = 2 * C1;
  run_stack(m, m->i_decl[0], m->Dl[0], g->xdec[0], r1, b, s);
  SampleArgs sa;
  sa.inv_t = c->samp_inv_t;
  sa.seed = c->samp_seed;
  sa.chunk = g->d_n + PHOTON_MAX_LEVELS;
  sa.C1 = C1;
  sa.C2 = C / C1;
  for (int i = 0; i < C1; ++i) {
    const float* x = i == 0 ? g->xdec[0] : g->xs;
    launch_rmsnorm(m->dt, x, (const float*)m->ptr(m->i_decl_g[0]), g->hn, G1, d, i == 0 ? C1 : 1,
                   i == 0 ? C1 - 1 : 0, eps, s);
    const long long ld = out_logits ? (long long)C1 * V : V;
    float* lg = out_logits ? out_logits + (size_t)i * V : g->logits;
    gemm(m, b, g->hn, d, m->ptr(m->i_head), d, G1, V, d, epi(EPI_STORE_F32, lg, ld), s);
    sa.i = i;
    launch_argmax(lg, ld, G1, V, i, C1, force, out_tokens, g->used, g->next_ids, c->d_err, sa, s);
    if (i + 1 < C1) {
      launch_embed_f32(m->dt, g->next_ids, m->ptr(m->i_embed), g->xs, G1, d, V, c->d_err, s);
      StackRun rs = r1;
      rs.q_len = 1;
      rs.p0 = C1 + i;
      run_stack(m, m->i_decl[0], m->Dl[0], g->xs, rs, b, s);
    }
  }
  launch_advance(g->d_n + PHOTON_MAX_LEVELS, 1, 0, s);  // chunks generated (sampling keys)
  // the top encoder's next input
  const int CL = m->Cl[L - 1];
  const void* top_in;
  if (mode == PHOTON_MODE_REC) {
    top_in = force_a ? force_a : g->ahat[L - 1];
  } else {
    launch_embed(m->dt, g->used, m->ptr(m->i_embed), g->emb, B * C, d, V, c->d_err, s);
    const void* prev = g->emb;
    for (int l = 1; l < L; ++l) {
      const int Cl = m->Cl[l - 1], q = C / gen_prod(m, l), rows = B * q;
      gemm(m, b, prev, (long long)Cl * d, m->ptr(m->i_chl[l - 1]), (long long)Cl * d, rows, d, Cl * d,
           epi(EPI_STORE_F32, g->xre[l - 1], d), s);
      StackRun re;
      re.G = B;
      re.q_len = q;
      re.p0_dev = g->d_n + (l - 1);
      re.n_plan = g->cap[l - 1];
      re.kc = g->kc[l - 1];
      re.vc = g->vc[l - 1];
      re.layer_bytes = g->layer[l - 1];
      re.cap = g->cap[l - 1];
      run_stack(m, m->i_encl[l - 1], m->El[l - 1], g->xre[l - 1], re, b, s);
      launch_rmsnorm(m->dt, g->xre[l - 1], (const float*)m->ptr(m->i_encl_g[l - 1]), g->sre[l - 1], rows, d, 1, 0,
                     eps, s);
      prev = g->sre[l - 1];
    }
    top_in = prev;
  }
  gemm(m, b, top_in, (long long)CL * d, m->ptr(m->i_chl[L - 1]), (long long)CL * d, B, d, CL * d,
       epi(EPI_STORE_F32, g->xt, d), s);
  StackRun rt;
  rt.G = B;
  rt.q_len = 1;
  rt.p0_dev = g->d_n + (L - 1);
  rt.n_plan = g->cap[L - 1];
  rt.kc = g->kc[L - 1];
  rt.vc = g->vc[L - 1];
  rt.layer_bytes = g->layer[L - 1];
  rt.cap = g->cap[L - 1];
  run_stack(m, m->i_encl[L - 1], m->El[L - 1], g->xt, rt, b, s);
  launch_rmsnorm(m->dt, g->xt, (const float*)m->ptr(m->i_encl_g[L - 1]), c->o, B, d, 1, 0, eps, s);
  // positions: the top grows by one entry; in HierGen level l by C / P(l)
  launch_advance(g->d_n + (L - 1), 1, 0, s);
  if (mode == PHOTON_MODE_HIER)
    for (int l = 1; l < L; ++l) launch_advance(g->d_n + (l - 1), C / gen_prod(m, l), 0, s);
}

static int gen_decode_step(photon_model* m, photon_cache* c, int mode, int32_t* d_out_tokens, float* d_out_logits,
                           const int32_t* d_force_tokens, const void* d_force_a, cudaStream_t s) {
  GenCache* g = c->gen;
  const int L = m->NL;
  if (mode == PHOTON_MODE_REC && L < 2) return fail(PHOTON_ERR_ARG, "RecGen needs at least two levels");
  if (mode == PHOTON_MODE_HIER && c->mode != PHOTON_MODE_HIER && L >= 2)
    return fail(PHOTON_ERR_MODE, "HierGen needs the lower encoder caches, discarded by a RecGen prefill");
  if (c->steps >= c->max_new) return fail(PHOTON_ERR_CAPACITY, "cache is full (%d steps)", c->max_new);
  c->stream = s;
  const bool plain = !d_out_logits && !d_force_tokens && !d_force_a;
  bool replay = plain && graphs_enabled() && c->steps >= 1 && !g->graph_failed[mode];
  if (replay && m->ggraph_owner[mode] != c) {
    cudaGraph_t gr = nullptr;
    const unsigned long long n0 = launch_total();
    bool ok = cudaStreamBeginCapture(c->cap, cudaStreamCaptureModeRelaxed) == cudaSuccess;
    if (ok) {
      gen_enqueue(m, c, mode, g->tok_out, nullptr, nullptr, nullptr, c->cap);
      ok = cudaStreamEndCapture(c->cap, &gr) == cudaSuccess && gr;
    }
    const long long captured = (long long)(launch_total() - n0);
    note_launch(-captured);
    m->ggraph_kernels[mode] = ok ? captured : 0;
    if (ok && m->ggraph[mode]) {
      cudaGraphExecUpdateResultInfo info;
      if (cudaGraphExecUpdate(m->ggraph[mode], gr, &info) != cudaSuccess) {
        cudaGetLastError();
        cudaGraphExecDestroy(m->ggraph[mode]);
        m->ggraph[mode] = nullptr;
      }
    }
    if (ok && !m->ggraph[mode]) ok = cudaGraphInstantiate(&m->ggraph[mode], gr, 0) == cudaSuccess;
    if (gr) cudaGraphDestroy(gr);
    if (!ok) {
      cudaGetLastError();
      m->ggraph[mode] = nullptr;
      m->ggraph_owner[mode] = nullptr;
      g->graph_failed[mode] = true;
      replay = false;
    } else {
      m->ggraph_owner[mode] = c;
    }
  }
  if (replay) {
    CK(cudaGraphLaunch(m->ggraph[mode], s));
    note_launch(m->ggraph_kernels[mode]);
    c->graph_steps += 1;
    if (d_out_tokens != g->tok_out)
      CK(cudaMemcpyAsync(d_out_tokens, g->tok_out, (size_t)c->B * m->C * sizeof(int32_t), cudaMemcpyDeviceToDevice,
                         s));
  } else {
    gen_enqueue(m, c, mode, d_out_tokens, d_out_logits, d_force_tokens, d_force_a, s);
  }
  CK(cudaGetLastError());
  g->n[L - 1] += 1;
  if (mode == PHOTON_MODE_HIER)
    for (int l = 1; l < L; ++l) g->n[l - 1] += m->C / gen_prod(m, l);
  c->N = g->n[L - 1];
  c->N1 = (L >= 2 && mode == PHOTON_MODE_HIER) ? g->n[0] : 0;
  if (L >= 2) {
    c->a_hat = g->ahat[L - 1];
    c->ahat_latest = g->ahat[L - 1];
    c->has_a_hat = true;
    if (mode == PHOTON_MODE_HIER) {
      c->a = g->sre[L - 2];
      c->has_a = true;
    }
  }
  c->steps += 1;
  return PHOTON_OK;
}


extern "C" {

int photon_prefill(photon_model* m, const photon_cache* prefix, const int32_t* d_tokens, int32_t B,
                   int32_t T, int32_t mode, int32_t max_new_chunks, void* stream, photon_cache** out) {
  if (m && m->general) {
    g_err.clear();
    if (!out) return fail(PHOTON_ERR_ARG, "out is NULL");
    *out = nullptr;
    if (prefix) return fail(PHOTON_ERR_ARG, "shared prefixes are not supported for this model");
    if (!d_tokens || B <= 0 || T <= 0 || T % m->C) return fail(PHOTON_ERR_ARG, "T must be a positive multiple of C");
    if (mode != PHOTON_MODE_HIER && mode != PHOTON_MODE_REC) return fail(PHOTON_ERR_ARG, "unknown mode %d", mode);
    if (max_new_chunks < 0) return fail(PHOTON_ERR_ARG, "max_new_chunks must be >= 0");
    return gen_prefill(m, d_tokens, B, T, mode, max_new_chunks, (cudaStream_t)stream, out);
  }
  return prefill_impl(m, prefix, d_tokens, B, T, mode, max_new_chunks, stream, out, nullptr);
}

int photon_prefill_shell(photon_model* m, const photon_cache* prefix, int32_t B, int32_t T, int32_t mode,
                         int32_t max_new_chunks, void* stream, photon_cache** out) {
  if (m && m->general) {
    g_err.clear();
    if (out) *out = nullptr;
    return fail(PHOTON_ERR_ARG, "shell caches are built for two-level models only");
  }
  return prefill_impl(m, prefix, nullptr, B, T, mode, max_new_chunks, stream, out, nullptr, true);
}

int photon_model_set_kv_pages(photon_model* m, int32_t page_rows, int32_t pool_pages) {
  g_err.clear();
  if (!m) return fail(PHOTON_ERR_ARG, "model is NULL");
  if (m->general || m->vanilla) return fail(PHOTON_ERR_ARG, "paged top KV is built for two-level models only");
  if (page_rows < 0 || pool_pages < 0 || (page_rows == 0) != (pool_pages == 0))
    return fail(PHOTON_ERR_ARG, "page_rows and pool_pages must both be positive (or both 0 to drop the pool)");
  if (m->kv_paged_caches) return fail(PHOTON_ERR_ARG, "%d paged caches still hold pages", m->kv_paged_caches);
  const size_t page = (size_t)m->H * page_rows * m->dh * m->es;
  const size_t total = (size_t)m->Ltop * 2 * (size_t)pool_pages * page;
  if (pool_pages > 0 && total / pool_pages / 2 / m->Ltop != page) return fail(PHOTON_ERR_ARG, "pool size overflows");
  // pages released by freed caches: their work has to finish before the arrays go
  for (auto& p : m->kv_pending) {
    cudaEventSynchronize(p.first);
    cudaEventDestroy(p.first);
  }
  m->kv_pending.clear();
  m->kv_free.clear();
  char* old_pool = m->kv_pool;
  m->kv_pool = nullptr;
  m->kv_page_rows = m->kv_pool_pages = 0;
  if (old_pool) CK(cudaFree(old_pool));
  if (pool_pages == 0) return PHOTON_OK;
  if (cudaMalloc(&m->kv_pool, total) != cudaSuccess) {
    cudaGetLastError();
    m->kv_pool = nullptr;
    return fail(PHOTON_ERR_OOM, "KV page pool of %zu bytes does not fit", total);
  }
  m->kv_page_rows = page_rows;
  m->kv_pool_pages = pool_pages;
  m->kv_free.resize(pool_pages);
  for (int i = 0; i < pool_pages; ++i) m->kv_free[i] = pool_pages - 1 - i;  // taken from the back: 0, 1, ...
  return PHOTON_OK;
}

int photon_prefill_paged(photon_model* m, const photon_cache* prefix, const int32_t* d_tokens, int32_t B,
                         int32_t T, int32_t mode, int32_t max_new_chunks, void* stream, photon_cache** out) {
  g_err.clear();
  if (out) *out = nullptr;
  if (!m) return fail(PHOTON_ERR_ARG, "model is NULL");
  if (m->general || m->vanilla) return fail(PHOTON_ERR_ARG, "paged top KV is built for two-level models only");
  if (!m->kv_pool) return fail(PHOTON_ERR_ARG, "the model has no KV page pool (photon_model_set_kv_pages)");
  return prefill_impl(m, prefix, d_tokens, B, T, mode, max_new_chunks, stream, out, nullptr, false, true);
}

int photon_cache_state_buffer(photon_cache* c, int32_t which, void** d_ptr, size_t* bytes) {
  g_err.clear();
  if (!c || !d_ptr || !bytes) return fail(PHOTON_ERR_ARG, "NULL cache or output pointer");
  photon_model* m = c->m;
  if (m->general) return fail(PHOTON_ERR_ARG, "state buffers are listed for two-level models only");
  *d_ptr = nullptr;
  *bytes = 0;
  switch (which) {
    case PHOTON_STATE_TOP_K:
    case PHOTON_STATE_TOP_V:
      if (c->paged) return fail(PHOTON_ERR_ARG, "a paged cache's top KV is not one buffer");
      *d_ptr = which == PHOTON_STATE_TOP_K ? c->top_k : c->top_v;
      *bytes = c->top_layer * m->Ltop;
      break;
    case PHOTON_STATE_L1_K:
    case PHOTON_STATE_L1_V:
      if (c->l1_k) {
        *d_ptr = which == PHOTON_STATE_L1_K ? c->l1_k : c->l1_v;
        *bytes = c->l1_layer * m->L1;
      }
      break;
    case PHOTON_STATE_PENDING_O:
      *d_ptr = c->o;
      *bytes = (size_t)c->B * m->d * m->es;
      break;
    default:
      return fail(PHOTON_ERR_ARG, "state %d is not a prefill state buffer", which);
  }
  return PHOTON_OK;
}

int photon_decode_step_ex(photon_model* m, photon_cache* c, int32_t mode, int32_t* d_out_tokens,
                          float* d_out_logits, const int32_t* d_force_tokens,
                          const void* d_force_a, void* stream) {
  g_err.clear();
  if (!m || !c || c->m != m) return fail(PHOTON_ERR_ARG, "model/cache mismatch");
  if (!d_out_tokens) return fail(PHOTON_ERR_ARG, "output token buffer is NULL");
  if (mode != PHOTON_MODE_HIER && mode != PHOTON_MODE_REC) return fail(PHOTON_ERR_ARG, "unknown mode %d", mode);
  if (m->general) return gen_decode_step(m, c, mode, d_out_tokens, d_out_logits, d_force_tokens, d_force_a,
                                         (cudaStream_t)stream);
  if (mode == PHOTON_MODE_HIER && (c->mode != PHOTON_MODE_HIER || !c->l1_k))
    return fail(PHOTON_ERR_MODE, "HierGen needs the level-1 KV, discarded by a RecGen prefill");
  if (c->steps >= c->max_new) return fail(PHOTON_ERR_CAPACITY, "cache is full (%d steps)", c->max_new);
  if (mode == PHOTON_MODE_HIER && !m->group_ptr[G_ENC1]) RET(ensure_encoder(m, (cudaStream_t)stream));
  cudaStream_t s = (cudaStream_t)stream;
  c->stream = s;
  if (c->paged) RET(kv_map_through(c, c->N - c->n_pre, s));  // the top slot this step appends
  const int C2 = m->C2;
  // The plain step (no hooks, no logits) is captured once per mode, after
  // one eager step has configured every kernel, and replayed afterwards.
  // Capture runs on the cache's own stream (capturing executes nothing), so
  // the caller's stream may be any stream, the legacy default one included;
  // the graph is launched on the caller's stream.
  const bool plain = !d_out_logits && !d_force_tokens && !d_force_a;
  bool replay = plain && c->cap != nullptr && graphs_enabled() && c->steps >= 1 && !c->graph_failed[mode];
  if (replay && m->graph_owner[mode] != c) {
    // capture this cache's step; update the model's executable in place when
    // the topology matches, otherwise instantiate a new one
    cudaGraph_t g = nullptr;
    // the launch counter counts kernels that run: captured launches are
    // taken back here and added again at every replay
    const unsigned long long n0 = launch_total();
    bool ok = cudaStreamBeginCapture(c->cap, cudaStreamCaptureModeRelaxed) == cudaSuccess;
    if (ok) {
      enqueue_decode(m, c, mode, c->tok_out, nullptr, nullptr, nullptr, c->cap);
      ok = cudaStreamEndCapture(c->cap, &g) == cudaSuccess && g;
    }
    const long long captured = (long long)(launch_total() - n0);
    note_launch(-captured);
    m->graph_kernels[mode] = ok ? captured : 0;
    if (ok && m->graph[mode]) {
      cudaGraphExecUpdateResultInfo info;
      if (cudaGraphExecUpdate(m->graph[mode], g, &info) != cudaSuccess) {
        cudaGetLastError();
        cudaGraphExecDestroy(m->graph[mode]);
        m->graph[mode] = nullptr;
      }
    }
    if (ok && !m->graph[mode]) ok = cudaGraphInstantiate(&m->graph[mode], g, 0) == cudaSuccess;
    if (g) cudaGraphDestroy(g);
    if (!ok) {
      cudaGetLastError();
      m->graph[mode] = nullptr;
      m->graph_owner[mode] = nullptr;
      c->graph_failed[mode] = true;
      replay = false;
    } else {
      m->graph_owner[mode] = c;
    }
  }
  if (replay) {
    CK(cudaGraphLaunch(m->graph[mode], s));
    note_launch(m->graph_kernels[mode]);
    c->graph_steps += 1;
    if (d_out_tokens != c->tok_out)
      CK(cudaMemcpyAsync(d_out_tokens, c->tok_out, (size_t)c->B * m->C * sizeof(int32_t),
                         cudaMemcpyDeviceToDevice, s));
  } else {
    enqueue_decode(m, c, mode, d_out_tokens, d_out_logits, d_force_tokens, d_force_a, s);
  }
  CK(cudaGetLastError());
  if (mode == PHOTON_MODE_HIER) RET(note_encoder_use(m, s));
  c->N += 1;
  if (mode == PHOTON_MODE_HIER) {
    c->N1 += C2;
    c->has_a = true;
  }
  c->has_a_hat = true;
  c->ahat_latest = c->a_hat;
  c->steps += 1;
  return PHOTON_OK;
}

// ------------------------------------------------------------------ pipelined RecGen
static bool pipeline_enabled() {
  static const bool on = [] {
    const char* e = getenv("PHOTON_RECGEN_PIPELINE");
    return !(e && e[0] == '0');
  }();
  return on;
}

// Token-branch buffers, double-buffered A-hat, stream and events of the
// pipelined RecGen path (allocated on the first call, counted as cache memory).
static int prepare_pipeline(photon_model* m, photon_cache* c, cudaStream_t s) {
  if (c->pipe_ready) return PHOTON_OK;
  const int B = c->B, d = m->d, C = m->C, rows_c = B * C, rows_g = B * m->C2;
  const size_t es = m->es;
  Allocator al{s, &c->allocs, &c->kv_bytes};
  c->ahat_p[0] = al.get<void>((size_t)rows_g * d * es);
  c->ahat_p[1] = al.get<void>((size_t)rows_g * d * es);
  c->xd_k = al.get<float>((size_t)rows_c * d * 4);
  c->xn_k = al.get<void>((size_t)rows_c * d * es);
  c->q_k = al.get<void>((size_t)rows_c * d * es);
  c->att_k = al.get<void>((size_t)rows_c * d * es);
  c->hid_k = al.get<void>((size_t)rows_c * m->f * es);
  c->gemm_ws_k = al.get<float>(c->gemm_ws_bytes);
  c->attn_ws_k = al.get<float>(c->attn_ws_bytes);
  c->gemm_cnt_k = al.get<int>(kGemmTileCounters * sizeof(int));
  if (c->sn_x) {
    c->sn_x_k = al.get<void>((size_t)c->sn_rows * d * es);
    c->sn_ss_k = al.get<float>((size_t)c->sn_rows * kSsqCap * sizeof(float));
  }
  if (al.err != cudaSuccess) return fail(PHOTON_ERR_OOM, "device allocation failed (pipelined decode buffers)");
  CK(cudaMemsetAsync(c->gemm_cnt_k, 0, kGemmTileCounters * sizeof(int), s));
  if (!c->tstream) {
    CK(cudaStreamCreateWithFlags(&c->tstream, cudaStreamNonBlocking));
    for (int p = 0; p < 2; ++p) {
      CK(cudaEventCreateWithFlags(&c->ev_main[p], cudaEventDisableTiming));
      CK(cudaEventCreateWithFlags(&c->ev_tok[p], cudaEventDisableTiming));
    }
  }
  c->pipe_ready = true;
  return PHOTON_OK;
}

// Captures one half of a pipelined step (part DEC_MAIN or DEC_TOK, A-hat
// buffer `parity`) on the cache's capture stream; the launch counter keeps
// counting kernels that run (taken back here, added at every launch).
static bool capture_part(photon_model* m, photon_cache* c, int part, int parity, cudaGraphExec_t* exec,
                         long long* kernels) {
  cudaGraph_t g = nullptr;
  const unsigned long long n0 = launch_total();
  bool ok = cudaStreamBeginCapture(c->cap, cudaStreamCaptureModeRelaxed) == cudaSuccess;
  if (ok) {
    enqueue_decode(m, c, PHOTON_MODE_REC, c->tok_out, nullptr, nullptr, nullptr, c->cap, part, parity);
    ok = cudaStreamEndCapture(c->cap, &g) == cudaSuccess && g;
  }
  const long long captured = (long long)(launch_total() - n0);
  note_launch(-captured);
  if (ok && *exec) {  // same topology for every cache of this model: update in place
    cudaGraphExecUpdateResultInfo info;
    if (cudaGraphExecUpdate(*exec, g, &info) != cudaSuccess) {
      cudaGetLastError();
      cudaGraphExecDestroy(*exec);
      *exec = nullptr;
    }
  }
  if (ok && !*exec) ok = cudaGraphInstantiate(exec, g, 0) == cudaSuccess;
  if (g) cudaGraphDestroy(g);
  if (!ok) {
    cudaGetLastError();
    if (*exec) cudaGraphExecDestroy(*exec);
    *exec = nullptr;
    return false;
  }
  *kernels = captured;
  return true;
}

int photon_decode_rec_chunks(photon_model* m, photon_cache* c, int32_t n, int32_t* d_out_tokens,
                             void* stream) {
  g_err.clear();
  if (!m || !c || c->m != m) return fail(PHOTON_ERR_ARG, "model/cache mismatch");
  if (n < 0 || (n > 0 && !d_out_tokens)) return fail(PHOTON_ERR_ARG, "bad chunk count or output");
  if (n == 0) return PHOTON_OK;
  if (c->steps + n > c->max_new) return fail(PHOTON_ERR_CAPACITY, "cache is full (%d steps)", c->max_new);
  cudaStream_t s = (cudaStream_t)stream;
  c->stream = s;
  if (c->paged) RET(kv_map_through(c, c->N - c->n_pre + n - 1, s));  // the top slots of all n chunks
  const int B = c->B, C = m->C;
  const size_t pitch = (size_t)n * C * sizeof(int32_t), w = (size_t)C * sizeof(int32_t);
  int t = 0;
  // the first step of a cache runs eagerly (it configures every kernel)
  auto one_step = [&](int k) -> int {
    RET(photon_decode_step_ex(m, c, PHOTON_MODE_REC, c->tok_out, nullptr, nullptr, nullptr, stream));
    CK(cudaMemcpy2DAsync(d_out_tokens + (size_t)k * C, pitch, c->tok_out, w, w, B,
                         cudaMemcpyDeviceToDevice, s));
    return PHOTON_OK;
  };
  if (m->general) {  // any-L models: one (graph-replayed) step per chunk
    for (int k = 0; k < n; ++k) {
      RET(photon_decode_step_ex(m, c, PHOTON_MODE_REC, c->gen_tok_out(), nullptr, nullptr, nullptr, stream));
      CK(cudaMemcpy2DAsync(d_out_tokens + (size_t)k * C, pitch, c->gen_tok_out(), w, w, B, cudaMemcpyDeviceToDevice,
                           s));
    }
    return PHOTON_OK;
  }
  if (c->steps == 0) {
    RET(one_step(0));
    t = 1;
  }
  bool pipe = pipeline_enabled() && graphs_enabled() && c->cap != nullptr && t < n;
  if (pipe) RET(prepare_pipeline(m, c, s));
  if (pipe && m->pg_owner != c) {
    for (int p = 0; p < 2 && pipe; ++p)
      pipe = capture_part(m, c, DEC_MAIN, p, &m->pg[0][p], &m->pg_kernels[0]) &&
             capture_part(m, c, DEC_TOK, p, &m->pg[1][p], &m->pg_kernels[1]);
    m->pg_owner = pipe ? c : nullptr;
  }
  if (!pipe) {
    for (; t < n; ++t) RET(one_step(t));
    return PHOTON_OK;
  }
  // main chain of chunk k on the caller's stream; token branch of chunk k on
  // the token stream, overlapping the main chain of chunk k + 1
  int last = 0;
  for (; t < n; ++t) {
    const int p = c->steps & 1;
    CK(cudaStreamWaitEvent(s, c->ev_tok[p], 0));  // token branch of two chunks ago released A-hat[p]
    CK(cudaGraphLaunch(m->pg[0][p], s));
    note_launch(m->pg_kernels[0]);
    CK(cudaEventRecord(c->ev_main[p], s));
    CK(cudaStreamWaitEvent(c->tstream, c->ev_main[p], 0));
    CK(cudaGraphLaunch(m->pg[1][p], c->tstream));
    note_launch(m->pg_kernels[1]);
    CK(cudaMemcpy2DAsync(d_out_tokens + (size_t)t * C, pitch, c->tok_out, w, w, B,
                         cudaMemcpyDeviceToDevice, c->tstream));
    CK(cudaEventRecord(c->ev_tok[p], c->tstream));
    c->N += 1;
    c->steps += 1;
    c->graph_steps += 1;
    c->has_a_hat = true;
    c->ahat_latest = c->ahat_p[p];
    last = p;
  }
  CK(cudaStreamWaitEvent(s, c->ev_tok[last], 0));  // everything joins the caller's stream
  return PHOTON_OK;
}

int photon_decode_step_hier(photon_model* m, photon_cache* c, int32_t* d_out_tokens,
                            float* d_out_logits, void* stream) {
  return photon_decode_step_ex(m, c, PHOTON_MODE_HIER, d_out_tokens, d_out_logits, nullptr, nullptr,
                               stream);
}

int photon_decode_step_rec(photon_model* m, photon_cache* c, int32_t* d_out_tokens,
                           float* d_out_logits, void* stream) {
  return photon_decode_step_ex(m, c, PHOTON_MODE_REC, d_out_tokens, d_out_logits, nullptr, nullptr,
                               stream);
}

int photon_free_cache(photon_cache* c) {
  g_err.clear();
  if (!c) return fail(PHOTON_ERR_ARG, "cache is NULL");
  if (c->dependents) return fail(PHOTON_ERR_ARG, "%d caches still read this prefix", c->dependents);
  photon_model* m = c->m;
  for (int k = 0; k < 2; ++k) {
    if (m->graph_owner[k] == c) m->graph_owner[k] = nullptr;  // its buffers are going away
    if (m->ggraph_owner[k] == c) m->ggraph_owner[k] = nullptr;
  }
  if (m->pg_owner == c) m->pg_owner = nullptr;
  // Stream-ordered release: the helper streams' pending work is joined into
  // the cache's stream, the buffers go back to the pool on that stream, and
  // streams and events are destroyed at once (the driver releases them when
  // their work completes).  The next allocation on the same stream reuses the
  // memory without waiting on the host.
  cudaStream_t helpers[3] = {c->side, c->tstream, c->hi};
  for (cudaStream_t h : helpers) {
    if (!h) continue;
    cudaEvent_t e = nullptr;
    CK(cudaEventCreateWithFlags(&e, cudaEventDisableTiming));
    CK(cudaEventRecord(e, h));
    CK(cudaStreamWaitEvent(c->stream, e, 0));
    cudaEventDestroy(e);
  }
  for (cudaStream_t h : helpers)
    if (h) cudaStreamDestroy(h);
  if (c->cap) cudaStreamDestroy(c->cap);  // only ever captured into, never run
  for (int p = 0; p < 2; ++p) {
    if (c->ev_main[p]) cudaEventDestroy(c->ev_main[p]);
    if (c->ev_tok[p]) cudaEventDestroy(c->ev_tok[p]);
  }
  if (c->ev_fork) cudaEventDestroy(c->ev_fork);
  if (c->ev_join_hi) cudaEventDestroy(c->ev_join_hi);
  if (c->ev_join) cudaEventDestroy(c->ev_join);
  if (c->paged) {  // pages come back once the work queued so far has finished
    kv_release(m, c, c->stream);
    m->kv_paged_caches--;
  }
  free_list(c->allocs, c->stream);
  // a cache built on a prefix may run on another stream than the prefix's
  // eventual free: finish its work before the prefix can be released
  if (c->prefix) {
    CK(cudaStreamSynchronize(c->stream));
    c->prefix->dependents--;
  }
  CK(cudaGetLastError());
  m->live_caches--;
  if (c->mode == PHOTON_MODE_HIER) m->hier_caches--;
  for (auto& e : c->tk_plans) top_step_free(e.plan);  // host-side launch descriptions only
  delete c->gen;
  delete c;
  return PHOTON_OK;
}

int photon_cache_set_sampling(photon_cache* c, float temperature, uint64_t seed) {
  g_err.clear();
  if (!c) return fail(PHOTON_ERR_ARG, "cache is NULL");
  if (!(temperature >= 0.f) || !std::isfinite(temperature))
    return fail(PHOTON_ERR_ARG, "temperature must be finite and >= 0");
  if (temperature > 0.f && !std::isfinite(1.0f / temperature))
    return fail(PHOTON_ERR_ARG, "temperature %g is too small", (double)temperature);
  c->samp_inv_t = temperature > 0.f ? 1.0f / temperature : 0.f;
  c->samp_seed = seed;
  // captured steps carry the old parameters: capture again on the next step
  photon_model* m = c->m;
  for (int k = 0; k < 2; ++k) {
    if (m->graph_owner[k] == c) m->graph_owner[k] = nullptr;
    if (m->ggraph_owner[k] == c) m->ggraph_owner[k] = nullptr;
  }
  if (m->pg_owner == c) m->pg_owner = nullptr;
  return PHOTON_OK;
}

int photon_cache_set_top_p(photon_cache* c, float top_p) {
  g_err.clear();
  if (!c) return fail(PHOTON_ERR_ARG, "cache is NULL");
  if (!(top_p > 0.f && top_p <= 1.f)) return fail(PHOTON_ERR_ARG, "top_p must be in (0, 1]");
  c->samp_top_p = top_p;
  photon_model* m = c->m;
  for (int k = 0; k < 2; ++k)
    if (m->graph_owner[k] == c) m->graph_owner[k] = nullptr;
  if (m->pg_owner == c) m->pg_owner = nullptr;
  return PHOTON_OK;
}

int photon_sample_logits(const float* d_logits, int32_t rows, int32_t V, float temperature, float top_p,
                         uint64_t seed, const int32_t* d_chunk, int32_t C1, int32_t C2, int32_t i,
                         int32_t* d_out, void* stream) {
  g_err.clear();
  if (!d_logits || !d_chunk || !d_out) return fail(PHOTON_ERR_ARG, "NULL buffer");
  if (rows <= 0 || V <= 0 || C1 <= 0 || C2 <= 0 || i < 0 || i >= C1) return fail(PHOTON_ERR_ARG, "bad shape");
  if (!(temperature > 0.f) || !std::isfinite(1.0f / temperature) || !(top_p > 0.f && top_p <= 1.f))
    return fail(PHOTON_ERR_ARG, "need temperature > 0 and top_p in (0, 1]");
  SampleArgs sa;
  sa.inv_t = 1.0f / temperature;
  sa.seed = seed;
  sa.chunk = d_chunk;
  sa.C1 = C1;
  sa.C2 = C2;
  sa.i = i;
  launch_sample_topp(d_logits, V, rows, V, 0, 1, sa, top_p, nullptr, d_out, nullptr, nullptr, nullptr,
                     (cudaStream_t)stream);
  CK(cudaGetLastError());
  return PHOTON_OK;
}

int photon_cache_info(photon_cache* c, photon_cache_stats* out) {
  g_err.clear();
  if (!c || !out) return fail(PHOTON_ERR_ARG, "NULL argument");
  memset(out, 0, sizeof(*out));
  CK(cudaStreamSynchronize(c->stream));
  int err = 0;
  CK(cudaMemcpy(&err, c->d_err, sizeof(int), cudaMemcpyDeviceToHost));
  out->B = c->B;
  out->T = c->T;
  out->mode = c->mode;
  out->N = c->N;
  out->N1 = c->N1;
  out->n_prefix = c->n_pre;
  out->n1_prefix = c->n1_pre;
  out->capacity = c->Ncap;
  out->steps = c->steps;
  out->max_new_chunks = c->max_new;
  out->device_error = err;
  out->l1_resident = c->l1_k != nullptr;
  out->kv_bytes = c->kv_bytes;
  out->workspace_bytes = c->ws_bytes;
  out->graph_steps = c->graph_steps;
  out->graph_kernels = c->gen ? (int32_t)std::max(c->m->ggraph_owner[0] == c ? c->m->ggraph_kernels[0] : 0,
                                                 c->m->ggraph_owner[1] == c ? c->m->ggraph_kernels[1] : 0)
                       : (c->mode >= 0 && c->mode < 2 && c->m->graph_owner[c->mode] == c)
                           ? (int32_t)c->m->graph_kernels[c->mode]
                           : c->m->pg_owner == c ? (int32_t)(c->m->pg_kernels[0] + c->m->pg_kernels[1]) : 0;
  return PHOTON_OK;
}

int photon_export_state(photon_cache* c, int32_t which, int32_t layer, void* d_dst, size_t dst_bytes,
                        size_t* out_bytes, void* stream) {
  g_err.clear();
  if (!c) return fail(PHOTON_ERR_ARG, "cache is NULL");
  photon_model* m = c->m;
  cudaStream_t s = (cudaStream_t)stream;
  const size_t es = m->es, hd = (size_t)m->H * m->dh;
  const char* src = nullptr;
  size_t rows = 0, width = 0, pitch = 0;
  switch (which) {
    case PHOTON_STATE_TOP_K:
    case PHOTON_STATE_TOP_V: {
      if (layer < 0 || layer >= m->Ltop) return fail(PHOTON_ERR_ARG, "layer out of range");
      const int n = c->N - c->n_pre;
      src = (which == PHOTON_STATE_TOP_K ? c->top_k : c->top_v) + layer * c->top_layer;
      if (c->paged) {  // gathered page by page into [B][H][n][dh]
        const size_t row = (size_t)m->dh * es, P = (size_t)m->kv_page_rows, bytes = (size_t)c->B * m->H * n * row;
        if (out_bytes) *out_bytes = bytes;
        if (!d_dst || bytes == 0) return PHOTON_OK;
        if (dst_bytes < bytes) return fail(PHOTON_ERR_ARG, "destination holds %zu bytes, need %zu", dst_bytes, bytes);
        for (int b = 0; b < c->B; ++b)
          for (int lp = 0; (size_t)lp * P < (size_t)n; ++lp) {
            const int phys = c->kv_table_host[(size_t)b * c->kv_tab_len + lp];
            const size_t r = std::min(P, (size_t)n - lp * P);
            CK(cudaMemcpy2DAsync((char*)d_dst + ((size_t)b * m->H * n + lp * P) * row, (size_t)n * row,
                                 src + (size_t)phys * m->H * P * row, P * row, r * row, m->H,
                                 cudaMemcpyDeviceToDevice, s));
          }
        return PHOTON_OK;
      }
      rows = (size_t)c->B * m->H;
      width = (size_t)n * m->dh * es;
      pitch = (size_t)c->Ncap * m->dh * es;
      break;
    }
    case PHOTON_STATE_L1_K:
    case PHOTON_STATE_L1_V: {
      if (!c->l1_k) return fail(PHOTON_ERR_ARG, "level-1 KV was discarded (RecGen cache)");
      if (layer < 0 || layer >= m->L1) return fail(PHOTON_ERR_ARG, "layer out of range");
      const int n = c->N1 - c->n1_pre;
      src = (which == PHOTON_STATE_L1_K ? c->l1_k : c->l1_v) + layer * c->l1_layer;
      rows = (size_t)c->B * m->H;
      width = (size_t)n * m->dh * es;
      pitch = (size_t)c->N1cap * m->dh * es;
      break;
    }
    case PHOTON_STATE_PENDING_O:
      src = (const char*)c->o;
      rows = 1;
      width = pitch = (size_t)c->B * m->d * es;
      break;
    case PHOTON_STATE_A_HAT:
    case PHOTON_STATE_A:
      if (which == PHOTON_STATE_A_HAT ? !c->has_a_hat : !c->has_a)
        return fail(PHOTON_ERR_ARG, "no decode step has produced this state yet");
      src = (const char*)(which == PHOTON_STATE_A_HAT ? (c->ahat_latest ? c->ahat_latest : c->a_hat) : c->a);
      rows = 1;
      width = pitch = (size_t)c->B * m->C2 * m->d * es;
      break;
    default:
      return fail(PHOTON_ERR_ARG, "unknown state %d", which);
  }
  (void)hd;
  const size_t bytes = rows * width;
  if (out_bytes) *out_bytes = bytes;
  if (!d_dst || bytes == 0) return PHOTON_OK;
  if (dst_bytes < bytes) return fail(PHOTON_ERR_ARG, "destination holds %zu bytes, need %zu", dst_bytes, bytes);
  CK(cudaMemcpy2DAsync(d_dst, width, src, pitch, width, rows, cudaMemcpyDeviceToDevice, s));
  return PHOTON_OK;
}

int photon_gemm(int32_t dtype, const void* d_A, int64_t lda, const void* d_W, int64_t ldw, int32_t M,
                int32_t N, int32_t K, float* d_C, int64_t ldc, int32_t path, int32_t splits,
                int32_t swap, void* stream) {
  g_err.clear();
  if (dtype != 0 && dtype != 1) return fail(PHOTON_ERR_ARG, "dtype must be 0 or 1");
  if (!d_A || !d_W || !d_C || M <= 0 || N <= 0 || K <= 0) return fail(PHOTON_ERR_ARG, "bad GEMM arguments");
  cudaStream_t s = (cudaStream_t)stream;
  GemmArgs g;
  g.A = d_A;
  g.lda = lda;
  g.W = d_W;
  g.ldw = ldw;
  g.M = M;
  g.N = N;
  g.K = K;
  g.ep = epi(EPI_STORE_F32, d_C, ldc);
  if (path == 1) {
    launch_gemm_simt(dtype, g, s);
    CK(cudaGetLastError());
    return PHOTON_OK;
  }
  if (dtype != DT_BF16 || !tma_available()) {
    if (path == 2) return fail(PHOTON_ERR_ARG, "the tcgen05 path needs bf16 and TMA");
    launch_gemm_simt(dtype, g, s);
    CK(cudaGetLastError());
    return PHOTON_OK;
  }
  // split-K scratch only when the plan needs it (partials + zeroed tile counters)
  const size_t wsb = gemm_tc_workspace_bytes(M, N, K, splits > 0 ? splits : 0, swap);
  float* ws = nullptr;
  int* cnt = nullptr;
  if (wsb) {
    CK(pool_malloc((void**)&ws, wsb, s));
    CK(pool_malloc((void**)&cnt, kGemmTileCounters * sizeof(int), s));
    CK(cudaMemsetAsync(cnt, 0, kGemmTileCounters * sizeof(int), s));
  }
  GemmWorkspace w{ws, wsb, cnt, kGemmTileCounters};
  int* err = nullptr;
  bool ok = launch_gemm_tc(g, w, err, s, splits > 0 ? splits : 0, swap);
  if (!ok && path == 0) {
    launch_gemm_simt(dtype, g, s);
    ok = true;
  }
  if (ws) cudaFreeAsync(ws, s);
  if (cnt) cudaFreeAsync(cnt, s);
  if (!ok) return fail(PHOTON_ERR_ARG, "shape not supported by the tcgen05 kernel");
  CK(cudaGetLastError());
  return PHOTON_OK;
}

int photon_gemm_rmsnorm(const float* d_x, int64_t ldx, const float* d_g, float eps, const void* d_W,
                        int64_t ldw, int32_t M, int32_t N, int32_t K, float* d_C, int64_t ldc,
                        void* stream) {
  g_err.clear();
  if (!d_x || !d_g || !d_W || !d_C || M <= 0 || N <= 0 || K <= 0 || ldx < K || ldw < K || ldc < N ||
      !(eps >= 0.f))
    return fail(PHOTON_ERR_ARG, "bad GEMM arguments");
  if (ldx % 4 || reinterpret_cast<uintptr_t>(d_x) % 16 || reinterpret_cast<uintptr_t>(d_g) % 16)
    return fail(PHOTON_ERR_ARG, "x rows and g must be 16-byte aligned");
  cudaStream_t s = (cudaStream_t)stream;
  GemmArgs g;
  g.W = d_W;
  g.ldw = ldw;
  g.M = M;
  g.N = N;
  g.K = K;
  g.ep = epi(EPI_STORE_F32, d_C, ldc);
  if (tma_available() && gemm_tc_fuses_norm(M, N, K)) {
    g.norm_x = d_x;
    g.norm_ld = ldx;
    g.norm_g = d_g;
    g.norm_eps = eps;
    GemmWorkspace w{nullptr, 0, nullptr, 0};
    if (!launch_gemm_tc(g, w, nullptr, s)) return fail(PHOTON_ERR_ARG, "fused RMSNorm GEMM rejected the shape");
    CK(cudaGetLastError());
    return PHOTON_OK;
  }
  // separate norm into a bf16 copy, then the library's GEMM (the norm
  // kernel reads rows with stride K)
  if (ldx != K) return fail(PHOTON_ERR_ARG, "this shape takes the unfused path, which needs ldx == K");
  void* xn = nullptr;
  CK(pool_malloc(&xn, (size_t)M * K * 2, s));
  launch_rmsnorm(DT_BF16, d_x, d_g, xn, M, K, 1, 0, eps, s);
  g.A = xn;
  g.lda = K;
  const size_t wsb = gemm_tc_workspace_bytes(M, N, K);
  float* ws = nullptr;
  int* cnt = nullptr;
  if (wsb) {
    CK(pool_malloc((void**)&ws, wsb, s));
    CK(pool_malloc((void**)&cnt, kGemmTileCounters * sizeof(int), s));
    CK(cudaMemsetAsync(cnt, 0, kGemmTileCounters * sizeof(int), s));
  }
  GemmWorkspace w{ws, wsb, cnt, kGemmTileCounters};
  launch_gemm(DT_BF16, g, w, nullptr, s);
  if (ws) cudaFreeAsync(ws, s);
  if (cnt) cudaFreeAsync(cnt, s);
  cudaFreeAsync(xn, s);
  CK(cudaGetLastError());
  return PHOTON_OK;
}

int photon_attn_decode_scratch_bytes(int32_t dtype, int32_t G, int32_t H, int32_t head_dim, int32_t cap,
                                     int32_t q_len, int32_t p0, uint64_t* out_bytes) {
  g_err.clear();
  if (!out_bytes) return fail(PHOTON_ERR_ARG, "out_bytes is NULL");
  if (dtype != 0 && dtype != 1) return fail(PHOTON_ERR_ARG, "dtype must be 0 or 1");
  if (G <= 0 || H <= 0 || (head_dim != 32 && head_dim != 64)) return fail(PHOTON_ERR_ARG, "bad shape");
  if (q_len < 1 || q_len > 4 || p0 < 0 || p0 + q_len > cap) return fail(PHOTON_ERR_ARG, "bad q_len/p0/cap");
  AttnArgs a;
  a.q_ld = (long long)H * head_dim;
  a.o_ld = a.q_ld;
  a.cap = cap;
  a.G = G;
  a.H = H;
  a.dh = head_dim;
  a.q_len = q_len;
  a.p0 = p0;
  *out_bytes = attn_decode_workspace_bytes(dtype, a);
  return PHOTON_OK;
}

int photon_attn_decode(int32_t dtype, const void* d_q, const void* d_k, const void* d_v, int32_t G,
                       int32_t H, int32_t head_dim, int32_t cap, int32_t q_len, int32_t p0, void* d_o,
                       int32_t* d_err, void* stream) {
  g_err.clear();
  if (dtype != 0 && dtype != 1) return fail(PHOTON_ERR_ARG, "dtype must be 0 or 1");
  if (!d_q || !d_k || !d_v || !d_o) return fail(PHOTON_ERR_ARG, "NULL buffer");
  if (G <= 0 || H <= 0 || (head_dim != 32 && head_dim != 64)) return fail(PHOTON_ERR_ARG, "bad shape");
  if (q_len < 1 || q_len > 4 || p0 < 0 || p0 + q_len > cap) return fail(PHOTON_ERR_ARG, "bad q_len/p0/cap");
  cudaStream_t s = (cudaStream_t)stream;
  AttnArgs a;
  a.Q = d_q;
  a.q_ld = (long long)H * head_dim;
  a.K = d_k;
  a.V = d_v;
  a.cap = cap;
  a.G = G;
  a.H = H;
  a.dh = head_dim;
  a.q_len = q_len;
  a.p0 = p0;
  a.O = d_o;
  a.o_ld = (long long)H * head_dim;
  a.scale = 1.0f / sqrtf((float)head_dim);
  const size_t wsb = attn_decode_workspace_bytes(dtype, a);
  float* ws = nullptr;
  if (wsb) CK(pool_malloc((void**)&ws, wsb, s));
  const bool ok = launch_attn_decode(dtype, a, ws, wsb, d_err, s);
  if (ws) cudaFreeAsync(ws, s);
  if (!ok) return fail(PHOTON_ERR_ARG, "decode attention rejected the shape");
  CK(cudaGetLastError());
  return PHOTON_OK;
}

int photon_attn_prefill(int32_t dtype, const void* d_q, const void* d_k, const void* d_v, const void* d_kp,
                        const void* d_vp, int32_t G, int32_t H, int32_t head_dim, int32_t cap, int32_t q_len,
                        int32_t p0, int32_t cap_pre, int32_t n_pre, int32_t path, void* d_o, int32_t* d_err,
                        void* stream) {
  g_err.clear();
  if (dtype != 0 && dtype != 1) return fail(PHOTON_ERR_ARG, "dtype must be 0 or 1");
  if (!d_q || !d_k || !d_v || !d_o) return fail(PHOTON_ERR_ARG, "NULL buffer");
  if (G <= 0 || H <= 0 || (head_dim != 32 && head_dim != 64)) return fail(PHOTON_ERR_ARG, "bad shape");
  if (q_len < 1 || n_pre < 0 || p0 < n_pre || p0 - n_pre + q_len > cap)
    return fail(PHOTON_ERR_ARG, "bad q_len/p0/n_pre/cap");
  if (n_pre > 0 && (!d_kp || !d_vp || n_pre > cap_pre)) return fail(PHOTON_ERR_ARG, "bad prefix");
  if (path < 0 || path > 3) return fail(PHOTON_ERR_ARG, "unknown path %d", path);
  cudaStream_t s = (cudaStream_t)stream;
  AttnArgs a;
  a.Q = d_q;
  a.q_ld = (long long)H * head_dim;
  a.K = d_k;
  a.V = d_v;
  a.cap = cap;
  if (n_pre > 0) {
    a.Kp = d_kp;
    a.Vp = d_vp;
    a.cap_pre = cap_pre;
    a.n_pre = n_pre;
  }
  a.G = G;
  a.H = H;
  a.dh = head_dim;
  a.q_len = q_len;
  a.p0 = p0;
  a.O = d_o;
  a.o_ld = (long long)H * head_dim;
  a.scale = 1.0f / sqrtf((float)head_dim);
  const size_t wsb = n_pre > 0 ? attn_prefix_split_bytes(a) : 0;
  float* ws = nullptr;
  if (wsb) CK(pool_malloc((void**)&ws, wsb, s));
  const bool ok = launch_attn_prefill_path(dtype, a, path, ws, wsb, d_err, s);
  if (ws) cudaFreeAsync(ws, s);
  if (!ok) return fail(PHOTON_ERR_ARG, "path %d does not take this shape", path);
  CK(cudaGetLastError());
  return PHOTON_OK;
}

}  // extern "C"

// ============================================================== vanilla baseline
// A vanilla token-level Transformer of PHOTON's width on the same kernels:
// the baseline of the pages' throughput-per-memory comparison (explainer,
// 475x section).  It is a photon_model with its own tensor list (embed,
// L_van blocks, final gain, head), so weight generation, export, the block
// stack and the GEMM/attention dispatch are shared.

static void build_specs_vanilla(photon_model* m) {
  const long long d = m->d, V = m->V, f = m->f;
  auto add = [&](const std::string& n, int g, long long numel, bool gain) {
    m->t.push_back(TensorRec{n, g, 0, numel, gain});
  };
  m->i_embed = (int)m->t.size();
  add("embed", G_EMB, V * d, false);
  m->i_van = (int)m->t.size();
  for (int l = 0; l < m->L_van; ++l) {  // the layout BlockW expects (wq, wk, wv back to back)
    const std::string p = "van." + std::to_string(l) + ".";
    add(p + "g_attn", G_TOP, d, true);
    add(p + "wq", G_TOP, d * d, false);
    add(p + "wk", G_TOP, d * d, false);
    add(p + "wv", G_TOP, d * d, false);
    add(p + "wo", G_TOP, d * d, false);
    add(p + "g_mlp", G_TOP, d, true);
    add(p + "w1", G_TOP, f * d, false);
    add(p + "w2", G_TOP, d * f, false);
  }
  m->i_van_g = (int)m->t.size();
  add("van.g_final", G_TOP, d, true);
  m->i_head = (int)m->t.size();
  add("head", G_DEC, V * d, false);
  for (auto& r : m->t) {
    const size_t bytes = (size_t)r.numel * (r.gain ? 4 : m->es);
    r.offset = m->group_bytes[r.group];
    m->group_bytes[r.group] += (bytes + 255) & ~size_t(255);
  }
}

struct photon_vanilla_cache {
  photon_model* m = nullptr;
  int B = 0, T = 0, N = 0, cap = 0, max_new = 0, steps = 0, graph_steps = 0;
  cudaStream_t stream = nullptr;
  cudaStream_t cap_s = nullptr;  // capture stream: only ever captured into
  std::vector<void*> allocs;
  size_t kv_bytes = 0, ws_bytes = 0;
  char* kc = nullptr;
  char* vc = nullptr;
  size_t layer_bytes = 0;  // [B][H][cap][dh] per layer
  float2* rope = nullptr;
  float* x = nullptr;
  void *xn = nullptr, *q = nullptr, *att = nullptr, *hid = nullptr, *hn = nullptr;
  float* gemm_ws = nullptr;
  size_t gemm_ws_bytes = 0;
  int* gemm_cnt = nullptr;
  float* attn_ws = nullptr;
  size_t attn_ws_bytes = 0;
  void* sn_x = nullptr;
  float* sn_ss = nullptr;
  unsigned long long* amax_part = nullptr;
  int amax_tiles = 0;
  float* logits = nullptr;     // head output when the argmax is not fused
  int32_t* next_ids = nullptr; // [B] the token the next step feeds
  int32_t* tok_out = nullptr;  // [B] choices of graph-replayed steps
  int* d_err = nullptr;
  int* d_pos = nullptr;        // {position of the next fed token, 0}
};

static Bufs vanilla_bufs(photon_vanilla_cache* c) {
  Bufs b{c->xn, c->q, c->att, c->hid, c->rope, c->gemm_ws, c->gemm_ws_bytes, c->gemm_cnt, c->attn_ws,
         c->attn_ws_bytes, c->d_err};
  b.sn_x = c->sn_x;
  b.sn_ss = c->sn_ss;
  b.sn_cap = c->sn_x ? kSsqCap : 0;
  return b;
}

// One decode step: embed the pending token, run the stack at the next
// position (appending its KV), final norm, head and greedy choice.
static void enqueue_vanilla(photon_model* m, photon_vanilla_cache* c, int32_t* out, float* logits,
                            const int32_t* force, cudaStream_t s) {
  const int B = c->B, d = m->d, V = m->V;
  Bufs b = vanilla_bufs(c);
  launch_embed_f32(m->dt, c->next_ids, m->ptr(m->i_embed), c->x, B, d, V, c->d_err, s);
  StackRun r;
  r.G = B;
  r.q_len = 1;
  r.kc = c->kc;
  r.vc = c->vc;
  r.layer_bytes = c->layer_bytes;
  r.cap = c->cap;
  r.p0_dev = c->d_pos;
  r.n_plan = c->cap;
  r.sn_rows = c->sn_x ? B : 0;
  run_stack(m, m->i_van, m->L_van, c->x, r, b, s);
  launch_rmsnorm(m->dt, c->x, (const float*)m->ptr(m->i_van_g), c->hn, B, d, 1, 0, m->cfg.norm_eps, s);
  if (c->amax_tiles > 0 && !logits) {
    Epilogue e = epi(EPI_ARGMAX, nullptr, V);
    e.argmax_part = c->amax_part;
    e.argmax_tiles = c->amax_tiles;
    gemm(m, b, c->hn, d, m->ptr(m->i_head), d, B, V, d, e, s);
    launch_argmax_partials(c->amax_part, c->amax_tiles, B, V, 0, 1, force, out, nullptr, c->next_ids,
                           c->d_err, nullptr, s);
  } else {
    float* lg = logits ? logits : c->logits;
    gemm(m, b, c->hn, d, m->ptr(m->i_head), d, B, V, d, epi(EPI_STORE_F32, lg, V), s);
    launch_argmax(lg, V, B, V, 0, 1, force, out, nullptr, c->next_ids, c->d_err, SampleArgs{}, s);
  }
  launch_advance(c->d_pos, 1, 0, s);
}

extern "C" {

int photon_vanilla_init(const photon_vanilla_config* cfg, uint64_t seed, photon_model** out) {
  g_err.clear();
  if (!out) return fail(PHOTON_ERR_ARG, "out is NULL");
  *out = nullptr;
  if (!cfg) return fail(PHOTON_ERR_ARG, "config is NULL");
  if (cfg->vocab <= 0 || cfg->d_model <= 0 || cfg->n_heads <= 0 || cfg->head_dim <= 0 || cfg->layers < 1 ||
      cfg->mlp_mult < 1)
    return fail(PHOTON_ERR_ARG, "non-positive model dimension");
  // the shared checks of the PHOTON config, on an equivalent one
  photon_config pc = {};
  pc.vocab = cfg->vocab;
  pc.d_model = cfg->d_model;
  pc.n_heads = cfg->n_heads;
  pc.head_dim = cfg->head_dim;
  pc.levels = 2;
  pc.chunk[0] = pc.chunk[1] = 1;
  pc.enc_layers[0] = 1;
  pc.enc_layers[1] = cfg->layers;
  pc.dec_layers[0] = pc.dec_layers[1] = 1;
  pc.mlp_mult = cfg->mlp_mult;
  pc.dtype = cfg->dtype;
  pc.init_std = cfg->init_std;
  pc.rope_theta = cfg->rope_theta;
  pc.norm_eps = cfg->norm_eps;
  RET(check_config(&pc));
  photon_model* m = new photon_model();
  m->cfg = pc;
  m->vanilla = true;
  m->L_van = cfg->layers;
  m->dt = cfg->dtype;
  m->es = dtype_size(m->dt);
  m->seed = seed;
  m->d = cfg->d_model;
  m->H = cfg->n_heads;
  m->dh = cfg->head_dim;
  m->V = cfg->vocab;
  m->C1 = m->C2 = m->C = 1;
  m->f = cfg->mlp_mult * cfg->d_model;
  m->L1 = m->Ltop = m->Ld1 = m->Ld2 = 0;
  m->use_tc = (m->dt == DT_BF16) && tma_available();
  build_specs_vanilla(m);
  for (int g = 0; g < G_COUNT; ++g) {
    if (m->group_bytes[g] == 0) continue;
    cudaError_t e = injected_alloc_failure() ? cudaErrorMemoryAllocation
                                             : cudaMalloc((void**)&m->group_ptr[g], m->group_bytes[g]);
    if (e != cudaSuccess) {
      cudaGetLastError();
      for (int k = 0; k < g; ++k)
        if (m->group_ptr[k]) cudaFree(m->group_ptr[k]);
      delete m;
      return fail(e == cudaErrorMemoryAllocation ? PHOTON_ERR_OOM : PHOTON_ERR_CUDA,
                  "weight allocation failed: %s", cudaGetErrorString(e));
    }
    generate_group(m, g, nullptr);
  }
  cudaError_t e = cudaStreamSynchronize(nullptr);
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e != cudaSuccess) {
    for (int g = 0; g < G_COUNT; ++g)
      if (m->group_ptr[g]) cudaFree(m->group_ptr[g]);
    delete m;
    return fail(PHOTON_ERR_CUDA, "weight generation failed: %s", cudaGetErrorString(e));
  }
  *out = m;
  return PHOTON_OK;
}

int photon_vanilla_prefill(photon_model* m, const int32_t* d_tokens, int32_t B, int32_t T,
                           int32_t max_new_tokens, void* stream, photon_vanilla_cache** out) {
  g_err.clear();
  if (!m || !out) return fail(PHOTON_ERR_ARG, "NULL model or out");
  *out = nullptr;
  if (!m->vanilla) return fail(PHOTON_ERR_ARG, "not a vanilla baseline model");
  if (!d_tokens) return fail(PHOTON_ERR_ARG, "tokens pointer is NULL");
  if (B <= 0 || T < 2 || max_new_tokens < 0) return fail(PHOTON_ERR_ARG, "need B > 0, T >= 2, max_new >= 0");
  if (B > 65535) return fail(PHOTON_ERR_ARG, "batch %d too large: at most 65535 (attention grid limit)", B);
  cudaStream_t s = (cudaStream_t)stream;
  const int d = m->d, V = m->V, H = m->H, dh = m->dh, L = m->L_van;
  const size_t es = m->es;
  photon_vanilla_cache* c = new photon_vanilla_cache();
  c->m = m;
  c->B = B;
  c->T = T;
  c->N = T - 1;
  c->cap = T - 1 + max_new_tokens;
  c->max_new = max_new_tokens;
  c->stream = s;
  Allocator al{s, &c->allocs, &c->kv_bytes};
  Allocator aw{s, &c->allocs, &c->ws_bytes};
  auto bail = [&](int code) {
    cudaGetLastError();
    if (c->cap_s) cudaStreamDestroy(c->cap_s);
    free_list(c->allocs, s);
    cudaStreamSynchronize(s);
    delete c;
    return code == PHOTON_ERR_OOM ? fail(code, "device allocation failed during prefill") : code;
  };
  c->layer_bytes = (size_t)B * H * c->cap * dh * es;
  c->kc = al.get<char>(c->layer_bytes * L);
  c->vc = al.get<char>(c->layer_bytes * L);
  if (upload_rope(m, &c->rope, c->cap) != PHOTON_OK) return bail(PHOTON_ERR_OOM);
  c->x = aw.get<float>((size_t)B * d * 4);
  c->xn = aw.get<void>((size_t)B * d * es);
  c->q = aw.get<void>((size_t)B * d * es);
  c->att = aw.get<void>((size_t)B * d * es);
  c->hn = aw.get<void>((size_t)B * d * es);
  c->hid = aw.get<void>((size_t)B * m->f * es);
  c->gemm_ws_bytes = std::max(block_ws_need(m, B), gemm_ws_need(m, B, V, d));
  c->gemm_ws = aw.get<float>(c->gemm_ws_bytes);
  c->gemm_cnt = aw.get<int>(kGemmTileCounters * sizeof(int));
  c->attn_ws_bytes = attn_ws_need(m->dt, B, H, dh, 1, c->cap);
  c->attn_ws = aw.get<float>(c->attn_ws_bytes);
  c->amax_tiles = m->use_tc ? gemm_tc_argmax_tiles(B, V, d) : 0;
  if (c->amax_tiles > 0)
    c->amax_part = aw.get<unsigned long long>((size_t)B * c->amax_tiles * 8);
  else
    c->logits = aw.get<float>((size_t)B * V * 4);
  if (m->use_tc && split_norm_enabled()) {
    c->sn_x = aw.get<void>((size_t)B * d * es);
    c->sn_ss = aw.get<float>((size_t)B * kSsqCap * sizeof(float));
  }
  c->next_ids = aw.get<int32_t>((size_t)B * 4);
  c->tok_out = aw.get<int32_t>((size_t)B * 4);
  c->d_err = aw.get<int>(16);
  c->d_pos = aw.get<int>(16);
  if (al.err != cudaSuccess || aw.err != cudaSuccess || !c->kc || !c->vc) return bail(PHOTON_ERR_OOM);
  if (cudaStreamCreateWithFlags(&c->cap_s, cudaStreamNonBlocking) != cudaSuccess) c->cap_s = nullptr;
  if (cudaMemsetAsync(c->d_err, 0, 16, s) != cudaSuccess ||
      cudaMemsetAsync(c->gemm_cnt, 0, kGemmTileCounters * sizeof(int), s) != cudaSuccess)
    return bail(PHOTON_ERR_CUDA);

  // prefill of the first T-1 tokens (temporaries released at the end)
  const long long rows = (long long)B * (T - 1);
  std::vector<void*> tmp;
  size_t tmp_bytes = 0;
  Allocator at{s, &tmp, &tmp_bytes};
  int32_t* ids = at.get<int32_t>((size_t)rows * 4);
  float* x = at.get<float>((size_t)rows * d * 4);
  void* xn = at.get<void>((size_t)rows * d * es);
  void* q = at.get<void>((size_t)rows * d * es);
  void* att = at.get<void>((size_t)rows * d * es);
  void* hid = at.get<void>((size_t)rows * m->f * es);
  const size_t pgw = block_ws_need(m, (int)rows);
  float* pws = at.get<float>(pgw);
  if (at.err != cudaSuccess) {
    free_list(tmp, s);
    return bail(PHOTON_ERR_OOM);
  }
  const size_t w_in = (size_t)T * sizeof(int32_t), w_pre = (size_t)(T - 1) * sizeof(int32_t);
  const int pos[4] = {T - 1, 0, 0, 0};  // pageable source: staged before the call returns
  if (cudaMemcpy2DAsync(ids, w_pre, d_tokens, w_in, w_pre, B, cudaMemcpyDeviceToDevice, s) != cudaSuccess ||
      cudaMemcpy2DAsync(c->next_ids, sizeof(int32_t), d_tokens + (T - 1), w_in, sizeof(int32_t), B,
                        cudaMemcpyDeviceToDevice, s) != cudaSuccess ||
      cudaMemcpyAsync(c->d_pos, pos, sizeof(pos), cudaMemcpyHostToDevice, s) != cudaSuccess) {
    free_list(tmp, s);
    return bail(fail(PHOTON_ERR_CUDA, "token staging failed"));
  }
  launch_embed_f32(m->dt, ids, m->ptr(m->i_embed), x, (int)rows, d, V, c->d_err, s);
  Bufs pb{xn, q, att, hid, c->rope, pws, pgw, c->gemm_cnt, nullptr, 0, c->d_err};
  StackRun r;
  r.G = B;
  r.q_len = T - 1;
  r.kc = c->kc;
  r.vc = c->vc;
  r.layer_bytes = c->layer_bytes;
  r.cap = c->cap;
  run_stack(m, m->i_van, L, x, r, pb, s);
  cudaError_t le = cudaGetLastError();
  free_list(tmp, s);
  if (le != cudaSuccess) return bail(fail(PHOTON_ERR_CUDA, "prefill launch failed: %s", cudaGetErrorString(le)));
  m->live_caches++;
  *out = c;
  return PHOTON_OK;
}

int photon_vanilla_decode_step(photon_model* m, photon_vanilla_cache* c, int32_t* d_out_tokens,
                               float* d_out_logits, const int32_t* d_force_tokens, void* stream) {
  g_err.clear();
  if (!m || !c || c->m != m || !m->vanilla) return fail(PHOTON_ERR_ARG, "model/cache mismatch");
  if (!d_out_tokens) return fail(PHOTON_ERR_ARG, "output token buffer is NULL");
  if (c->steps >= c->max_new) return fail(PHOTON_ERR_CAPACITY, "cache is full (%d steps)", c->max_new);
  cudaStream_t s = (cudaStream_t)stream;
  c->stream = s;
  // the plain step is captured once (on the cache's capture stream) and
  // replayed; the model keeps the executable and updates it for new caches
  const bool plain = !d_out_logits && !d_force_tokens;
  bool replay = plain && c->cap_s != nullptr && graphs_enabled() && c->steps >= 1 && !m->graph_failed_van;
  if (replay && m->graph_owner[0] != c) {
    cudaGraph_t g = nullptr;
    const unsigned long long n0 = launch_total();
    bool ok = cudaStreamBeginCapture(c->cap_s, cudaStreamCaptureModeRelaxed) == cudaSuccess;
    if (ok) {
      enqueue_vanilla(m, c, c->tok_out, nullptr, nullptr, c->cap_s);
      ok = cudaStreamEndCapture(c->cap_s, &g) == cudaSuccess && g;
    }
    const long long captured = (long long)(launch_total() - n0);
    note_launch(-captured);
    m->graph_kernels[0] = ok ? captured : 0;
    if (ok && m->graph[0]) {
      cudaGraphExecUpdateResultInfo info;
      if (cudaGraphExecUpdate(m->graph[0], g, &info) != cudaSuccess) {
        cudaGetLastError();
        cudaGraphExecDestroy(m->graph[0]);
        m->graph[0] = nullptr;
      }
    }
    if (ok && !m->graph[0]) ok = cudaGraphInstantiate(&m->graph[0], g, 0) == cudaSuccess;
    if (g) cudaGraphDestroy(g);
    if (!ok) {
      cudaGetLastError();
      m->graph[0] = nullptr;
      m->graph_owner[0] = nullptr;
      m->graph_failed_van = true;
      replay = false;
    } else {
      m->graph_owner[0] = c;
    }
  }
  if (replay) {
    CK(cudaGraphLaunch(m->graph[0], s));
    note_launch(m->graph_kernels[0]);
    c->graph_steps += 1;
    if (d_out_tokens != c->tok_out)
      CK(cudaMemcpyAsync(d_out_tokens, c->tok_out, (size_t)c->B * sizeof(int32_t), cudaMemcpyDeviceToDevice, s));
  } else {
    enqueue_vanilla(m, c, d_out_tokens, d_out_logits, d_force_tokens, s);
  }
  CK(cudaGetLastError());
  c->N += 1;
  c->steps += 1;
  return PHOTON_OK;
}

int photon_vanilla_cache_info(photon_vanilla_cache* c, photon_vanilla_stats* out) {
  g_err.clear();
  if (!c || !out) return fail(PHOTON_ERR_ARG, "NULL argument");
  memset(out, 0, sizeof(*out));
  CK(cudaStreamSynchronize(c->stream));
  int err = 0;
  CK(cudaMemcpy(&err, c->d_err, sizeof(int), cudaMemcpyDeviceToHost));
  out->B = c->B;
  out->N = c->N;
  out->capacity = c->cap;
  out->steps = c->steps;
  out->device_error = err;
  out->graph_steps = c->graph_steps;
  out->kv_bytes = c->kv_bytes;
  out->workspace_bytes = c->ws_bytes;
  return PHOTON_OK;
}

int photon_vanilla_free_cache(photon_vanilla_cache* c) {
  g_err.clear();
  if (!c) return fail(PHOTON_ERR_ARG, "cache is NULL");
  photon_model* m = c->m;
  if (m->graph_owner[0] == c) m->graph_owner[0] = nullptr;  // its buffers are going away
  if (c->cap_s) cudaStreamDestroy(c->cap_s);                 // only ever captured into
  free_list(c->allocs, c->stream);                             // stream-ordered
  CK(cudaGetLastError());
  m->live_caches--;
  delete c;
  return PHOTON_OK;
}

}  // extern "C"

// ============================================================== teacher-forced scoring
extern "C" {

// Scores sequences [0, B) of d_tokens in one pass (arguments checked by photon_score).
static int score_slice(photon_model* m, const int32_t* d_tokens, int32_t B, int32_t T, float* d_out_logprob,
                       void* stream) {
  cudaStream_t s = (cudaStream_t)stream;
  const int d = m->d, V = m->V, C = m->C, C1 = m->C1, C2 = m->C2;
  const size_t es = m->es, hd = (size_t)m->H * m->dh;
  const float eps = m->cfg.norm_eps;
  const int N = T / C, K = N - 1;
  const long long G = (long long)B * K;  // scored chunks (chunk k conditions chunk k + 1)
  const long long G2 = G * C2;           // their sub-chunks
  const int P = 2 * C1 - 1;              // token-decoder positions per sub-chunk
  const long long R = G2 * C1;           // scored tokens = B * (T - C)
  const long long rows_x = G2 * P;

  std::vector<void*> tmp;
  size_t tmp_bytes = 0;
  Allocator at{s, &tmp, &tmp_bytes};
  void* o_all = at.get<void>((size_t)B * N * d * es);
  if (at.err != cudaSuccess) {
    free_list(tmp, s);
    return fail(PHOTON_ERR_OOM, "device allocation failed during scoring");
  }
  // a1-a5 over the true tokens, keeping every top output
  photon_cache* c = nullptr;
  int rc = prefill_impl(m, nullptr, d_tokens, B, T, PHOTON_MODE_REC, 0, stream, &c, o_all);
  if (rc != PHOTON_OK) {
    free_list(tmp, s);
    return rc;
  }
  void* o_sel = at.get<void>((size_t)G * d * es);
  float* x2 = at.get<float>((size_t)G * C2 * d * 4);
  void* ahat = at.get<void>((size_t)G * C2 * d * es);
  float* c1 = at.get<float>((size_t)G2 * C1 * d * 4);
  float* xd = at.get<float>((size_t)rows_x * d * 4);
  int32_t* ids = C1 > 1 ? at.get<int32_t>((size_t)G2 * (C1 - 1) * 4) : nullptr;
  float* emb = C1 > 1 ? at.get<float>((size_t)G2 * (C1 - 1) * d * 4) : nullptr;
  void* xn = at.get<void>((size_t)rows_x * d * es);
  void* q = at.get<void>((size_t)rows_x * d * es);
  void* att = at.get<void>((size_t)rows_x * d * es);
  void* hid = at.get<void>((size_t)rows_x * m->f * es);
  void* hn = at.get<void>((size_t)rows_x * d * es);
  void* hsel = at.get<void>((size_t)R * d * es);
  int32_t* tg = at.get<int32_t>((size_t)R * 4);
  const size_t l2 = (size_t)G * hd * C2 * es, l1 = (size_t)G2 * hd * P * es;
  char* d2k = at.get<char>(l2 * m->Ld2);
  char* d2v = at.get<char>(l2 * m->Ld2);
  char* d1k = at.get<char>(l1 * m->Ld1);
  char* d1v = at.get<char>(l1 * m->Ld1);
  const long long S = std::min<long long>(R, 8192);  // head rows per slice
  float* lg = at.get<float>((size_t)S * V * 4);
  size_t gw = std::max(block_ws_need(m, (int)G * C2), block_ws_need(m, (int)rows_x));
  gw = std::max(gw, gemm_ws_need(m, (int)G, C2 * d, d));
  gw = std::max(gw, gemm_ws_need(m, (int)G2, C1 * d, d));
  gw = std::max(gw, gemm_ws_need(m, (int)S, V, d));
  float* pws = at.get<float>(gw);
  int* cnt = at.get<int>(kGemmTileCounters * sizeof(int));
  int* err = at.get<int>(16);
  if (at.err != cudaSuccess) {
    photon_free_cache(c);
    free_list(tmp, s);
    return fail(PHOTON_ERR_OOM, "device allocation failed during scoring");
  }
  cudaError_t ce = cudaSuccess;  // first failing call; work continues to the common release below
  auto ck = [&](cudaError_t e) {
    if (ce == cudaSuccess && e != cudaSuccess) ce = e;
  };
  ck(cudaMemsetAsync(cnt, 0, kGemmTileCounters * sizeof(int), s));
  ck(cudaMemsetAsync(err, 0, 16, s));
  Bufs b{xn, q, att, hid, c->rope, pws, gw, cnt, nullptr, 0, err};
  const cudaMemcpyKind dd = cudaMemcpyDeviceToDevice;

  // chunks 0..N-2 of every sequence condition chunks 1..N-1
  ck(cudaMemcpy2DAsync(o_sel, (size_t)K * d * es, o_all, (size_t)N * d * es, (size_t)K * d * es, B, dd, s));
  // a7, a8: Converter_2 and the level-2 decoder over its C2 positions -> A-hat
  gemm(m, b, o_sel, d, m->ptr(m->i_cv2), d, (int)G, C2 * d, d, epi(EPI_STORE_F32, x2, (long long)C2 * d), s);
  StackRun r2;
  r2.G = (int)G;
  r2.q_len = C2;
  r2.kc = d2k;
  r2.vc = d2v;
  r2.layer_bytes = l2;
  r2.cap = C2;
  run_stack(m, m->i_dec2, m->Ld2, x2, r2, b, s);
  launch_rmsnorm(m->dt, x2, (const float*)m->ptr(m->i_dec2_g), ahat, (int)(G * C2), d, 1, 0, eps, s);
  // a9: Converter_1 -- C1 conditioning vectors per sub-chunk
  gemm(m, b, ahat, d, m->ptr(m->i_cv1), d, (int)G2, C1 * d, d, epi(EPI_STORE_F32, c1, (long long)C1 * d), s);
  // token-decoder sequence of a sub-chunk: its conditioning, then its first C1 - 1 true tokens
  ck(cudaMemcpy2DAsync(xd, (size_t)P * d * 4, c1, (size_t)C1 * d * 4, (size_t)C1 * d * 4, G2, dd, s));
  if (C1 > 1) {
    for (int bb = 0; bb < B; ++bb)
      ck(cudaMemcpy2DAsync(ids + (size_t)bb * K * C2 * (C1 - 1), (size_t)(C1 - 1) * 4,
                           d_tokens + (size_t)bb * T + C, (size_t)C1 * 4, (size_t)(C1 - 1) * 4,
                           (size_t)K * C2, dd, s));
    launch_embed_f32(m->dt, ids, m->ptr(m->i_embed), emb, (int)(G2 * (C1 - 1)), d, V, err, s);
    ck(cudaMemcpy2DAsync(xd + (size_t)C1 * d, (size_t)P * d * 4, emb, (size_t)(C1 - 1) * d * 4,
                         (size_t)(C1 - 1) * d * 4, G2, dd, s));
  }
  // a10: the token decoder, one causal pass over the P positions of every sub-chunk
  StackRun r1;
  r1.G = (int)G2;
  r1.q_len = P;
  r1.kc = d1k;
  r1.vc = d1v;
  r1.layer_bytes = l1;
  r1.cap = P;
  run_stack(m, m->i_dec1, m->Ld1, xd, r1, b, s);
  launch_rmsnorm(m->dt, xd, (const float*)m->ptr(m->i_dec1_g), hn, (int)rows_x, d, 1, 0, eps, s);
  // rows C1-1 .. P-1 of a sub-chunk predict its C1 tokens; targets = tokens C .. T-1
  ck(cudaMemcpy2DAsync(hsel, (size_t)C1 * d * es, (char*)hn + (size_t)(C1 - 1) * d * es, (size_t)P * d * es,
                       (size_t)C1 * d * es, G2, dd, s));
  ck(cudaMemcpy2DAsync(tg, (size_t)(T - C) * 4, d_tokens + C, (size_t)T * 4, (size_t)(T - C) * 4, B, dd, s));
  // a11: head and log-softmax, a slice of rows at a time
  for (long long r0 = 0; r0 < R; r0 += S) {
    const int rows = (int)std::min<long long>(S, R - r0);
    gemm(m, b, (char*)hsel + (size_t)r0 * d * es, d, m->ptr(m->i_head), d, rows, V, d,
         epi(EPI_STORE_F32, lg, V), s);
    launch_logprob(lg, V, tg + r0, d_out_logprob + r0, rows, err, s);
  }
  int herr = 0;
  ck(cudaGetLastError());
  cudaError_t le = ce;
  if (le == cudaSuccess) le = cudaMemcpyAsync(&herr, err, sizeof(int), cudaMemcpyDeviceToHost, s);
  photon_free_cache(c);  // stream-ordered releases after the read above
  free_list(tmp, s);
  if (le == cudaSuccess) le = cudaStreamSynchronize(s);
  if (le != cudaSuccess) return fail(PHOTON_ERR_CUDA, "scoring failed: %s", cudaGetErrorString(le));
  if (herr) return fail(PHOTON_ERR_DEVICE_CHECK, "device check failed during scoring (code %d)", herr);
  return PHOTON_OK;
}

int photon_score(photon_model* m, const int32_t* d_tokens, int32_t B, int32_t T, float* d_out_logprob,
                 void* stream) {
  g_err.clear();
  if (!m || !d_tokens || !d_out_logprob) return fail(PHOTON_ERR_ARG, "NULL argument");
  if (m->vanilla) return fail(PHOTON_ERR_ARG, "a vanilla baseline model takes the photon_vanilla_* calls");
  if (m->general) return fail(PHOTON_ERR_ARG, "teacher-forced scoring is available for two-level models only");
  if (B <= 0 || T <= m->C || T % m->C)
    return fail(PHOTON_ERR_ARG, "T = %d must be a multiple of C1*C2 = %d longer than one chunk", T, m->C);
  // The decoders run over (sequence, chunk, sub-chunk) groups, which the
  // attention kernels index in a grid dimension of at most 65535 (times the
  // query length where a split-K combine follows).  Whole sequences are
  // scored a slice at a time so that a slice stays within it.
  const long long K = T / m->C - 1, P = 2LL * m->C1 - 1;
  const long long per_seq = K * m->C2 * std::max(1LL, std::min(P, 4LL));
  constexpr long long kMaxGroups = 65535;
  if (per_seq > kMaxGroups)
    return fail(PHOTON_ERR_ARG, "T = %d is too long to score: at most %lld chunks per sequence", T,
                kMaxGroups / ((long long)m->C2 * std::max(1LL, std::min(P, 4LL))) + 1);
  const int bs = (int)std::min<long long>(B, kMaxGroups / per_seq);
  for (int b0 = 0; b0 < B; b0 += bs)
    RET(score_slice(m, d_tokens + (size_t)b0 * T, std::min(bs, B - b0), T,
                    d_out_logprob + (size_t)b0 * (T - m->C), stream));
  return PHOTON_OK;
}

}  // extern "C"

// ============================================================== multi-query aggregation
// PHOTON explainer, quality section: several slightly varied queries, their
// outputs combined by majority vote or best-of-N.  Kernels in k_aggregate.cu.
namespace photon {
void launch_vote(const int32_t* cand, int Q, int N, int L, int b0, int len, int32_t* choice, double* score,
                 cudaStream_t s);
void launch_best(const float* logprob, int Q, int N, int L, int b0, int len, int32_t* choice, double* score,
                 cudaStream_t s);
}  // namespace photon

extern "C" {

int photon_aggregate(int32_t mode, const int32_t* d_cand, const float* d_logprob, int32_t Q, int32_t N,
                     int32_t L, int32_t span_begin, int32_t span_len, int32_t* d_choice, double* d_score,
                     void* stream) {
  g_err.clear();
  if (mode != PHOTON_AGG_VOTE && mode != PHOTON_AGG_BEST) return fail(PHOTON_ERR_ARG, "unknown aggregation mode %d", mode);
  if (Q < 0 || N <= 0 || L < 0 || span_begin < 0 || span_len < 0 || (long long)span_begin + span_len > L)
    return fail(PHOTON_ERR_ARG, "bad shape: Q = %d, N = %d, L = %d, span [%d, %d + %d)", Q, N, L, span_begin,
                span_begin, span_len);
  if (Q == 0) return PHOTON_OK;
  if (!d_choice) return fail(PHOTON_ERR_ARG, "d_choice is NULL");
  cudaStream_t s = (cudaStream_t)stream;
  if (mode == PHOTON_AGG_VOTE) {
    if (!d_cand) return fail(PHOTON_ERR_ARG, "majority vote needs d_cand");
    launch_vote(d_cand, Q, N, L, span_begin, span_len, d_choice, d_score, s);
  } else {
    if (!d_logprob) return fail(PHOTON_ERR_ARG, "best-of-N needs d_logprob");
    launch_best(d_logprob, Q, N, L, span_begin, span_len, d_choice, d_score, s);
  }
  CK(cudaGetLastError());
  return PHOTON_OK;
}

int photon_multi_query(photon_model* m, const photon_cache* prefix, const int32_t* d_prompts, int32_t Q,
                       int32_t N, int32_t T, int32_t n_chunks, float temperature, float top_p, uint64_t seed,
                       int32_t mode, int32_t* d_cand, int32_t* d_choice, double* d_score, void* stream) {
  g_err.clear();
  if (!m || !d_prompts || !d_cand || !d_choice) return fail(PHOTON_ERR_ARG, "NULL argument");
  if (m->general) return fail(PHOTON_ERR_ARG, "multi-query aggregation is available for two-level models only");
  if (m->vanilla) return fail(PHOTON_ERR_ARG, "a vanilla baseline model takes the photon_vanilla_* calls");
  if (mode != PHOTON_AGG_VOTE && mode != PHOTON_AGG_BEST) return fail(PHOTON_ERR_ARG, "unknown aggregation mode %d", mode);
  if (Q <= 0 || N <= 0 || n_chunks <= 0 || (long long)Q * N > (1ll << 30))
    return fail(PHOTON_ERR_ARG, "bad group shape: Q = %d, N = %d, n_chunks = %d", Q, N, n_chunks);
  if (!(temperature >= 0.f) || !std::isfinite(temperature) ||
      (temperature > 0.f && !std::isfinite(1.0f / temperature)))
    return fail(PHOTON_ERR_ARG, "temperature must be finite, >= 0 and not subnormal");
  if (!(top_p > 0.f && top_p <= 1.f)) return fail(PHOTON_ERR_ARG, "top_p must be in (0, 1]");
  if (mode == PHOTON_AGG_BEST && prefix)
    return fail(PHOTON_ERR_ARG, "best-of-N scores the whole context and takes no prefix cache");
  if ((long long)n_chunks * m->C > (1ll << 30)) return fail(PHOTON_ERR_ARG, "n_chunks too large");
  cudaStream_t s = (cudaStream_t)stream;
  const int rows = Q * N, C = m->C, Lc = n_chunks * C;

  // every row decodes n_chunks chunks in RecGen mode, drawing with its own row's noise
  photon_cache* c = nullptr;
  RET(prefill_impl(m, prefix, d_prompts, rows, T, PHOTON_MODE_REC, n_chunks, stream, &c, nullptr));
  int rc = photon_cache_set_sampling(c, temperature, seed);
  if (rc == PHOTON_OK) rc = photon_cache_set_top_p(c, top_p);
  if (rc == PHOTON_OK) rc = photon_decode_rec_chunks(m, c, n_chunks, d_cand, stream);
  int herr = 0;
  cudaError_t le = cudaSuccess;
  if (rc == PHOTON_OK) le = cudaMemcpyAsync(&herr, c->d_err, sizeof(int), cudaMemcpyDeviceToHost, s);
  const std::string decode_msg = g_err;
  const int frc = photon_free_cache(c);
  if (rc != PHOTON_OK) {
    g_err = decode_msg;
    return rc;
  }
  if (frc != PHOTON_OK) return frc;
  if (le == cudaSuccess) le = cudaStreamSynchronize(s);
  if (le != cudaSuccess) return fail(PHOTON_ERR_CUDA, "multi-query decode failed: %s", cudaGetErrorString(le));
  if (herr) return fail(PHOTON_ERR_DEVICE_CHECK, "device check failed during decode (code %d)", herr);

  if (mode == PHOTON_AGG_VOTE) {
    RET(photon_aggregate(PHOTON_AGG_VOTE, d_cand, nullptr, Q, N, Lc, 0, Lc, d_choice, d_score, stream));
    CK(cudaStreamSynchronize(s));
    return PHOTON_OK;
  }
  // best-of-N: teacher-forced log-probabilities of prompt + continuation,
  // summed over the continuation (score index t covers token t + C)
  const int Tf = T + Lc;
  std::vector<void*> tmp;
  size_t tmp_bytes = 0;
  Allocator at{s, &tmp, &tmp_bytes};
  int32_t* full = at.get<int32_t>((size_t)rows * Tf * sizeof(int32_t));
  float* lp = at.get<float>((size_t)rows * (Tf - C) * sizeof(float));
  if (at.err != cudaSuccess) {
    free_list(tmp, s);
    return fail(PHOTON_ERR_OOM, "device allocation failed during best-of-N scoring");
  }
  const cudaMemcpyKind dd = cudaMemcpyDeviceToDevice;
  cudaError_t ce = cudaMemcpy2DAsync(full, (size_t)Tf * 4, d_prompts, (size_t)T * 4, (size_t)T * 4, rows, dd, s);
  if (ce == cudaSuccess)
    ce = cudaMemcpy2DAsync(full + T, (size_t)Tf * 4, d_cand, (size_t)Lc * 4, (size_t)Lc * 4, rows, dd, s);
  rc = ce == cudaSuccess ? photon_score(m, full, rows, Tf, lp, stream) : PHOTON_OK;
  if (ce == cudaSuccess && rc == PHOTON_OK)
    rc = photon_aggregate(PHOTON_AGG_BEST, nullptr, lp, Q, N, Tf - C, T - C, Lc, d_choice, d_score, stream);
  const std::string score_msg = g_err;
  free_list(tmp, s);
  if (ce != cudaSuccess) return fail(PHOTON_ERR_CUDA, "copying the scored rows failed: %s", cudaGetErrorString(ce));
  if (rc != PHOTON_OK) {
    g_err = score_msg;
    return rc;
  }
  CK(cudaStreamSynchronize(s));
  return PHOTON_OK;
}

}  // extern "C"
