// Host side of the libkvq C ABI: argument checks, the greedy allocator and
// plan builder, and the kernel launches. See kvq.h for the contract.
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <string>
#include <vector>

#include "common.cuh"

namespace kvq {
cudaError_t launch_energy(const void* k, int dtype, int64_t n_tokens, int n_kv,
                          unsigned long long* acc, uint32_t* status, cudaStream_t st);
cudaError_t launch_quantize_append(const QuantParams& p, int bits_v, cudaStream_t st);
size_t decode_workspace_bytes_for(int batch, int n_q, int n_kv, int bits_k, int bits_v,
                                  int64_t max_len);
cudaError_t launch_decode(const Plan* const* plans, const CacheMap& cm, int32_t* len,
                          int batch, int64_t max_len, const void* q, int q_dtype, int n_q, int n_kv,
                          int bits_k, int bits_v, float* out, void* ws, size_t ws_bytes,
                          uint32_t* status, cudaStream_t st, const void* k_new, const void* v_new,
                          int kv_dtype, int n_new, int64_t cap, int early, const double* theta,
                          float* rec_out);
size_t dense_workspace_bytes_for(int batch, int n_kv, int n_q, int64_t max_len);
cudaError_t launch_dense_decode(const void* k, const void* v, const int32_t* len, int batch,
                                int n_kv, int64_t cap, int64_t max_len, const void* q, int n_q,
                                float* out, void* ws, size_t ws_bytes, uint32_t* status,
                                cudaStream_t st);
cudaError_t launch_combine(const Plan* const* plans, const float* recs, int n_parts, int batch,
                           int n_q, int n_kv, float* out, cudaStream_t st);
void set_decode_stall(long long cycles);
void set_decode_deterministic(int on);
cudaError_t launch_window_push(const void* k, const void* v, int dtype, int n_new, int n_kv,
                               int32_t* len, int32_t* wlen, float* const* wins, int R,
                               int64_t cap, int batch, cudaStream_t st);
cudaError_t launch_window_record(const Plan* const* plans, const float* const* wins,
                                 const int32_t* len, const int32_t* wlen, int R, const void* q,
                                 int q_dtype, int n_q, int n_kv, int batch, float* recs,
                                 cudaStream_t st);
int window_parts(int R, int* tokens_per_part);
int window_parts_max();
cudaError_t launch_decode_window(const Plan* const* plans, const CacheMap& cm, int32_t* len,
                                 int batch, int64_t max_len, const void* q, int q_dtype, int n_q,
                                 int n_kv, int bits_k, int bits_v, float* out, void* ws,
                                 size_t ws_bytes, uint32_t* status, cudaStream_t st,
                                 const void* k_new, const void* v_new, int kv_dtype,
                                 int n_new, int64_t cap, int early, float* const* wins,
                                 int32_t* wlen, int R);

namespace {

thread_local std::string g_err;

int fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  std::vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_err = buf;
  return code;
}

int cuda_fail(cudaError_t e, const char* where) {
  return fail(KVQ_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

const double kD[9] = KVQ_CB_D;
const uint16_t kC16[KVQ_CB_N_C16] = KVQ_CB_C16;
const float kThr[KVQ_CB_N_THR] = KVQ_CB_THR;

int check_cfg(const kvq_cfg* cfg) {
  if (!cfg) return fail(KVQ_ERR_ARG, "cfg is NULL");
  if (cfg->head_dim != kHeadDim) return fail(KVQ_ERR_UNSUPPORTED, "head_dim %d (only 128)", cfg->head_dim);
  if (cfg->n_kv_heads < 1 || cfg->n_kv_heads > 4096) return fail(KVQ_ERR_ARG, "n_kv_heads %d", cfg->n_kv_heads);
  if (cfg->bits_k < 1 || cfg->bits_k > 8) return fail(KVQ_ERR_ARG, "bits_k %d not in 1..8", cfg->bits_k);
  if (cfg->bits_v < 1 || cfg->bits_v > 8) return fail(KVQ_ERR_ARG, "bits_v %d not in 1..8", cfg->bits_v);
  if (cfg->b_max != 8) return fail(KVQ_ERR_ARG, "b_max %d (must be 8)", cfg->b_max);
  const int mode = cfg->alloc_mode & ~KVQ_ALLOC_ROTATE_KEYS;
  if (mode != KVQ_ALLOC_GREEDY && mode != KVQ_ALLOC_UNIFORM)
    return fail(KVQ_ERR_ARG, "alloc_mode %d", cfg->alloc_mode);
  return KVQ_OK;
}

bool dtype_ok(int dt) { return dt == KVQ_BF16 || dt == KVQ_FP16 || dt == KVQ_FP32; }

// SplitMix64: n-th output of the stream seeded with s.
uint64_t splitmix64(uint64_t s, uint64_t n) {
  uint64_t z = s + (n + 1) * 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

// Greedy marginal-gain widths: bits_k * 64 steps from zero, each +1 bit to the
// block with the largest E_j (D(b_j) - D(b_j + 1)) below 8 (first index wins).
void greedy_widths(const double* E, int bits_k, uint8_t* w) {
  int b[kBlocks] = {0};
  for (int step = 0; step < kBlocks * bits_k; ++step) {
    int best = -1;
    double best_gain = 0.0;
    for (int j = 0; j < kBlocks; ++j) {
      if (b[j] >= 8) continue;
      const double gain = E[j] * (kD[b[j]] - kD[b[j] + 1]);
      if (best < 0 || gain > best_gain) {
        best = j;
        best_gain = gain;
      }
    }
    b[best] += 1;
  }
  for (int j = 0; j < kBlocks; ++j) w[j] = (uint8_t)b[j];
}

// Everything of a plan that follows from its widths: plan order (nonzero
// widths, width descending, block index ascending), K segment offsets, the
// decode schedule (half steps, classes). Zeroes those fields first.
void fill_schedule(Plan* pl) {
  pl->n_ranks = 0;
  std::memset(pl->order, 0, sizeof pl->order);
  std::memset(pl->seg_off, 0, sizeof pl->seg_off);
  pl->n_half = 0;
  std::memset(pl->hs_width, 0, sizeof pl->hs_width);
  std::memset(pl->hs_rank0, 0, sizeof pl->hs_rank0);
  std::memset(pl->hs_count, 0, sizeof pl->hs_count);
  pl->n_class = 0;
  std::memset(pl->cls_w, 0, sizeof pl->cls_w);
  std::memset(pl->cls_hs0, 0, sizeof pl->cls_hs0);
  std::memset(pl->cls_nhs, 0, sizeof pl->cls_nhs);
  std::memset(pl->cls_last, 0, sizeof pl->cls_last);
  std::memset(pl->cls_seg0, 0, sizeof pl->cls_seg0);
  int ranks = 0;
  for (int w = 8; w >= 1; --w)
    for (int j = 0; j < kBlocks; ++j)
      if (pl->width[j] == w) pl->order[ranks++] = (uint8_t)j;
  pl->n_ranks = ranks;
  int off = 0;
  for (int r = 0; r < ranks; ++r) {
    pl->seg_off[r] = (uint16_t)off;
    off += 2 * pl->width[pl->order[r]];
  }
  pl->seg_off[ranks] = (uint16_t)off;
  // decode schedule: runs of equal width cut into groups of at most 4 ranks
  int nh = 0;
  for (int r = 0; r < ranks;) {
    const int w = pl->width[pl->order[r]];
    int n = 0;
    while (r + n < ranks && n < 4 && pl->width[pl->order[r + n]] == w) ++n;
    pl->hs_width[nh] = (uint8_t)w;
    pl->hs_rank0[nh] = (uint8_t)r;
    pl->hs_count[nh] = (uint8_t)n;
    ++nh;
    r += n;
  }
  pl->n_half = (uint8_t)nh;
  // classes: maximal runs of half steps with one width
  int nc = 0;
  for (int hs = 0; hs < nh;) {
    int e = hs;
    while (e < nh && pl->hs_width[e] == pl->hs_width[hs]) ++e;
    pl->cls_w[nc] = pl->hs_width[hs];
    pl->cls_hs0[nc] = (uint8_t)hs;
    pl->cls_nhs[nc] = (uint8_t)(e - hs);
    pl->cls_last[nc] = pl->hs_count[e - 1];
    pl->cls_seg0[nc] = pl->seg_off[pl->hs_rank0[hs]];
    ++nc;
    hs = e;
  }
  pl->n_class = (uint8_t)nc;
}

// W (optional): query block energies of the query-weighted variant; the
// widths then come from the products E_j W_j, the key scales still from E.
void build_plan(const kvq_cfg* cfg, int layer, int kv_head, const double* E, Plan* pl,
                const double* W = nullptr) {
  std::memset(pl, 0, sizeof(Plan));
  pl->magic = KVQ_PLAN_MAGIC;
  pl->bits_k = cfg->bits_k;
  pl->bits_v = cfg->bits_v;
  pl->layer = layer;
  pl->kv_head = kv_head;
  pl->words_k = 128 * cfg->bits_k;
  pl->words_v = 128 * cfg->bits_v;
  if ((cfg->alloc_mode & ~KVQ_ALLOC_ROTATE_KEYS) == KVQ_ALLOC_UNIFORM) {
    for (int j = 0; j < kBlocks; ++j) pl->width[j] = (uint8_t)cfg->bits_k;
  } else if (W) {
    double EW[kBlocks];
    for (int j = 0; j < kBlocks; ++j) EW[j] = E[j] * W[j];
    greedy_widths(EW, cfg->bits_k, pl->width);
  } else {
    greedy_widths(E, cfg->bits_k, pl->width);
  }
  double tot = 0.0;
  for (int j = 0; j < kBlocks; ++j) tot += E[j];
  pl->energy_sum = tot;
  for (int j = 0; j < kBlocks; ++j) {
    const double a = tot > 0.0 ? std::sqrt(E[j] / (2.0 * tot)) : 0.0;
    pl->a_hat[j] = (float)a;
    pl->g[j] = a > 0.0 ? (float)(1.0 / a) : 0.f;
  }
  fill_schedule(pl);
  const uint64_t key = splitmix64(cfg->v_seed, ((uint64_t)(uint32_t)layer << 32) + (uint32_t)kv_head);
  for (int i = 0; i < kHeadDim; ++i)
    if (splitmix64(key, (uint64_t)i) >> 63) pl->v_sign[i >> 5] |= 1u << (i & 31);
  if (cfg->alloc_mode & KVQ_ALLOC_ROTATE_KEYS) {  // key rotation signs: outputs 128 + P
    pl->k_rot = 1;
    for (int P = 0; P < kHeadDim; ++P)
      if (splitmix64(key, (uint64_t)(kHeadDim + P)) >> 63) pl->k_sign[P >> 5] |= 1u << (P & 31);
  }
}

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

}  // namespace

// Lets the other translation units of the library report through
// kvq_last_error().
int set_last_error(int code, const char* msg) {
  g_err = msg;
  return code;
}

}  // namespace kvq

using namespace kvq;

extern "C" {

const char* kvq_version(void) { return "kvq 0.1 (sm_100a)"; }

const char* kvq_last_error(void) { return g_err.c_str(); }

size_t kvq_plan_bytes(void) { return KVQ_PLAN_BYTES; }

size_t kvq_tile_bytes(const kvq_cfg* cfg) {
  if (check_cfg(cfg) != KVQ_OK) return 0;
  return (size_t)tile_bytes(cfg->bits_k, cfg->bits_v);
}

size_t kvq_cache_bytes(const kvq_cfg* cfg, int64_t cap_tokens) {
  if (check_cfg(cfg) != KVQ_OK || cap_tokens < 0) return 0;
  const size_t tiles = (size_t)((cap_tokens + kTile - 1) / kTile);
  return tiles * cfg->n_kv_heads * (size_t)tile_bytes(cfg->bits_k, cfg->bits_v);
}

size_t kvq_alloc_workspace_bytes(const kvq_cfg* cfg) {
  if (check_cfg(cfg) != KVQ_OK) return 0;
  return align_up((size_t)cfg->n_kv_heads * kBlocks * 16, 256);
}

size_t kvq_decode_workspace_bytes(const kvq_cfg* cfg, int batch, int n_q_heads, int64_t max_len) {
  if (check_cfg(cfg) != KVQ_OK || batch < 1 || n_q_heads < 1 || max_len < 1 ||
      max_len > 0x7FFFFFFF || n_q_heads % cfg->n_kv_heads != 0 ||
      n_q_heads / cfg->n_kv_heads > 16)
    return 0;
  return decode_workspace_bytes_for(batch, n_q_heads, cfg->n_kv_heads, cfg->bits_k, cfg->bits_v,
                                    max_len);
}

int kvq_codebook(int bits, float* centroids, float* thresholds, double* distortion) {
  if (bits < 1 || bits > 8) return fail(KVQ_ERR_ARG, "bits %d not in 1..8", bits);
  const int n = 1 << bits;
  if (centroids)
    for (int m = 0; m < n; ++m) {
      __half h = __ushort_as_half(kC16[cb_c_off(bits) + m]);
      centroids[m] = __half2float(h);
    }
  if (thresholds)
    for (int m = 0; m < n - 1; ++m) thresholds[m] = kThr[cb_t_off(bits) + m];
  if (distortion) *distortion = kD[bits];
  return KVQ_OK;
}

int kvq_plan_build(const kvq_cfg* cfg, int layer, const double* E_host, int n_heads,
                   void* plans_host) {
  int rc = check_cfg(cfg);
  if (rc) return rc;
  if (!E_host || !plans_host || n_heads < 1) return fail(KVQ_ERR_ARG, "null pointer or n_heads < 1");
  for (int i = 0; i < n_heads * kBlocks; ++i)
    if (!(E_host[i] >= 0.0) || !std::isfinite(E_host[i]))
      return fail(KVQ_ERR_ARG, "energy %d is negative or not finite", i);
  Plan* out = reinterpret_cast<Plan*>(plans_host);
  for (int h = 0; h < n_heads; ++h) build_plan(cfg, layer, h, E_host + (size_t)h * kBlocks, out + h);
  return KVQ_OK;
}

int kvq_plan_check(const kvq_cfg* cfg, const void* plan_host) {
  int rc = check_cfg(cfg);
  if (rc) return rc;
  if (!plan_host) return fail(KVQ_ERR_ARG, "null plan");
  const Plan& p = *reinterpret_cast<const Plan*>(plan_host);
  if (p.magic != KVQ_PLAN_MAGIC) return fail(KVQ_ERR_ARG, "plan magic 0x%08x", p.magic);
  if (p.bits_k != cfg->bits_k || p.bits_v != cfg->bits_v)
    return fail(KVQ_ERR_ARG, "plan K%dV%d vs cfg K%dV%d", p.bits_k, p.bits_v, cfg->bits_k,
                cfg->bits_v);
  if (p.words_k != 128 * p.bits_k || p.words_v != 128 * p.bits_v)
    return fail(KVQ_ERR_ARG, "plan word counts");
  int sum = 0;
  for (int j = 0; j < kBlocks; ++j) {
    if (p.width[j] > 8) return fail(KVQ_ERR_ARG, "width of block %d is %d", j, p.width[j]);
    sum += p.width[j];
    if (!(p.g[j] >= 0.f) || !std::isfinite(p.g[j]) || !(p.a_hat[j] >= 0.f) ||
        !std::isfinite(p.a_hat[j]))
      return fail(KVQ_ERR_ARG, "scales of block %d", j);
  }
  if (sum != kBlocks * p.bits_k)
    return fail(KVQ_ERR_ARG, "widths sum to %d bits per block pair, not %d", sum,
                kBlocks * p.bits_k);
  if (p.k_rot > 1) return fail(KVQ_ERR_ARG, "k_rot %d", p.k_rot);
  Plan q = p;
  fill_schedule(&q);
  const bool same =
      q.n_ranks == p.n_ranks && !std::memcmp(q.order, p.order, sizeof q.order) &&
      !std::memcmp(q.seg_off, p.seg_off, sizeof q.seg_off) && q.n_half == p.n_half &&
      !std::memcmp(q.hs_width, p.hs_width, sizeof q.hs_width) &&
      !std::memcmp(q.hs_rank0, p.hs_rank0, sizeof q.hs_rank0) &&
      !std::memcmp(q.hs_count, p.hs_count, sizeof q.hs_count) && q.n_class == p.n_class &&
      !std::memcmp(q.cls_w, p.cls_w, sizeof q.cls_w) &&
      !std::memcmp(q.cls_hs0, p.cls_hs0, sizeof q.cls_hs0) &&
      !std::memcmp(q.cls_nhs, p.cls_nhs, sizeof q.cls_nhs) &&
      !std::memcmp(q.cls_last, p.cls_last, sizeof q.cls_last) &&
      !std::memcmp(q.cls_seg0, p.cls_seg0, sizeof q.cls_seg0);
  if (!same) return fail(KVQ_ERR_ARG, "plan order or decode schedule inconsistent with the widths");
  return KVQ_OK;
}

int kvq_plan_build_weighted(const kvq_cfg* cfg, int layer, const double* E_host,
                            const double* Eq_host, int n_q_heads, void* plans_host) {
  int rc = check_cfg(cfg);
  if (rc) return rc;
  const int n_kv = cfg->n_kv_heads;
  if (!E_host || !Eq_host || !plans_host) return fail(KVQ_ERR_ARG, "null pointer");
  if (n_q_heads < 1 || n_q_heads % n_kv != 0)
    return fail(KVQ_ERR_ARG, "n_q_heads %d vs n_kv_heads %d", n_q_heads, n_kv);
  for (int i = 0; i < n_kv * kBlocks; ++i)
    if (!(E_host[i] >= 0.0) || !std::isfinite(E_host[i]))
      return fail(KVQ_ERR_ARG, "energy %d is negative or not finite", i);
  for (int i = 0; i < n_q_heads * kBlocks; ++i)
    if (!(Eq_host[i] >= 0.0) || !std::isfinite(Eq_host[i]))
      return fail(KVQ_ERR_ARG, "query energy %d is negative or not finite", i);
  const int G = n_q_heads / n_kv;
  Plan* out = reinterpret_cast<Plan*>(plans_host);
  for (int h = 0; h < n_kv; ++h) {
    double W[kBlocks];  // the group's mean query energy, summed in increasing g
    for (int j = 0; j < kBlocks; ++j) {
      double acc = 0.0;
      for (int g = 0; g < G; ++g) acc += Eq_host[(size_t)(h * G + g) * kBlocks + j];
      W[j] = acc / G;
    }
    build_plan(cfg, layer, h, E_host + (size_t)h * kBlocks, out + h, W);
  }
  return KVQ_OK;
}

size_t kvq_energy_workspace_bytes(int n_heads) {
  if (n_heads < 1 || n_heads > 65535) return 0;
  return align_up((size_t)n_heads * kBlocks * 16, 256);
}

int kvq_block_energy(const void* x_dev, int dtype, int64_t n_tokens, int n_heads, void* ws_dev,
                     size_t ws_bytes, double* energy_host, uint32_t* status_dev,
                     kvq_stream_t stream) {
  if (!x_dev || !ws_dev || !energy_host) return fail(KVQ_ERR_ARG, "null pointer");
  if (!dtype_ok(dtype)) return fail(KVQ_ERR_ARG, "dtype %d", dtype);
  if (n_tokens < 1) return fail(KVQ_ERR_ARG, "n_tokens %lld < 1", (long long)n_tokens);
  if (n_heads < 1 || n_heads > 65535) return fail(KVQ_ERR_ARG, "n_heads %d", n_heads);
  if (ws_bytes < kvq_energy_workspace_bytes(n_heads))
    return fail(KVQ_ERR_WORKSPACE, "energy workspace too small");
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  auto* acc = reinterpret_cast<unsigned long long*>(ws_dev);
  cudaError_t e = launch_energy(x_dev, dtype, n_tokens, n_heads, acc, status_dev, st);
  if (e != cudaSuccess) return cuda_fail(e, "energy kernel");
  std::vector<unsigned long long> h_acc((size_t)n_heads * kBlocks * 2);
  e = cudaMemcpyAsync(h_acc.data(), acc, h_acc.size() * 8, cudaMemcpyDeviceToHost, st);
  if (e != cudaSuccess) return cuda_fail(e, "energy copy");
  e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(e, "energy sync");
  for (size_t i = 0; i < (size_t)n_heads * kBlocks; ++i) {
    const unsigned __int128 s = ((unsigned __int128)h_acc[2 * i + 1] << 64) | h_acc[2 * i];
    energy_host[i] = std::ldexp((double)s, -32) / (double)n_tokens;
  }
  return KVQ_OK;
}

int kvq_alloc_bits(const kvq_cfg* cfg, int layer, const void* k_dev, int k_dtype, int64_t n_tokens,
                   void* ws_dev, size_t ws_bytes, void* plans_dev, void* plans_host,
                   double* energy_host, uint32_t* status_dev, kvq_stream_t stream) {
  int rc = check_cfg(cfg);
  if (rc) return rc;
  if (!k_dev || !ws_dev || !plans_dev) return fail(KVQ_ERR_ARG, "null device pointer");
  if (!dtype_ok(k_dtype)) return fail(KVQ_ERR_ARG, "k_dtype %d", k_dtype);
  if (n_tokens < 1) return fail(KVQ_ERR_ARG, "n_tokens %lld < 1", (long long)n_tokens);
  if (ws_bytes < kvq_alloc_workspace_bytes(cfg)) return fail(KVQ_ERR_WORKSPACE, "alloc workspace too small");
  const int n_kv = cfg->n_kv_heads;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  auto* acc = reinterpret_cast<unsigned long long*>(ws_dev);
  cudaError_t e = launch_energy(k_dev, k_dtype, n_tokens, n_kv, acc, status_dev, st);
  if (e != cudaSuccess) return cuda_fail(e, "energy kernel");
  std::vector<unsigned long long> h_acc((size_t)n_kv * kBlocks * 2);
  e = cudaMemcpyAsync(h_acc.data(), acc, h_acc.size() * 8, cudaMemcpyDeviceToHost, st);
  if (e != cudaSuccess) return cuda_fail(e, "energy copy");
  e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(e, "energy sync");
  std::vector<double> E((size_t)n_kv * kBlocks);
  for (size_t i = 0; i < E.size(); ++i) {
    const unsigned __int128 s = ((unsigned __int128)h_acc[2 * i + 1] << 64) | h_acc[2 * i];
    E[i] = std::ldexp((double)s, -32) / (double)n_tokens;
  }
  std::vector<Plan> plans(n_kv);
  for (int h = 0; h < n_kv; ++h) build_plan(cfg, layer, h, E.data() + (size_t)h * kBlocks, &plans[h]);
  e = cudaMemcpyAsync(plans_dev, plans.data(), (size_t)n_kv * sizeof(Plan), cudaMemcpyHostToDevice, st);
  if (e != cudaSuccess) return cuda_fail(e, "plan copy");
  e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(e, "plan sync");
  if (plans_host) std::memcpy(plans_host, plans.data(), (size_t)n_kv * sizeof(Plan));
  if (energy_host) std::memcpy(energy_host, E.data(), E.size() * sizeof(double));
  return KVQ_OK;
}

static int quantize_append_impl(const kvq_cfg* cfg, const void* const* plans_dev,
                                const void* k_dev, const void* v_dev, int dtype, int batch,
                                int n_new, const CacheMap& cm, int32_t* len_dev,
                                int64_t cap_tokens, const double* theta, uint32_t* status_dev,
                                kvq_stream_t stream) {
  int rc = check_cfg(cfg);
  if (rc) return rc;
  if (!plans_dev || !(cm.caches || cm.table) || !len_dev || !status_dev)
    return fail(KVQ_ERR_ARG, "null device pointer");
  if (!dtype_ok(dtype)) return fail(KVQ_ERR_ARG, "dtype %d", dtype);
  if (batch < 1 || batch > 65535) return fail(KVQ_ERR_ARG, "batch %d", batch);
  if (n_new < 0 || cap_tokens < 0 || cap_tokens > 0x7FFFFFFF)
    return fail(KVQ_ERR_ARG, "n_new %d / cap_tokens %lld", n_new, (long long)cap_tokens);
  if (n_new == 0) return KVQ_OK;
  if (!k_dev || !v_dev) return fail(KVQ_ERR_ARG, "null k/v pointer");
  if (n_new > (1 << 24)) return fail(KVQ_ERR_ARG, "n_new %d too large", n_new);
  QuantParams p;
  p.plans = reinterpret_cast<const Plan* const*>(plans_dev);
  p.k = k_dev;
  p.v = v_dev;
  p.dtype = dtype;
  p.batch = batch;
  p.n_new = n_new;
  p.n_kv = cfg->n_kv_heads;
  p.cm = cm;
  p.len = len_dev;
  p.cap = cap_tokens;
  p.tile_bytes = tile_bytes(cfg->bits_k, cfg->bits_v);
  p.status = status_dev;
  p.rope = theta ? 1 : 0;
  for (int j = 0; j < 64; ++j) p.theta[j] = theta ? theta[j] : 0.0;
  p.wins = nullptr;
  p.wlen = nullptr;
  p.R = 0;
  cudaError_t e = launch_quantize_append(p, cfg->bits_v, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "quantize_append");
  return KVQ_OK;
}

// RoPE block frequencies theta_j = base^(-2j/128), fp64.
static bool rope_thetas(double base, double* theta) {
  if (!(base > 1.0) || !std::isfinite(base)) return false;
  for (int j = 0; j < 64; ++j) theta[j] = std::pow(base, -2.0 * j / 128.0);
  return true;
}

int kvq_quantize_append(const kvq_cfg* cfg, const void* const* plans_dev, const void* k_dev,
                        const void* v_dev, int dtype, int batch, int n_new, void* const* cache_dev,
                        int32_t* len_dev, int64_t cap_tokens, uint32_t* status_dev,
                        kvq_stream_t stream) {
  return quantize_append_impl(cfg, plans_dev, k_dev, v_dev, dtype, batch, n_new,
                              contiguous_map(cache_dev), len_dev, cap_tokens, nullptr, status_dev,
                              stream);
}

int kvq_quantize_append_rope(const kvq_cfg* cfg, const void* const* plans_dev, const void* k_dev,
                             const void* v_dev, int dtype, int batch, int n_new,
                             void* const* cache_dev, int32_t* len_dev, int64_t cap_tokens,
                             double rope_base, uint32_t* status_dev, kvq_stream_t stream) {
  double theta[64];
  if (!rope_thetas(rope_base, theta)) return fail(KVQ_ERR_ARG, "rope_base %g", rope_base);
  return quantize_append_impl(cfg, plans_dev, k_dev, v_dev, dtype, batch, n_new,
                              contiguous_map(cache_dev), len_dev, cap_tokens, theta, status_dev,
                              stream);
}

}  // extern "C"

namespace {

// kvq_decode_attn and kvq_decode_attn_partial: exactly one of out_dev (final
// outputs) and rec_out (merged records of this context shard) is set.
int decode_impl(const kvq_cfg* cfg, const void* const* plans_dev, const CacheMap& cm,
                const int32_t* len_dev, int batch, int64_t max_len, const void* q_dev, int q_dtype,
                int n_q_heads, float* out_dev, float* rec_out, void* ws_dev, size_t ws_bytes,
                uint32_t* status_dev, kvq_stream_t stream) {
  int rc = check_cfg(cfg);
  if (rc) return rc;
  if (!plans_dev || !(cm.caches || cm.table) || !len_dev || !q_dev || !(out_dev || rec_out) ||
      !ws_dev || !status_dev)
    return fail(KVQ_ERR_ARG, "null device pointer");
  if (rec_out && (reinterpret_cast<uintptr_t>(rec_out) & 15))
    return fail(KVQ_ERR_ARG, "records not 16-byte aligned");
  if (!dtype_ok(q_dtype)) return fail(KVQ_ERR_ARG, "q_dtype %d", q_dtype);
  if (batch < 1 || batch > 65535) return fail(KVQ_ERR_ARG, "batch %d", batch);
  if (max_len < 1 || max_len > 0x7FFFFFFF)
    return fail(KVQ_ERR_ARG, "max_len %lld", (long long)max_len);
  if (n_q_heads < 1 || n_q_heads % cfg->n_kv_heads != 0 || n_q_heads / cfg->n_kv_heads > 16)
    return fail(KVQ_ERR_ARG, "n_q_heads %d vs n_kv_heads %d", n_q_heads, cfg->n_kv_heads);
  if (reinterpret_cast<uintptr_t>(ws_dev) & 15)
    return fail(KVQ_ERR_ARG, "decode workspace not 16-byte aligned");
  if (ws_bytes < kvq_decode_workspace_bytes(cfg, batch, n_q_heads, max_len))
    return fail(KVQ_ERR_WORKSPACE, "decode workspace %zu < %zu", ws_bytes,
                kvq_decode_workspace_bytes(cfg, batch, n_q_heads, max_len));
  cudaError_t e = launch_decode(reinterpret_cast<const Plan* const*>(plans_dev), cm,
                                const_cast<int32_t*>(len_dev), batch, max_len, q_dev, q_dtype,
                                n_q_heads, cfg->n_kv_heads, cfg->bits_k, cfg->bits_v, out_dev,
                                ws_dev, ws_bytes, status_dev, reinterpret_cast<cudaStream_t>(stream),
                                nullptr, nullptr, 0, 0, 0, 0, nullptr, rec_out);
  if (e != cudaSuccess) return cuda_fail(e, rec_out ? "decode_attn_partial" : "decode_attn");
  return KVQ_OK;
}

int append_decode_impl(const kvq_cfg* cfg, const void* const* plans_dev, const void* k_dev,
                       const void* v_dev, int kv_dtype, int n_new, const CacheMap& cm,
                       int32_t* len_dev, int64_t cap_tokens, int batch, int64_t max_len,
                       const void* q_dev, int q_dtype, int n_q_heads, float* out_dev, void* ws_dev,
                       size_t ws_bytes, int step_flags, double rope_base, uint32_t* status_dev,
                       kvq_stream_t stream) {
  int rc = check_cfg(cfg);
  if (rc) return rc;
  if (!plans_dev || !len_dev || !q_dev || !out_dev || !ws_dev || !status_dev)
    return fail(KVQ_ERR_ARG, "null device pointer");
  if (n_new < 0 || n_new > 64) return fail(KVQ_ERR_ARG, "n_new %d not in 0..64", n_new);
  if (n_new > 0 && (!k_dev || !v_dev)) return fail(KVQ_ERR_ARG, "null k/v pointer");
  if (step_flags & ~(KVQ_STEP_EARLY | KVQ_STEP_ROPE))
    return fail(KVQ_ERR_ARG, "step_flags 0x%x", step_flags);
  double theta[64];
  if ((step_flags & KVQ_STEP_ROPE) && !rope_thetas(rope_base, theta))
    return fail(KVQ_ERR_ARG, "rope_base %g", rope_base);
  if (!dtype_ok(kv_dtype) || !dtype_ok(q_dtype)) return fail(KVQ_ERR_ARG, "bad dtype");
  if (batch < 1 || batch > 65535) return fail(KVQ_ERR_ARG, "batch %d", batch);
  if (max_len < 1 || max_len > 0x7FFFFFFF || cap_tokens < 0 || cap_tokens > 0x7FFFFFFF)
    return fail(KVQ_ERR_ARG, "max_len %lld / cap_tokens %lld", (long long)max_len,
                (long long)cap_tokens);
  if (n_q_heads < 1 || n_q_heads % cfg->n_kv_heads != 0 || n_q_heads / cfg->n_kv_heads > 16)
    return fail(KVQ_ERR_ARG, "n_q_heads %d vs n_kv_heads %d", n_q_heads, cfg->n_kv_heads);
  if (reinterpret_cast<uintptr_t>(ws_dev) & 15)
    return fail(KVQ_ERR_ARG, "decode workspace not 16-byte aligned");
  if (ws_bytes < kvq_decode_workspace_bytes(cfg, batch, n_q_heads, max_len))
    return fail(KVQ_ERR_WORKSPACE, "decode workspace %zu < %zu", ws_bytes,
                kvq_decode_workspace_bytes(cfg, batch, n_q_heads, max_len));
  cudaError_t e = launch_decode(reinterpret_cast<const Plan* const*>(plans_dev), cm, len_dev,
                                batch, max_len, q_dev, q_dtype, n_q_heads, cfg->n_kv_heads,
                                cfg->bits_k, cfg->bits_v, out_dev, ws_dev, ws_bytes, status_dev,
                                reinterpret_cast<cudaStream_t>(stream), k_dev, v_dev, kv_dtype,
                                n_new, cap_tokens, (step_flags & KVQ_STEP_EARLY) ? 1 : 0,
                                (step_flags & KVQ_STEP_ROPE) ? theta : nullptr, nullptr);
  if (e != cudaSuccess) return cuda_fail(e, "append_decode");
  return KVQ_OK;
}

// Checks a page description and turns it into the kernels' cache map; the
// capacity of a sequence is its block-table row.
int paged_map(const kvq_cfg* cfg, const kvq_pages* pg, CacheMap* cm, int64_t* cap_tokens) {
  int rc = check_cfg(cfg);
  if (rc) return rc;
  if (!pg || !pg->pool || !pg->block_table) return fail(KVQ_ERR_ARG, "null page description");
  if (reinterpret_cast<uintptr_t>(pg->pool) & 15)
    return fail(KVQ_ERR_ARG, "page pool not 16-byte aligned");
  const size_t pb = kvq_page_bytes(cfg, pg->page_tiles);
  if (pb == 0) return fail(KVQ_ERR_ARG, "page_tiles %d (a power of two, 1..2^20)", pg->page_tiles);
  if (pg->max_pages < 1 || pg->n_pages < 1)
    return fail(KVQ_ERR_ARG, "max_pages %d / n_pages %lld", pg->max_pages,
                (long long)pg->n_pages);
  const int64_t cap = (int64_t)pg->max_pages * pg->page_tiles * 32;
  if (cap > 0x7FFFFFFF) return fail(KVQ_ERR_ARG, "block-table capacity %lld tokens", (long long)cap);
  int shift = 0;
  while ((1 << shift) < pg->page_tiles) ++shift;
  *cm = CacheMap{};
  cm->pool = reinterpret_cast<uint8_t*>(pg->pool);
  cm->table = pg->block_table;
  cm->n_pages = pg->n_pages;
  cm->page_bytes = (int64_t)pb;
  cm->max_pages = pg->max_pages;
  cm->page_shift = shift;
  *cap_tokens = cap;
  return KVQ_OK;
}

}  // namespace

extern "C" {

int kvq_decode_attn(const kvq_cfg* cfg, const void* const* plans_dev, const void* const* cache_dev,
                    const int32_t* len_dev, int batch, int64_t max_len, const void* q_dev,
                    int q_dtype, int n_q_heads, float* out_dev, void* ws_dev, size_t ws_bytes,
                    uint32_t* status_dev, kvq_stream_t stream) {
  if (!out_dev) return fail(KVQ_ERR_ARG, "null device pointer");
  return decode_impl(cfg, plans_dev, contiguous_map(cache_dev), len_dev, batch, max_len, q_dev,
                     q_dtype, n_q_heads, out_dev, nullptr, ws_dev, ws_bytes, status_dev, stream);
}

int kvq_decode_attn_partial(const kvq_cfg* cfg, const void* const* plans_dev,
                            const void* const* cache_dev, const int32_t* len_dev, int batch,
                            int64_t max_len, const void* q_dev, int q_dtype, int n_q_heads,
                            float* rec_dev, void* ws_dev, size_t ws_bytes, uint32_t* status_dev,
                            kvq_stream_t stream) {
  if (!rec_dev) return fail(KVQ_ERR_ARG, "null device pointer");
  return decode_impl(cfg, plans_dev, contiguous_map(cache_dev), len_dev, batch, max_len, q_dev,
                     q_dtype, n_q_heads, nullptr, rec_dev, ws_dev, ws_bytes, status_dev, stream);
}

int kvq_combine_partials(const kvq_cfg* cfg, const void* const* plans_dev, int n_parts,
                         const float* recs_dev, int batch, int n_q_heads, float* out_dev,
                         kvq_stream_t stream) {
  int rc = check_cfg(cfg);
  if (rc) return rc;
  if (!plans_dev || !recs_dev || !out_dev) return fail(KVQ_ERR_ARG, "null device pointer");
  if (reinterpret_cast<uintptr_t>(recs_dev) & 15)
    return fail(KVQ_ERR_ARG, "records not 16-byte aligned");
  if (n_parts < 1 || n_parts > 65535) return fail(KVQ_ERR_ARG, "n_parts %d", n_parts);
  if (batch < 1 || batch > 65535) return fail(KVQ_ERR_ARG, "batch %d", batch);
  if (n_q_heads < 1 || n_q_heads % cfg->n_kv_heads != 0 || n_q_heads / cfg->n_kv_heads > 16)
    return fail(KVQ_ERR_ARG, "n_q_heads %d vs n_kv_heads %d", n_q_heads, cfg->n_kv_heads);
  cudaError_t e = launch_combine(reinterpret_cast<const Plan* const*>(plans_dev), recs_dev,
                                 n_parts, batch, n_q_heads, cfg->n_kv_heads, out_dev,
                                 reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "combine_partials");
  return KVQ_OK;
}

int kvq_debug_decode_stall(long long cycles) {
  if (cycles < 0 || cycles > (1ll << 40)) return fail(KVQ_ERR_ARG, "stall cycles %lld", cycles);
  set_decode_stall(cycles);
  return KVQ_OK;
}

int kvq_set_decode_deterministic(int on) {
  set_decode_deterministic(on);
  return KVQ_OK;
}

// ---------------------------------------------------------- recent window
constexpr int kRecFloats = 132;  // merged record: m, l, 2 unused, o[128]

size_t kvq_window_bytes(const kvq_cfg* cfg, int R) {
  if (check_cfg(cfg) != KVQ_OK || R < 0 || R > (1 << 20)) return 0;
  return (size_t)2 * R * cfg->n_kv_heads * kHeadDim * sizeof(float);
}

int kvq_window_append(const kvq_cfg* cfg, const void* const* plans_dev, const void* k_dev,
                      const void* v_dev, int kv_dtype, int n_new, void* const* cache_dev,
                      int32_t* len_dev, int64_t cap_tokens, void* const* win_dev,
                      int32_t* wlen_dev, int R, int batch, uint32_t* status_dev,
                      kvq_stream_t stream) {
  int rc = check_cfg(cfg);
  if (rc) return rc;
  if (R < 0 || R > (1 << 20)) return fail(KVQ_ERR_ARG, "window R %d", R);
  if (!wlen_dev || (R > 0 && !win_dev)) return fail(KVQ_ERR_ARG, "null window pointer");
  if (R == 0)  // no window: every token is quantized at once
    return quantize_append_impl(cfg, plans_dev, k_dev, v_dev, kv_dtype, batch, n_new,
                                contiguous_map(cache_dev), len_dev, cap_tokens, nullptr,
                                status_dev, stream);
  if (!plans_dev || !cache_dev || !len_dev || !status_dev)
    return fail(KVQ_ERR_ARG, "null device pointer");
  if (!dtype_ok(kv_dtype)) return fail(KVQ_ERR_ARG, "dtype %d", kv_dtype);
  if (batch < 1 || batch > 65535) return fail(KVQ_ERR_ARG, "batch %d", batch);
  if (n_new < 0 || n_new > (1 << 24) || cap_tokens < 0 || cap_tokens > 0x7FFFFFFF)
    return fail(KVQ_ERR_ARG, "n_new %d / cap_tokens %lld", n_new, (long long)cap_tokens);
  if (n_new == 0) return KVQ_OK;
  if (!k_dev || !v_dev) return fail(KVQ_ERR_ARG, "null k/v pointer");
  const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  QuantParams p;
  p.plans = reinterpret_cast<const Plan* const*>(plans_dev);
  p.k = k_dev;
  p.v = v_dev;
  p.dtype = kv_dtype;
  p.batch = batch;
  p.n_new = n_new;
  p.n_kv = cfg->n_kv_heads;
  p.cm = contiguous_map(cache_dev);
  p.len = len_dev;
  p.cap = cap_tokens;
  p.tile_bytes = tile_bytes(cfg->bits_k, cfg->bits_v);
  p.status = status_dev;
  p.rope = 0;
  for (int j = 0; j < 64; ++j) p.theta[j] = 0.0;
  p.wins = reinterpret_cast<const float* const*>(win_dev);
  p.wlen = wlen_dev;
  p.R = R;
  cudaError_t e = launch_quantize_append(p, cfg->bits_v, st);
  if (e != cudaSuccess) return cuda_fail(e, "window_append (evictions)");
  e = launch_window_push(k_dev, v_dev, kv_dtype, n_new, cfg->n_kv_heads, len_dev, wlen_dev,
                         reinterpret_cast<float* const*>(win_dev), R, cap_tokens, batch, st);
  if (e != cudaSuccess) return cuda_fail(e, "window_append (ring)");
  return KVQ_OK;
}

// The packed tokens' records, then up to window_parts_max() window record parts.
static size_t window_records_bytes(int batch, int n_q_heads) {
  return ((size_t)(1 + window_parts_max()) * batch * n_q_heads * kRecFloats * sizeof(float) +
          255) / 256 * 256;
}

size_t kvq_window_decode_workspace_bytes(const kvq_cfg* cfg, int batch, int n_q_heads,
                                         int64_t max_len) {
  const size_t d = kvq_decode_workspace_bytes(cfg, batch, n_q_heads, max_len);
  return d ? d + window_records_bytes(batch, n_q_heads) : 0;
}

int kvq_decode_attn_window(const kvq_cfg* cfg, const void* const* plans_dev,
                           const void* const* cache_dev, const int32_t* len_dev,
                           const void* const* win_dev, const int32_t* wlen_dev, int R, int batch,
                           int64_t max_len, const void* q_dev, int q_dtype, int n_q_heads,
                           float* out_dev, void* ws_dev, size_t ws_bytes, uint32_t* status_dev,
                           kvq_stream_t stream) {
  int rc = check_cfg(cfg);
  if (rc) return rc;
  if (R < 0 || R > (1 << 20)) return fail(KVQ_ERR_ARG, "window R %d", R);
  if (!wlen_dev || (R > 0 && !win_dev) || !out_dev || !ws_dev)
    return fail(KVQ_ERR_ARG, "null device pointer");
  if (batch < 1 || batch > 65535) return fail(KVQ_ERR_ARG, "batch %d", batch);
  if (n_q_heads < 1 || n_q_heads % cfg->n_kv_heads != 0 || n_q_heads / cfg->n_kv_heads > 16)
    return fail(KVQ_ERR_ARG, "n_q_heads %d vs n_kv_heads %d", n_q_heads, cfg->n_kv_heads);
  const size_t rb = window_records_bytes(batch, n_q_heads);
  if (ws_bytes < kvq_window_decode_workspace_bytes(cfg, batch, n_q_heads, max_len))
    return fail(KVQ_ERR_WORKSPACE, "window decode workspace %zu < %zu", ws_bytes,
                kvq_window_decode_workspace_bytes(cfg, batch, n_q_heads, max_len));
  float* recs = reinterpret_cast<float*>(ws_dev);
  float* rec_win = recs + (size_t)batch * n_q_heads * kRecFloats;
  // the packed tokens: one merged record per query head (part 0)
  rc = decode_impl(cfg, plans_dev, contiguous_map(cache_dev), len_dev, batch, max_len, q_dev,
                   q_dtype, n_q_heads, nullptr, recs, reinterpret_cast<uint8_t*>(ws_dev) + rb,
                   ws_bytes - rb, status_dev, stream);
  if (rc) return rc;
  const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = launch_window_record(reinterpret_cast<const Plan* const*>(plans_dev),
                                       reinterpret_cast<const float* const*>(win_dev), len_dev,
                                       wlen_dev, R, q_dev, q_dtype, n_q_heads, cfg->n_kv_heads,
                                       batch, rec_win, st);
  if (e != cudaSuccess) return cuda_fail(e, "decode_attn_window (window)");
  int per_part = 0;
  const int parts = window_parts(R, &per_part);
  e = launch_combine(reinterpret_cast<const Plan* const*>(plans_dev), recs, 1 + parts, batch,
                     n_q_heads, cfg->n_kv_heads, out_dev, st);
  if (e != cudaSuccess) return cuda_fail(e, "decode_attn_window (combine)");
  return KVQ_OK;
}

int kvq_append_decode_window(const kvq_cfg* cfg, const void* const* plans_dev, const void* k_dev,
                             const void* v_dev, int kv_dtype, int n_new, void* const* cache_dev,
                             int32_t* len_dev, int64_t cap_tokens, void* const* win_dev,
                             int32_t* wlen_dev, int R, int batch, int64_t max_len,
                             const void* q_dev, int q_dtype, int n_q_heads, float* out_dev,
                             void* ws_dev, size_t ws_bytes, int step_flags, uint32_t* status_dev,
                             kvq_stream_t stream) {
  int rc = check_cfg(cfg);
  if (rc) return rc;
  if (step_flags & ~KVQ_STEP_EARLY) return fail(KVQ_ERR_ARG, "step_flags 0x%x", step_flags);
  if (R < 0 || R > (1 << 20)) return fail(KVQ_ERR_ARG, "window R %d", R);
  if (R == 0 || n_new < 1 || n_new > std::min(R, 64)) {  // the two calls
    rc = kvq_window_append(cfg, plans_dev, k_dev, v_dev, kv_dtype, n_new, cache_dev, len_dev,
                           cap_tokens, win_dev, wlen_dev, R, batch, status_dev, stream);
    if (rc) return rc;
    return kvq_decode_attn_window(cfg, plans_dev, reinterpret_cast<const void* const*>(cache_dev),
                                  len_dev, reinterpret_cast<const void* const*>(win_dev), wlen_dev,
                                  R, batch, max_len, q_dev, q_dtype, n_q_heads, out_dev, ws_dev,
                                  ws_bytes, status_dev, stream);
  }
  if (!plans_dev || !cache_dev || !len_dev || !win_dev || !wlen_dev || !q_dev || !out_dev ||
      !ws_dev || !status_dev || !k_dev || !v_dev)
    return fail(KVQ_ERR_ARG, "null device pointer");
  if (!dtype_ok(kv_dtype) || !dtype_ok(q_dtype)) return fail(KVQ_ERR_ARG, "bad dtype");
  if (batch < 1 || batch > 65535) return fail(KVQ_ERR_ARG, "batch %d", batch);
  if (max_len < 1 || max_len > 0x7FFFFFFF || cap_tokens < 0 || cap_tokens > 0x7FFFFFFF)
    return fail(KVQ_ERR_ARG, "max_len %lld / cap_tokens %lld", (long long)max_len,
                (long long)cap_tokens);
  if (n_q_heads < 1 || n_q_heads % cfg->n_kv_heads != 0 || n_q_heads / cfg->n_kv_heads > 16)
    return fail(KVQ_ERR_ARG, "n_q_heads %d vs n_kv_heads %d", n_q_heads, cfg->n_kv_heads);
  if (reinterpret_cast<uintptr_t>(ws_dev) & 15)
    return fail(KVQ_ERR_ARG, "decode workspace not 16-byte aligned");
  if (ws_bytes < kvq_window_decode_workspace_bytes(cfg, batch, n_q_heads, max_len))
    return fail(KVQ_ERR_WORKSPACE, "window decode workspace %zu < %zu", ws_bytes,
                kvq_window_decode_workspace_bytes(cfg, batch, n_q_heads, max_len));
  // the fused step uses the decode part of the workspace (after the records)
  const size_t rb = window_records_bytes(batch, n_q_heads);
  cudaError_t e = launch_decode_window(
      reinterpret_cast<const Plan* const*>(plans_dev), contiguous_map(cache_dev), len_dev, batch,
      max_len, q_dev, q_dtype, n_q_heads, cfg->n_kv_heads, cfg->bits_k, cfg->bits_v, out_dev,
      reinterpret_cast<uint8_t*>(ws_dev) + rb, ws_bytes - rb, status_dev,
      reinterpret_cast<cudaStream_t>(stream), k_dev, v_dev, kv_dtype, n_new, cap_tokens,
      (step_flags & KVQ_STEP_EARLY) ? 1 : 0, reinterpret_cast<float* const*>(win_dev), wlen_dev,
      R);
  if (e != cudaSuccess) return cuda_fail(e, "append_decode_window");
  return KVQ_OK;
}

int kvq_append_decode(const kvq_cfg* cfg, const void* const* plans_dev, const void* k_dev,
                      const void* v_dev, int kv_dtype, int n_new, void* const* cache_dev,
                      int32_t* len_dev, int64_t cap_tokens, int batch, int64_t max_len,
                      const void* q_dev, int q_dtype, int n_q_heads, float* out_dev, void* ws_dev,
                      size_t ws_bytes, int step_flags, double rope_base, uint32_t* status_dev,
                      kvq_stream_t stream) {
  if (!cache_dev) return fail(KVQ_ERR_ARG, "null device pointer");
  return append_decode_impl(cfg, plans_dev, k_dev, v_dev, kv_dtype, n_new,
                            contiguous_map(cache_dev), len_dev, cap_tokens, batch, max_len, q_dev,
                            q_dtype, n_q_heads, out_dev, ws_dev, ws_bytes, step_flags, rope_base,
                            status_dev, stream);
}

size_t kvq_page_bytes(const kvq_cfg* cfg, int32_t page_tiles) {
  if (check_cfg(cfg) || page_tiles < 1 || page_tiles > (1 << 20) ||
      (page_tiles & (page_tiles - 1)))
    return 0;
  return (size_t)page_tiles * cfg->n_kv_heads * tile_bytes(cfg->bits_k, cfg->bits_v);
}

int kvq_paged_quantize_append(const kvq_cfg* cfg, const void* const* plans_dev, const void* k_dev,
                              const void* v_dev, int dtype, int batch, int n_new,
                              const kvq_pages* pages, int32_t* len_dev, double rope_base,
                              uint32_t* status_dev, kvq_stream_t stream) {
  CacheMap cm;
  int64_t cap = 0;
  int rc = paged_map(cfg, pages, &cm, &cap);
  if (rc) return rc;
  double theta[64];
  if (rope_base != 0.0 && !rope_thetas(rope_base, theta))
    return fail(KVQ_ERR_ARG, "rope_base %g", rope_base);
  return quantize_append_impl(cfg, plans_dev, k_dev, v_dev, dtype, batch, n_new, cm, len_dev, cap,
                              rope_base != 0.0 ? theta : nullptr, status_dev, stream);
}

int kvq_paged_decode_attn(const kvq_cfg* cfg, const void* const* plans_dev, const kvq_pages* pages,
                          const int32_t* len_dev, int batch, int64_t max_len, const void* q_dev,
                          int q_dtype, int n_q_heads, float* out_dev, void* ws_dev,
                          size_t ws_bytes, uint32_t* status_dev, kvq_stream_t stream) {
  CacheMap cm;
  int64_t cap = 0;
  int rc = paged_map(cfg, pages, &cm, &cap);
  if (rc) return rc;
  if (!out_dev) return fail(KVQ_ERR_ARG, "null device pointer");
  return decode_impl(cfg, plans_dev, cm, len_dev, batch, max_len, q_dev, q_dtype, n_q_heads,
                     out_dev, nullptr, ws_dev, ws_bytes, status_dev, stream);
}

int kvq_paged_decode_attn_partial(const kvq_cfg* cfg, const void* const* plans_dev,
                                  const kvq_pages* pages, const int32_t* len_dev, int batch,
                                  int64_t max_len, const void* q_dev, int q_dtype,
                                  int n_q_heads, float* rec_dev, void* ws_dev, size_t ws_bytes,
                                  uint32_t* status_dev, kvq_stream_t stream) {
  CacheMap cm;
  int64_t cap = 0;
  int rc = paged_map(cfg, pages, &cm, &cap);
  if (rc) return rc;
  if (!rec_dev) return fail(KVQ_ERR_ARG, "null device pointer");
  return decode_impl(cfg, plans_dev, cm, len_dev, batch, max_len, q_dev, q_dtype, n_q_heads,
                     nullptr, rec_dev, ws_dev, ws_bytes, status_dev, stream);
}

int kvq_paged_append_decode(const kvq_cfg* cfg, const void* const* plans_dev, const void* k_dev,
                            const void* v_dev, int kv_dtype, int n_new, const kvq_pages* pages,
                            int32_t* len_dev, int batch, int64_t max_len, const void* q_dev,
                            int q_dtype, int n_q_heads, float* out_dev, void* ws_dev,
                            size_t ws_bytes, int step_flags, double rope_base,
                            uint32_t* status_dev, kvq_stream_t stream) {
  CacheMap cm;
  int64_t cap = 0;
  int rc = paged_map(cfg, pages, &cm, &cap);
  if (rc) return rc;
  return append_decode_impl(cfg, plans_dev, k_dev, v_dev, kv_dtype, n_new, cm, len_dev, cap,
                            batch, max_len, q_dev, q_dtype, n_q_heads, out_dev, ws_dev, ws_bytes,
                            step_flags, rope_base, status_dev, stream);
}

}  // extern "C"

extern "C" {

size_t kvq_bf16_decode_workspace_bytes(int batch, int n_kv_heads, int n_q_heads, int64_t max_len) {
  if (batch < 1 || n_kv_heads < 1 || n_q_heads < 1 || n_q_heads % n_kv_heads != 0 ||
      n_q_heads / n_kv_heads > 16 || max_len < 1)
    return 0;
  return dense_workspace_bytes_for(batch, n_kv_heads, n_q_heads, max_len);
}

int kvq_bf16_decode_attn(const void* k_dev, const void* v_dev, const int32_t* len_dev, int batch,
                         int n_kv_heads, int64_t cap_tokens, int64_t max_len, const void* q_dev,
                         int n_q_heads, float* out_dev, void* ws_dev, size_t ws_bytes,
                         uint32_t* status_dev, kvq_stream_t stream) {
  if (!k_dev || !v_dev || !len_dev || !q_dev || !out_dev || !ws_dev || !status_dev)
    return fail(KVQ_ERR_ARG, "null device pointer");
  if (batch < 1 || batch > 65535) return fail(KVQ_ERR_ARG, "batch %d", batch);
  if (n_kv_heads < 1 || n_kv_heads > 65535) return fail(KVQ_ERR_ARG, "n_kv_heads %d", n_kv_heads);
  if (n_q_heads < 1 || n_q_heads % n_kv_heads != 0 || n_q_heads / n_kv_heads > 16)
    return fail(KVQ_ERR_ARG, "n_q_heads %d vs n_kv_heads %d", n_q_heads, n_kv_heads);
  if (cap_tokens < 1 || max_len < 1 || max_len > 0x7FFFFFFF)
    return fail(KVQ_ERR_ARG, "cap_tokens %lld max_len %lld", (long long)cap_tokens,
                (long long)max_len);
  if ((reinterpret_cast<uintptr_t>(k_dev) | reinterpret_cast<uintptr_t>(v_dev) |
       reinterpret_cast<uintptr_t>(ws_dev)) & 15)
    return fail(KVQ_ERR_ARG, "k, v and workspace must be 16-byte aligned");
  if (reinterpret_cast<uintptr_t>(q_dev) & 3) return fail(KVQ_ERR_ARG, "q must be 4-byte aligned");
  const size_t need = kvq_bf16_decode_workspace_bytes(batch, n_kv_heads, n_q_heads, max_len);
  if (ws_bytes < need)
    return fail(KVQ_ERR_WORKSPACE, "bf16 decode workspace %zu < %zu", ws_bytes, need);
  cudaError_t e = launch_dense_decode(k_dev, v_dev, len_dev, batch, n_kv_heads, cap_tokens,
                                      max_len, q_dev, n_q_heads, out_dev, ws_dev, ws_bytes,
                                      status_dev, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "bf16_decode_attn");
  return KVQ_OK;
}

}  // extern "C"
