// Decode attention for callers that cannot hand the library any scratch
// memory.
//
// kvq_decode_attn needs a workspace for its split partials, and the caller
// provides it. Some callers cannot allocate device memory at the point where
// they decode: a serving loop being recorded into a CUDA graph (cudaMalloc is
// not a capturable operation), an application whose device memory all
// belongs to a pool or arena this library cannot reach, or code that must not
// risk the device-wide synchronization cudaMalloc / cudaFree can cause in the
// middle of a step. kvq_decode_attn_noalloc serves them: it runs the same
// kernels, with the split partials placed in a fixed array that lives in the
// library's own device memory (loaded with the library, held until the
// process exits, on every GPU that uses the library).
#include <cuda_runtime.h>

#include <mutex>

#include "common.cuh"

namespace kvq {
cudaError_t launch_decode(const Plan* const* plans, const CacheMap& cm, int32_t* len,
                          int batch, int64_t max_len, const void* q, int q_dtype, int n_q, int n_kv,
                          int bits_k, int bits_v, float* out, void* ws, size_t ws_bytes,
                          uint32_t* status, cudaStream_t st, const void* k_new, const void* v_new,
                          int kv_dtype, int n_new, int64_t cap, int early, const double* theta,
                          float* rec_out);
int set_last_error(int code, const char* msg);
}  // namespace kvq

namespace {

constexpr size_t kScratchBytes = size_t(16) << 20;  // 16 MiB per device
constexpr int kMaxDevices = 64;

// The scratch itself. In host code this name is only a stand-in for the
// symbol: its device address comes from cudaGetSymbolAddress, per device.
static __device__ __align__(256) unsigned char g_decode_scratch[kScratchBytes];

std::mutex g_mu;
void* g_scratch_addr[kMaxDevices] = {nullptr};

// Device address of the scratch on the current device, looked up once per
// device (with that device current) and cached.
cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_decode_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" KVQ_API size_t kvq_decode_noalloc_scratch_bytes(void) { return kScratchBytes; }

extern "C" KVQ_API int kvq_decode_attn_noalloc(const kvq_cfg* cfg, const void* const* plans_dev,
                                               const void* const* cache_dev,
                                               const int32_t* len_dev, int batch, int64_t max_len,
                                               const void* q_dev, int q_dtype, int n_q_heads,
                                               float* out_dev, uint32_t* status_dev,
                                               kvq_stream_t stream) {
  // The same checks as kvq_decode_attn; the workspace it would need must fit
  // in the fixed scratch.
  const size_t need = kvq_decode_workspace_bytes(cfg, batch, n_q_heads, max_len);
  if (need == 0)
    return kvq::set_last_error(KVQ_ERR_ARG, "kvq_decode_attn_noalloc: invalid cfg, batch, "
                                            "n_q_heads or max_len");
  if (need > kScratchBytes)
    return kvq::set_last_error(KVQ_ERR_WORKSPACE,
                               "kvq_decode_attn_noalloc: this call needs more split-partial "
                               "scratch than the fixed 16 MiB (use kvq_decode_attn with a "
                               "workspace, or fewer sequences / query heads / a smaller max_len)");
  if (!plans_dev || !cache_dev || !len_dev || !q_dev || !out_dev || !status_dev)
    return kvq::set_last_error(KVQ_ERR_ARG, "kvq_decode_attn_noalloc: null device pointer");
  if (q_dtype != KVQ_BF16 && q_dtype != KVQ_FP16 && q_dtype != KVQ_FP32)
    return kvq::set_last_error(KVQ_ERR_ARG, "kvq_decode_attn_noalloc: bad q_dtype");
  if (n_q_heads % cfg->n_kv_heads != 0 || n_q_heads / cfg->n_kv_heads > 16)
    return kvq::set_last_error(KVQ_ERR_ARG, "kvq_decode_attn_noalloc: n_q_heads must be a "
                                            "multiple of n_kv_heads with G <= 16");
  void* scratch = nullptr;
  cudaError_t e = scratch_address(&scratch);
  if (e != cudaSuccess)
    return kvq::set_last_error(KVQ_ERR_CUDA, cudaGetErrorString(e));
  // The scratch is laid out like a workspace: split records (written before
  // they are read) from its start, and the per-(sequence, KV head) counter and
  // bucket blocks, which must be zero when a call starts, at fixed distances
  // from its end. The array is zero when the library is loaded, every
  // completed call clears the blocks it used, and no call's records reach the
  // blocks of another call that fits (kvq.h, kvq_decode_attn).
  e = kvq::launch_decode(reinterpret_cast<const kvq::Plan* const*>(plans_dev),
                         kvq::contiguous_map(cache_dev), const_cast<int32_t*>(len_dev), batch, max_len, q_dev, q_dtype, n_q_heads,
                         cfg->n_kv_heads, cfg->bits_k, cfg->bits_v, out_dev, scratch,
                         kScratchBytes, status_dev, reinterpret_cast<cudaStream_t>(stream),
                         nullptr, nullptr, 0, 0, 0, 0, nullptr, nullptr);
  if (e != cudaSuccess) return kvq::set_last_error(KVQ_ERR_CUDA, cudaGetErrorString(e));
  return KVQ_OK;
}
