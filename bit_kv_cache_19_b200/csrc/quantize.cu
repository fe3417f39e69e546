// Block energy and quantize-append kernels.
//
// "RoPE-Aware Bit Allocation for KV-Cache Quantization", abstract: per layer
// and KV head a label-free energy score of each RoPE block drives the greedy
// bit allocation; keys are then quantized with per-block integer widths on
// top of TurboQuant-MSE and values with uniform TQ-MSE, into the packed
// cache of the serving path. Readings adopted (energy on a 2^-32 integer
// grid, fp16 norm, Gaussian Lloyd-Max codes, randomised Hadamard on values,
// tile record layout) are stated in kvq.h.
#include "quant_dev.cuh"

namespace kvq {

// ----------------------------------------------------------------- energy
// acc[h][j] = (lo, hi) 128-bit sum over tokens and the two coordinates of
// block j of min(floor(k^2 2^32), 2^64 - 1). Integer atomics: the total does
// not depend on the order of the additions.
__global__ void __launch_bounds__(128) energy_kernel(const void* __restrict__ k, int dtype,
                                                    int64_t n_tokens, int n_kv, int chunk,
                                                    unsigned long long* __restrict__ acc,
                                                    uint32_t* status) {
  const int h = blockIdx.y;
  const int i = threadIdx.x;  // coordinate
  const int64_t t0 = (int64_t)blockIdx.x * chunk;
  const int64_t t1 = min(n_tokens, t0 + chunk);
  unsigned long long lo = 0, hi = 0;
  bool bad = false;
  for (int64_t t = t0; t < t1; ++t) {
    const float x = load_as_float(k, dtype, ((size_t)t * n_kv + h) * kHeadDim + i);
    unsigned long long term = 0;
    if (isfinite(x)) {
      const double s = (double)x * (double)x * 4294967296.0;  // exact for <= 26-bit significands
      term = s >= 18446744073709551616.0 ? 0xFFFFFFFFFFFFFFFFull : (unsigned long long)s;
    } else {
      bad = true;
    }
    lo += term;
    hi += (lo < term);
  }
  __shared__ unsigned long long s_lo[kHeadDim], s_hi[kHeadDim];
  s_lo[i] = lo;
  s_hi[i] = hi;
  __syncthreads();
  if (i < kBlocks) {
    unsigned long long a = s_lo[i], b = s_lo[i + kBlocks];
    unsigned long long l = a + b;
    unsigned long long hsum = s_hi[i] + s_hi[i + kBlocks] + (l < a);
    unsigned long long* dst = acc + ((size_t)h * kBlocks + i) * 2;
    unsigned long long old = atomicAdd(dst, l);
    if (old + l < old) hsum += 1;
    if (hsum) atomicAdd(dst + 1, hsum);
  }
  if (bad && status) atomicOr(status, KVQ_FLAG_NONFINITE);
}

// --------------------------------------------------------------- quantize
__constant__ float c_thr[KVQ_CB_N_THR] = KVQ_CB_THR;

struct QuantParams {
  const Plan* const* plans;  // [batch] -> [n_kv] plans
  const void* k;
  const void* v;
  int dtype;
  int batch, n_new, n_kv;
  uint8_t* const* caches;  // [batch]
  const int32_t* len;
  int64_t cap;
  int tile_bytes;
  uint32_t* status;
};

// One CTA = the new tokens of one 32-token tile of one (sequence, KV head).
__global__ void __launch_bounds__(256) quantize_append_kernel(QuantParams p) {
  const int b = blockIdx.z, h = blockIdx.y;
  const int len0 = p.len[b];
  if (len0 < 0 || (int64_t)len0 + p.n_new > p.cap) {
    if (threadIdx.x == 0 && blockIdx.x == 0 && h == 0) atomicOr(p.status, KVQ_FLAG_CAPACITY);
    return;
  }
  const int tile = len0 / kTile + blockIdx.x;
  const int t_lo = max(len0, tile * kTile), t_hi = min(len0 + p.n_new, tile * kTile + kTile);
  if (t_lo >= t_hi) return;
  uint8_t* rec = p.caches[b];
  if ((reinterpret_cast<uintptr_t>(rec) & 15) != 0) {
    if (threadIdx.x == 0) atomicOr(p.status, KVQ_FLAG_BAD_PLAN);
    return;
  }
  rec += ((size_t)tile * p.n_kv + h) * p.tile_bytes;

  __shared__ Plan s_plan;
  __shared__ float s_thr[KVQ_CB_N_THR];
  __shared__ uint8_t s_kc[kTile][kHeadDim];
  __shared__ uint8_t s_vc[kTile][kHeadDim];
  __shared__ uint32_t s_flags;
  {
    const uint32_t* src = reinterpret_cast<const uint32_t*>(p.plans[b] + h);
    uint32_t* dst = reinterpret_cast<uint32_t*>(&s_plan);
    for (int i = threadIdx.x; i < KVQ_PLAN_BYTES / 4; i += blockDim.x) dst[i] = src[i];
    for (int i = threadIdx.x; i < KVQ_CB_N_THR; i += blockDim.x) s_thr[i] = c_thr[i];
    if (threadIdx.x == 0) s_flags = 0;
  }
  __syncthreads();
  const Plan& pl = s_plan;
  const int bv = pl.bits_v;
  if (pl.magic != KVQ_PLAN_MAGIC || pl.bits_k < 1 || pl.bits_k > 8 || bv < 1 || bv > 8 ||
      p.tile_bytes != tile_bytes(pl.bits_k, bv)) {
    if (threadIdx.x == 0) atomicOr(p.status, KVQ_FLAG_BAD_PLAN);
    return;
  }

  // ---- codes of the new tokens: one warp per token
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint32_t flags = 0;
  for (int t = t_lo + warp; t < t_hi; t += blockDim.x >> 5) {
    const int tt = t - tile * kTile;
    const size_t row = (((size_t)b * p.n_new + (t - len0)) * p.n_kv + h) * kHeadDim;
    __half kn, vn;
    warp_token_codes(pl, s_thr, p.k, p.v, p.dtype, row, lane, s_kc[tt], s_vc[tt], kn, vn, flags);
    if (lane == 0) {
      __half* norms = reinterpret_cast<__half*>(rec + 512 * (pl.bits_k + bv));
      norms[tt] = kn;
      norms[kTile + tt] = vn;
    }
  }
  if (flags) atomicOr(&s_flags, flags);
  __syncthreads();

  // ---- assemble segment words: keep older tokens' bits, write the new ones,
  //      zero positions past the new length
  const int old_n = max(0, len0 - tile * kTile);  // positions holding older tokens
  assemble_tile_words(reinterpret_cast<uint32_t*>(rec), reinterpret_cast<const uint32_t*>(rec),
                      nullptr, pl, s_kc, s_vc, old_n,
                      t_lo - tile * kTile, t_hi - tile * kTile, threadIdx.x, blockDim.x);
  if (threadIdx.x == 0 && s_flags) atomicOr(p.status, s_flags);
}

__global__ void bump_len_kernel(int32_t* len, int batch, int n_new, int64_t cap) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b < batch && len[b] >= 0 && (int64_t)len[b] + n_new <= cap) len[b] += n_new;
}

// ------------------------------------------------------------- launchers
cudaError_t launch_energy(const void* k, int dtype, int64_t n_tokens, int n_kv,
                          unsigned long long* acc, uint32_t* status, cudaStream_t st) {
  const int chunk = 256;
  const int64_t nchunks = (n_tokens + chunk - 1) / chunk;
  if (nchunks > 0x7FFFFFFF) return cudaErrorInvalidValue;
  cudaError_t e = cudaMemsetAsync(acc, 0, (size_t)n_kv * kBlocks * 16, st);
  if (e != cudaSuccess) return e;
  energy_kernel<<<dim3((unsigned)nchunks, n_kv), 128, 0, st>>>(k, dtype, n_tokens, n_kv, chunk,
                                                                acc, status);
  return cudaGetLastError();
}

cudaError_t launch_quantize_append(const QuantParams& p, cudaStream_t st) {
  const int tiles = (p.n_new + kTile - 1) / kTile + 1;
  quantize_append_kernel<<<dim3(tiles, p.n_kv, p.batch), 256, 0, st>>>(p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  bump_len_kernel<<<(p.batch + 255) / 256, 256, 0, st>>>(const_cast<int32_t*>(p.len), p.batch,
                                                          p.n_new, p.cap);
  return cudaGetLastError();
}

}  // namespace kvq
