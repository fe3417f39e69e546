// Recent-token window beside the packed cache: the most recent R tokens of a
// sequence stay as appended (a ring of fp32 rows), older ones are quantized
// in order as they leave, and decode attends over both.
//
// "RoPE-Aware Bit Allocation for KV-Cache Quantization", abstract: the
// paper's K3V2 result is stated for a packed cache without an fp16
// recent-key buffer, naming such a buffer as an option of the serving path.
// Reading adopted: keys and values of the R most recent tokens are kept
// exactly (the appended 16-bit values, held in fp32), token t in ring slot
// t mod R; a token is quantized with the layer's plan, exactly as without a
// window, once R newer tokens follow it.
//
// * Append: the oldest max(0, wlen + n_new - R) of (window, new tokens) are
//   quantize-appended by the bulk quantize kernel (which reads them from the
//   ring or from the new rows), then window_push_kernel copies the remaining
//   new tokens into the ring and updates both lengths.
// * Decode: the packed tokens give one merged record per query head (the
//   partial decode); window_record_kernel gives the window's record in the
//   same form (base-2 maximum, sum, and o in the value-rotation domain: each
//   window value enters as H (s . v), so the combine's inverse rotation
//   returns it); the combine kernel merges the two records.
#include <algorithm>
#include <atomic>

#include "splitk.cuh"

namespace kvq {

constexpr int kWinThreads = 256;
constexpr int kWinWarps = kWinThreads / 32;

// One CTA per sequence: the new tokens that stay in the window go to their
// ring slots (converted to fp32), then len += evicted, wlen = min(R, wlen +
// n_new). A sequence whose append does not fit the capacity is left as it
// is (the quantize kernel flagged it).
__global__ void __launch_bounds__(kWinThreads) window_push_kernel(
    const void* __restrict__ k, const void* __restrict__ v, int dtype, int n_new, int n_kv,
    int32_t* len, int32_t* wlen, float* const* wins, int R, int64_t cap) {
  const int b = blockIdx.x;
  const int len0 = len[b];
  const int w0 = min(max(wlen[b], 0), R);
  const int n_add = max(0, w0 + n_new - R);
  if (len0 < 0 || (int64_t)len0 + n_add > cap) return;
  const int j0 = max(0, n_add - w0);  // first new token that stays in the window
  const int per_tok = n_kv * kHeadDim;
  if (j0 < n_new) {
    float* wk = wins[b];
    float* wv = wk + (size_t)R * n_kv * kHeadDim;
    const int64_t n_el = (int64_t)(n_new - j0) * per_tok;
    for (int64_t e = threadIdx.x; e < n_el; e += kWinThreads) {
      const int j = j0 + (int)(e / per_tok), x = (int)(e % per_tok);
      const int slot = (int)(((int64_t)len0 + w0 + j) % R);
      const size_t src = ((size_t)b * n_new + j) * per_tok + x;
      wk[(size_t)slot * per_tok + x] = load_as_float(k, dtype, src);
      wv[(size_t)slot * per_tok + x] = load_as_float(v, dtype, src);
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    len[b] = len0 + n_add;
    wlen[b] = min(R, w0 + n_new);
  }
}

// One CTA per (KV head, sequence): the window's record of each of the G
// query heads, (m, l, -, -, o[128]) with m the base-2 maximum logit, l =
// sum 2^(s - m) and o = sum 2^(s - m) H (s . v) (value-rotation domain).
// Warp w takes window tokens w, w + 8, ...; each keeps per head a running
// maximum, sum and o (4 coordinates per lane); the warps merge in shared
// memory. Logits in fp32: s = (q . k) log2(e) / sqrt(128).
__global__ void __launch_bounds__(kWinThreads) window_record_kernel(
    const Plan* const* plans, const float* const* wins, const int32_t* len,
    const int32_t* wlen, int R, const void* __restrict__ q, int q_dtype, int n_q, int n_kv,
    float* __restrict__ recs) {
  extern __shared__ __align__(16) float wsm[];  // q' [G][128], then [warps][G][132]
  const int h = blockIdx.x, b = blockIdx.y, G = n_q / n_kv;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float* qs = wsm;
  float* mg = wsm + G * kHeadDim;
  const Plan& pl = plans[b][h];
  for (int e = threadIdx.x; e < G * kHeadDim; e += kWinThreads)
    qs[e] = load_as_float(q, q_dtype, ((size_t)b * n_q + (size_t)h * G) * kHeadDim + e) *
            0.12751743074f;  // log2(e) / sqrt(128)
  __syncthreads();
  const int w = R > 0 ? min(max(wlen[b], 0), R) : 0;
  const int len0 = max(len[b], 0);
  const float* wk = w > 0 ? wins[b] : nullptr;
  const float* wv = w > 0 ? wk + (size_t)R * n_kv * kHeadDim : nullptr;
  float m[16], l[16], o[16][4];
#pragma unroll
  for (int g = 0; g < 16; ++g) {
    m[g] = -INFINITY;
    l[g] = 0.f;
#pragma unroll
    for (int r = 0; r < 4; ++r) o[g][r] = 0.f;
  }
  for (int t = warp; t < w; t += kWinWarps) {
    const int slot = (int)(((int64_t)len0 + t) % R);
    const size_t row = ((size_t)slot * n_kv + h) * kHeadDim;
    float kx[4], y[4];
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int i = lane + 32 * r;
      kx[r] = wk[row + i];
      const float x = wv[row + i];
      y[r] = ((pl.v_sign[i >> 5] >> (i & 31)) & 1u) ? -x : x;
    }
    // y = H (s . v): butterflies h = 1..16 across lanes, then 32 and 64
#pragma unroll
    for (int hh = 1; hh < 32; hh <<= 1) {
      const bool upper = (lane & hh) != 0;
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const float x = __shfl_xor_sync(0xffffffffu, y[r], hh);
        y[r] = upper ? x - y[r] : y[r] + x;
      }
    }
    {
      const float a0 = y[0] + y[1], a1 = y[0] - y[1], a2 = y[2] + y[3], a3 = y[2] - y[3];
      y[0] = a0 + a2;
      y[2] = a0 - a2;
      y[1] = a1 + a3;
      y[3] = a1 - a3;
    }
#pragma unroll
    for (int g = 0; g < 16; ++g) {
      if (g >= G) break;
      float s = 0.f;
#pragma unroll
      for (int r = 0; r < 4; ++r) s = fmaf(qs[g * kHeadDim + lane + 32 * r], kx[r], s);
#pragma unroll
      for (int mm = 16; mm; mm >>= 1) s += __shfl_xor_sync(0xffffffffu, s, mm);
      const float mn = fmaxf(m[g], s);
      const float a = ex2(m[g] - mn), pr = ex2(s - mn);
      l[g] = l[g] * a + pr;
#pragma unroll
      for (int r = 0; r < 4; ++r) o[g][r] = o[g][r] * a + pr * y[r];
      m[g] = mn;
    }
  }
  // warps -> shared records -> one merged record per head
#pragma unroll
  for (int g = 0; g < 16; ++g) {
    if (g >= G) break;
    float* dst = mg + ((size_t)warp * G + g) * kPartStride;
    if (lane == 0) {
      dst[0] = m[g];
      dst[1] = l[g];
    }
#pragma unroll
    for (int r = 0; r < 4; ++r) dst[kRecO + lane + 32 * r] = o[g][r];
  }
  __syncthreads();
  merge_records<kWinThreads, kWinWarps>(mg, kWinWarps, (size_t)G * kPartStride, G,
                                        recs + ((size_t)b * n_q + (size_t)h * G) * kPartStride);
}

size_t window_record_smem(int G) {
  return ((size_t)G * kHeadDim + (size_t)kWinWarps * G * kPartStride) * sizeof(float);
}

cudaError_t launch_window_push(const void* k, const void* v, int dtype, int n_new, int n_kv,
                               int32_t* len, int32_t* wlen, float* const* wins, int R,
                               int64_t cap, int batch, cudaStream_t st) {
  window_push_kernel<<<batch, kWinThreads, 0, st>>>(k, v, dtype, n_new, n_kv, len, wlen, wins, R,
                                                   cap);
  return cudaGetLastError();
}

cudaError_t launch_window_record(const Plan* const* plans, const float* const* wins,
                                 const int32_t* len, const int32_t* wlen, int R, const void* q,
                                 int q_dtype, int n_q, int n_kv, int batch, float* recs,
                                 cudaStream_t st) {
  static std::atomic<unsigned long long> cap_set{0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const unsigned long long bit = 1ull << (dev & 63);
  if (!(cap_set.load() & bit)) {  // once per device: the largest query group
    e = cudaFuncSetAttribute(window_record_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)window_record_smem(16));
    if (e != cudaSuccess) return e;
    cap_set.fetch_or(bit);
  }
  window_record_kernel<<<dim3(n_kv, batch), kWinThreads, window_record_smem(n_q / n_kv), st>>>(
      plans, wins, len, wlen, R, q, q_dtype, n_q, n_kv, recs);
  return cudaGetLastError();
}

}  // namespace kvq
