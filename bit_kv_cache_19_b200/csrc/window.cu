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
//   partial decode); window_record_kernel gives the window's records in the
//   same form (base-2 maximum, sum, and o in the value-rotation domain: each
//   window value enters as H (s . v), so the combine's inverse rotation
//   returns it), one per part of the window (up to 32 CTAs per KV head and
//   sequence); the combine kernel merges all of them.
#include <algorithm>
#include <atomic>

#include "splitk.cuh"

namespace kvq {

constexpr int kWinThreads = 256;
constexpr int kWinWarps = kWinThreads / 32;
constexpr int kWinParts = 32;  // window record parts per (KV head, sequence), at most

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

// Window records of the G query heads of a (KV head, sequence), split over
// grid.z CTAs: CTA z takes window tokens [z C, z C + C) and writes record
// part z, (m, l, -, -, o[128]) with m the base-2 maximum logit, l =
// sum 2^(s - m) and o = sum 2^(s - m) H (s . v) (value-rotation domain);
// the combine merges the parts with the packed tokens' record. A CTA takes
// its tokens 16 at a time, staged in shared memory: the keys as read, the
// values rotated (two tokens per warp, loads issued together; the fp32
// butterflies of the value quantizer); then one thread per (token, head)
// forms a logit (fp32, s = (q . k) log2(e) / sqrt(128)), one warp per head
// updates the running maximum and sum, and one thread per (coordinate, head
// set) updates o.
constexpr int kWinSub = 16;                // tokens staged at a time
constexpr int kWinKStride = kHeadDim + 1;  // padded key rows (a token per lane, no conflicts)

__global__ void __launch_bounds__(kWinThreads) window_record_kernel(
    const Plan* const* plans, const float* const* wins, const int32_t* len,
    const int32_t* wlen, int R, int C, const void* __restrict__ q, int q_dtype, int n_q,
    int n_kv, int batch, float* __restrict__ recs) {
  __shared__ __align__(16) float qs[16 * kHeadDim];           // q' [G][128]
  __shared__ __align__(16) float ks[kWinSub * kWinKStride];    // staged keys
  __shared__ __align__(16) float ys[kWinSub * kHeadDim];       // staged rotated values
  __shared__ float ps[16 * kWinSub];                           // logits, then weights
  __shared__ float st[48];                                     // max, sum, rescale per head
  const int h = blockIdx.x, b = blockIdx.y, z = blockIdx.z, G = n_q / n_kv;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const Plan& pl = plans[b][h];
  for (int e = tid; e < G * kHeadDim; e += kWinThreads)
    qs[e] = load_as_float(q, q_dtype, ((size_t)b * n_q + (size_t)h * G) * kHeadDim + e) *
            0.12751743074f;  // log2(e) / sqrt(128)
  if (tid < 16) {
    st[tid] = -INFINITY;
    st[16 + tid] = 0.f;
  }
  const int w = R > 0 ? min(max(wlen[b], 0), R) : 0;
  const int len0 = max(len[b], 0);
  const int t_lo = z * C, t_hi = min(w, t_lo + C);
  const float* wk = t_lo < t_hi ? wins[b] : nullptr;
  const float* wv = t_lo < t_hi ? wk + (size_t)R * n_kv * kHeadDim : nullptr;
  const int ci = tid & (kHeadDim - 1), cg = tid >> 7;  // o: coordinate, first head
  const int lt = tid & (kWinSub - 1), lg = tid >> 4;   // logit: token, head
  float o[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) o[k] = 0.f;
  uint32_t vsgn = 0;  // value signs of this lane's coordinates lane + 32 r
#pragma unroll
  for (int r = 0; r < 4; ++r) vsgn |= ((pl.v_sign[r] >> lane) & 1u) << r;
  __syncthreads();
  for (int c0 = t_lo; c0 < t_hi; c0 += kWinSub) {
    const int n = min(kWinSub, t_hi - c0);
    // ---- stage: tokens warp and warp + 8 of the sub-chunk
    {
      float kx[2][4], y[2][4];
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int t = warp + 8 * u;
        if (t < n) {
          const size_t row =
              ((size_t)((int)(((int64_t)len0 + c0 + t) % R)) * n_kv + h) * kHeadDim;
#pragma unroll
          for (int r = 0; r < 4; ++r) {
            kx[u][r] = wk[row + lane + 32 * r];
            const float x = wv[row + lane + 32 * r];
            y[u][r] = ((vsgn >> r) & 1u) ? -x : x;
          }
        }
      }
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int t = warp + 8 * u;
        if (t < n) {  // warp-uniform
#pragma unroll
          for (int r = 0; r < 4; ++r) ks[t * kWinKStride + lane + 32 * r] = kx[u][r];
          // y = H (s . v): butterflies h = 1..16 across lanes, then 32 and 64
#pragma unroll
          for (int hh = 1; hh < 32; hh <<= 1) {
            const bool upper = (lane & hh) != 0;
#pragma unroll
            for (int r = 0; r < 4; ++r) {
              const float x = __shfl_xor_sync(0xffffffffu, y[u][r], hh);
              y[u][r] = upper ? x - y[u][r] : y[u][r] + x;
            }
          }
          const float a0 = y[u][0] + y[u][1], a1 = y[u][0] - y[u][1];
          const float a2 = y[u][2] + y[u][3], a3 = y[u][2] - y[u][3];
          ys[t * kHeadDim + lane] = a0 + a2;
          ys[t * kHeadDim + lane + 32] = a1 + a3;
          ys[t * kHeadDim + lane + 64] = a0 - a2;
          ys[t * kHeadDim + lane + 96] = a1 - a3;
        }
      }
    }
    __syncthreads();
    // ---- logit of token lt for head lg (four partial sums for latency)
    if (lg < G) {
      const float* kr = ks + lt * kWinKStride;
      const float* qr = qs + lg * kHeadDim;
      float a[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 8
      for (int i = 0; i < kHeadDim; i += 4) {
#pragma unroll
        for (int u = 0; u < 4; ++u) a[u] = fmaf(qr[i + u], kr[i + u], a[u]);
      }
      ps[lg * kWinSub + lt] = lt < n ? (a[0] + a[1]) + (a[2] + a[3]) : -INFINITY;
    }
    __syncthreads();
    // ---- one warp per head: running maximum, weights 2^(s - m), sum
    for (int g = warp; g < G; g += kWinWarps) {
      const float s = lane < kWinSub ? ps[g * kWinSub + lane] : -INFINITY;
      float mx = s;
#pragma unroll
      for (int mm = 16; mm; mm >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, mm));
      const float m_old = st[g], m_new = fmaxf(m_old, mx);
      const bool none = m_new == -INFINITY;  // no finite logit yet
      const float pr = none ? 0.f : ex2(s - m_new);
      float sum = pr;
#pragma unroll
      for (int mm = 16; mm; mm >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, mm);
      if (lane < kWinSub) ps[g * kWinSub + lane] = pr;
      if (lane == 0) {
        const float alpha = none ? 1.f : ex2(m_old - m_new);  // 0 from -inf
        st[32 + g] = alpha;
        st[16 + g] = st[16 + g] * alpha + sum;
        st[g] = m_new;
      }
    }
    __syncthreads();
    // ---- o of coordinate ci for heads cg, cg + 2, ...: rescale, add the sub-chunk
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const int g = cg + 2 * k;
      if (g < G) {
        const float* pg = ps + g * kWinSub;
        float acc = o[k] * st[32 + g];
#pragma unroll
        for (int t = 0; t < kWinSub; ++t)
          if (t < n) acc = fmaf(pg[t], ys[t * kHeadDim + ci], acc);
        o[k] = acc;
      }
    }
    __syncthreads();  // the next sub-chunk overwrites the staged rows
  }
  float* dst = recs + ((size_t)z * batch * n_q + (size_t)b * n_q + (size_t)h * G) * kPartStride;
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const int g = cg + 2 * k;
    if (g < G) dst[(size_t)g * kPartStride + kRecO + ci] = o[k];
  }
  if (tid < G) {
    dst[(size_t)tid * kPartStride] = st[tid];
    dst[(size_t)tid * kPartStride + 1] = st[16 + tid];
    dst[(size_t)tid * kPartStride + 2] = 0.f;
    dst[(size_t)tid * kPartStride + 3] = 0.f;
  }
}

// The most window record parts of any call (the workspace is sized for it).
int window_parts_max() { return kWinParts; }

// Window record parts of a window of R tokens: at most kWinParts CTAs per
// (KV head, sequence), each over a multiple of 16 tokens.
int window_parts(int R, int* tokens_per_part) {
  const int P = std::max(1, std::min(kWinParts, (R + kWinSub - 1) / kWinSub));
  const int per = (R + P - 1) / P;
  *tokens_per_part = std::max(kWinSub, (per + kWinSub - 1) / kWinSub * kWinSub);
  return P;
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
  int C = kWinSub;
  const int P = window_parts(R, &C);
  window_record_kernel<<<dim3(n_kv, batch, P), kWinThreads, 0, st>>>(
      plans, wins, len, wlen, R, C, q, q_dtype, n_q, n_kv, batch, recs);
  return cudaGetLastError();
}

}  // namespace kvq
