// Block energy and quantize-append kernels.
//
// "RoPE-Aware Bit Allocation for KV-Cache Quantization", abstract: per layer
// and KV head a label-free energy score of each RoPE block drives the greedy
// bit allocation; keys are then quantized with per-block integer widths on
// top of TurboQuant-MSE and values with uniform TQ-MSE, into the packed
// cache of the serving path. Readings adopted (energy on a 2^-32 integer
// grid, fp16 norm, Gaussian Lloyd-Max codes, randomised Hadamard on values,
// tile record layout) are stated in kvq.h.
#include "common.cuh"

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

// Number of width-w thresholds strictly below z (NaN -> 0): branch-free
// binary search over the sorted 2^w - 1 thresholds.
__device__ __forceinline__ int code_of(const float* thr, int w, float z) {
  const float* t = thr + cb_t_off(w);
  int c = 0;
  for (int step = 1 << (w - 1); step; step >>= 1)
    if (t[c + step - 1] < z) c += step;
  return c;
}

// Fixed-order fp32 sum of squares of a 128-vector held as v[q] = x[lane + 32 q]:
// p = ((v0^2 + v1^2) + v2^2) + v3^2, then p += p(lane ^ m) for m = 16..1.
__device__ __forceinline__ float sumsq_tree(const float (&v)[4]) {
  float p = __fadd_rn(__fadd_rn(__fadd_rn(__fmul_rn(v[0], v[0]), __fmul_rn(v[1], v[1])),
                                __fmul_rn(v[2], v[2])),
                      __fmul_rn(v[3], v[3]));
#pragma unroll
  for (int m = 16; m; m >>= 1) p = __fadd_rn(p, __shfl_xor_sync(0xffffffffu, p, m));
  return p;
}

// Norm n (fp16 value), reciprocal r, flags, for a warp-held 128-vector.
__device__ __forceinline__ void norm_and_recip(const float (&v)[4], bool finite, __half& n16,
                                               float& r, uint32_t& flags) {
  if (!finite) {
    n16 = __float2half_rn(0.f);
    r = 0.f;
    flags |= KVQ_FLAG_NONFINITE;
    return;
  }
  const float s = __fsqrt_rn(sumsq_tree(v));
  n16 = __float2half_rn(s);
  if (__hisinf(n16)) {
    n16 = __ushort_as_half((unsigned short)0x7BFF);  // 65504
    flags |= KVQ_FLAG_NORM_SAT;
  }
  const float n = __half2float(n16);
  r = n > 0.f ? __frcp_rn(n) : 0.f;
}

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
    float kx[4], vx[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      kx[q] = load_as_float(p.k, p.dtype, row + lane + 32 * q);
      vx[q] = load_as_float(p.v, p.dtype, row + lane + 32 * q);
    }
    const bool kfin = __all_sync(0xffffffffu, isfinite(kx[0]) && isfinite(kx[1]) &&
                                                  isfinite(kx[2]) && isfinite(kx[3]));
    const bool vfin = __all_sync(0xffffffffu, isfinite(vx[0]) && isfinite(vx[1]) &&
                                                  isfinite(vx[2]) && isfinite(vx[3]));
    // keys: z_i = (k_i r) g_j, width b_j
    __half kn;
    float kr;
    norm_and_recip(kx, kfin, kn, kr, flags);
    const bool klive = kfin && __half2float(kn) > 0.f;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int i = lane + 32 * q, j = i & 63, w = pl.width[j];
      int c = 0;
      if (w > 0 && klive) c = code_of(s_thr, w, __fmul_rn(__fmul_rn(kx[q], kr), pl.g[j]));
      s_kc[tt][i] = (uint8_t)c;
    }
    // values: y = H (s . v) by the fixed fp32 butterfly graph, z = y r
    __half vn;
    float vr;
    norm_and_recip(vx, vfin, vn, vr, flags);
    const bool vlive = vfin && __half2float(vn) > 0.f;
    float y[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int i = lane + 32 * q;
      const float x = vfin ? vx[q] : 0.f;
      y[q] = ((pl.v_sign[i >> 5] >> (i & 31)) & 1u) ? -x : x;
    }
#pragma unroll
    for (int hh = 1; hh < 32; hh <<= 1) {
      const bool upper = (lane & hh) != 0;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float o = __shfl_xor_sync(0xffffffffu, y[q], hh);
        y[q] = upper ? __fsub_rn(o, y[q]) : __fadd_rn(y[q], o);
      }
    }
    {  // h = 32: (q0, q1), (q2, q3); h = 64: (q0, q2), (q1, q3)
      float a0 = __fadd_rn(y[0], y[1]), a1 = __fsub_rn(y[0], y[1]);
      float a2 = __fadd_rn(y[2], y[3]), a3 = __fsub_rn(y[2], y[3]);
      y[0] = __fadd_rn(a0, a2);
      y[2] = __fsub_rn(a0, a2);
      y[1] = __fadd_rn(a1, a3);
      y[3] = __fsub_rn(a1, a3);
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      int c = 0;
      if (vlive) c = code_of(s_thr, bv, __fmul_rn(y[q], vr));
      s_vc[tt][lane + 32 * q] = (uint8_t)c;
    }
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
  const int new_lo = t_lo - tile * kTile, new_hi = t_hi - tile * kTile;
  uint32_t* words = reinterpret_cast<uint32_t*>(rec);
  const int words_k = 128 * pl.bits_k;
  for (int wi = threadIdx.x; wi < words_k + 128 * bv; wi += blockDim.x) {
    int f, k, jj = 0, w = 0, pcoord = 0;
    bool is_k = wi < words_k;
    if (is_k) {
      int lo = 0, hi = pl.n_ranks;  // largest rank r with seg_off[r] <= wi
      while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (pl.seg_off[mid] <= wi) lo = mid; else hi = mid;
      }
      jj = pl.order[lo];
      w = pl.width[jj];
      f = 2 * w;
      k = wi - pl.seg_off[lo];
    } else {
      pcoord = (wi - words_k) / bv;
      k = (wi - words_k) - pcoord * bv;
      f = bv;
    }
    uint32_t nw = 0, keep = 0;
    const int s0 = (32 * k) / f, s1 = (32 * k + 31) / f;
    for (int s = s0; s <= s1 && s < kTile; ++s) {
      const int tok = is_k ? token_of_slot_k(s) : token_of_slot_v(s);
      const int fb = s * f - 32 * k + 32;  // bit position + 32, in (32 - f, 64)
      uint32_t field;
      if (tok >= new_lo && tok < new_hi) {
        field = is_k ? (uint32_t)s_kc[tok][jj] | ((uint32_t)s_kc[tok][jj + 64] << w)
                     : (uint32_t)s_vc[tok][pcoord];
        nw |= (uint32_t)(((unsigned long long)field << fb) >> 32);
      } else if (tok < old_n) {
        field = (f == 32) ? 0xFFFFFFFFu : ((1u << f) - 1u);
        keep |= (uint32_t)(((unsigned long long)field << fb) >> 32);
      }
    }
    words[wi] = keep ? ((words[wi] & keep) | nw) : nw;
  }
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
