// Block energy and quantize-append kernels.
//
// "RoPE-Aware Bit Allocation for KV-Cache Quantization", abstract: per layer
// and KV head a label-free energy score of each RoPE block drives the greedy
// bit allocation; keys are then quantized with per-block integer widths on
// top of TurboQuant-MSE and values with uniform TQ-MSE, into the packed
// cache of the serving path. Readings adopted (energy on a 2^-32 integer
// grid, fp16 norm, Gaussian Lloyd-Max codes, randomised Hadamard on values,
// tile record layout, the optional rotation of keys inside each width group)
// are stated in kvq.h. Tile records are found through the cache map, so the
// same kernel fills contiguous and paged caches.
#include <algorithm>

#include "quant_dev.cuh"

namespace kvq {

// ----------------------------------------------------------------- energy
// Square term of one key element on the 2^-32 grid: floor(x^2 2^32),
// saturating at 2^64 - 1; non-finite elements give 0 and set `bad`. For
// 16-bit inputs x^2 2^32 is exact in fp32 (a square of <= 11 significant
// bits, a power-of-two scale); fp32 inputs use fp64 (48-bit square).
template <bool WIDE>
__device__ __forceinline__ unsigned long long square_term(float x, bool& bad) {
  if (!isfinite(x)) {
    bad = true;
    return 0ull;
  }
  if (!WIDE) {
    const float s = x * x * 4294967296.0f;
    return s >= 18446744073709551616.0f ? 0xFFFFFFFFFFFFFFFFull : (unsigned long long)s;
  }
  const double s = (double)x * (double)x * 4294967296.0;
  return s >= 18446744073709551616.0 ? 0xFFFFFFFFFFFFFFFFull : (unsigned long long)s;
}

// acc[h][j] = (lo, hi) 128-bit sum over tokens and the two coordinates of
// block j of the square terms. One thread per coordinate; 8 tokens' loads
// in flight; the low and high 32-bit halves of the terms are summed apart
// (no carries while streaming) and joined at the end. Integer sums: the
// total does not depend on the order of the additions.
template <bool WIDE>
__global__ void __launch_bounds__(128) energy_kernel(const void* __restrict__ k, int dtype,
                                                    int64_t n_tokens, int n_kv, int chunk,
                                                    unsigned long long* __restrict__ acc,
                                                    uint32_t* status) {
  const int h = blockIdx.y;
  const int i = threadIdx.x;  // coordinate
  const int64_t t0 = (int64_t)blockIdx.x * chunk;
  const int64_t t1 = min(n_tokens, t0 + chunk);
  unsigned long long slo = 0, shi = 0;  // sums of the terms' low / high 32-bit halves
  bool bad = false;
  const size_t stride = (size_t)n_kv * kHeadDim;
  size_t e = ((size_t)t0 * n_kv + h) * kHeadDim + i;
  int64_t t = t0;
  for (; t + 8 <= t1; t += 8, e += 8 * stride) {
    float x[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) x[u] = load_as_float(k, dtype, e + u * stride);
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const unsigned long long term = square_term<WIDE>(x[u], bad);
      slo += term & 0xFFFFFFFFull;
      shi += term >> 32;
    }
  }
  for (; t < t1; ++t, e += stride) {
    const unsigned long long term = square_term<WIDE>(load_as_float(k, dtype, e), bad);
    slo += term & 0xFFFFFFFFull;
    shi += term >> 32;
  }
  // 128-bit value shi 2^32 + slo
  const unsigned long long lo = slo + (shi << 32);
  const unsigned long long hi = (shi >> 32) + (lo < slo ? 1ull : 0ull);
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


// Work item = the new tokens of one 32-token tile of one (sequence, KV head):
// item = (b n_kv + h) tiles_max + i, tile = len0 / 32 + i.
struct Item {
  int b, h, tile, len0, t_lo, t_hi;
  int n_add, w0;  // tokens quantized for the sequence; window tokens among them
  bool fits;      // capacity allows the append
  bool live;      // and the item has tokens to quantize
};

template <bool WIN>
__device__ __forceinline__ Item item_of(const QuantParams& p, int item) {
  Item it;
  const int bh = item / p.tiles_max, ti = item - bh * p.tiles_max;
  it.b = bh / p.n_kv;
  it.h = bh - it.b * p.n_kv;
  it.len0 = p.len[it.b];
  it.w0 = 0;
  it.n_add = p.n_new;
  if (WIN) {
    it.w0 = min(max(p.wlen[it.b], 0), p.R);
    it.n_add = max(0, it.w0 + p.n_new - p.R);
  }
  it.tile = it.len0 / kTile + ti;
  it.t_lo = max(it.len0, it.tile * kTile);
  it.t_hi = min(it.len0 + it.n_add, it.tile * kTile + kTile);
  it.fits = it.len0 >= 0 && (int64_t)it.len0 + it.n_add <= p.cap;
  it.live = it.fits && it.t_lo < it.t_hi;
  return it;
}

// Source rows of the token at position t (>= len0) of an item: the window
// ring (fp32) for the first w0 tokens of a window append, else the new
// tokens' rows (element offsets; returns the dtype).
__device__ __forceinline__ int token_source(const QuantParams& p, const Item& it, int t,
                                            const void*& k, const void*& v, size_t& row) {
  const int i = t - it.len0;
  if (i < it.w0) {
    const int slot = t % p.R;
    const float* w = p.wins[it.b];
    k = w;
    v = w + (size_t)p.R * p.n_kv * kHeadDim;
    row = ((size_t)slot * p.n_kv + it.h) * kHeadDim;
    return KVQ_FP32;
  }
  k = p.k;
  v = p.v;
  row = (((size_t)it.b * p.n_new + (i - it.w0)) * p.n_kv + it.h) * kHeadDim;
  return p.dtype;
}

// Element i of a row of the input type DT (KVQ_BF16 / FP16 / FP32) as fp32.
template <int DT>
__device__ __forceinline__ float in_elem(const void* base, size_t i) {
  if constexpr (DT == KVQ_BF16) return __bfloat162float(static_cast<const __nv_bfloat16*>(base)[i]);
  else if constexpr (DT == KVQ_FP16) return __half2float(static_cast<const __half*>(base)[i]);
  else return static_cast<const float*>(base)[i];
}

// Code of a width-W value from the thresholds held in registers (W <= 3):
// the same binary search as code_of_w, its steps resolved by selects.
template <int W>
__device__ __forceinline__ uint32_t code_of_reg(const float (&t)[7], float z) {
  if constexpr (W == 1) {
    return t[0] < z ? 1u : 0u;
  } else if constexpr (W == 2) {
    const uint32_t c = t[1] < z ? 2u : 0u;
    return c + ((c ? t[2] : t[0]) < z ? 1u : 0u);
  } else {
    const uint32_t c2 = t[3] < z ? 4u : 0u;
    const uint32_t c1 = (c2 ? t[5] : t[1]) < z ? 2u : 0u;
    const float tl = c2 ? (c1 ? t[6] : t[4]) : (c1 ? t[2] : t[0]);
    return c2 + c1 + (tl < z ? 1u : 0u);
  }
}

// Pass 1 of the bulk path for one token (one warp), input type DT known at
// compile time: the arithmetic and decisions of warp_token_pass (fixed
// sum-of-squares tree, IEEE norm and reciprocal, the same butterfly graph),
// with the lane's value signs precomputed (bit q: coordinate lane + 32 q)
// and, for value widths <= 3, the thresholds in registers.
template <int BV, int DT>
__device__ __forceinline__ void bulk_token_pass(const Plan& pl, const float* thr,
                                                const float (&tv)[7], uint32_t vsgn,
                                                const void* k, const void* v, size_t row,
                                                int lane, int p, float* kz_row, uint32_t* words,
                                                bool clear, __half& kn, __half& vn,
                                                uint32_t& flags) {
  float kx[4], vx[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    kx[q] = in_elem<DT>(k, row + lane + 32 * q);
    vx[q] = in_elem<DT>(v, row + lane + 32 * q);
  }
  const bool kfin = __all_sync(0xffffffffu, isfinite(kx[0]) && isfinite(kx[1]) &&
                                                isfinite(kx[2]) && isfinite(kx[3]));
  const bool vfin = __all_sync(0xffffffffu, isfinite(vx[0]) && isfinite(vx[1]) &&
                                                isfinite(vx[2]) && isfinite(vx[3]));
  float kr;
  norm_and_recip(kx, kfin, kn, kr, flags);
  const bool klive = kfin && __half2float(kn) > 0.f;
#pragma unroll
  for (int q = 0; q < 4; ++q)
    kz_row[lane + 32 * q] = klive ? __fmul_rn(kx[q], kr) : __int_as_float(0x7fc00000);
  float vr;
  norm_and_recip(vx, vfin, vn, vr, flags);
  const bool vlive = vfin && __half2float(vn) > 0.f;
  float y[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const float x = vfin ? vx[q] : 0.f;
    y[q] = ((vsgn >> q) & 1u) ? -x : x;
  }
#pragma unroll
  for (int hh = 1; hh < 32; hh <<= 1) {
    const float sg = (lane & hh) ? -1.f : 1.f;
#pragma unroll
    for (int q = 0; q < 4; ++q) y[q] = __fmaf_rn(y[q], sg, __shfl_xor_sync(0xffffffffu, y[q], hh));
  }
  {
    const float a0 = __fadd_rn(y[0], y[1]), a1 = __fsub_rn(y[0], y[1]);
    const float a2 = __fadd_rn(y[2], y[3]), a3 = __fsub_rn(y[2], y[3]);
    y[0] = __fadd_rn(a0, a2);
    y[2] = __fsub_rn(a0, a2);
    y[1] = __fadd_rn(a1, a3);
    y[3] = __fsub_rn(a1, a3);
  }
  uint32_t* vwords = words + kHeadDim * pl.bits_k + ((slot_v(p) * BV) >> 5) + BV * lane;
  const int off = (slot_v(p) * BV) & 31;
  const bool spill = off + BV > 32;
  constexpr uint32_t mask = (1u << BV) - 1u;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint32_t* w = vwords + BV * 32 * q;
    const float z = __fmul_rn(y[q], vr);  // 0 for a dead token (vr = 0)
    uint32_t c;
    if constexpr (BV <= 3) c = code_of_reg<BV>(tv, z);
    else c = (uint32_t)code_of_w<BV>(thr, z);
    c = vlive ? c : 0u;  // a select, not a branch, in the unrolled loop
    if (clear) atomicAnd(w, ~(mask << off));
    atomicOr(w, c << off);
    if (spill) {
      if (clear) atomicAnd(w + 1, ~(mask >> (32 - off)));
      atomicOr(w + 1, c >> (32 - off));
    }
  }
}

// CTAs loop over the work items. A tile's words are assembled in shared
// memory (from zero for a fresh tile, else from the record) by the two passes
// of quant_dev.cuh and written back whole. The plan is reloaded only when
// (b, h) changes. WIN: a window append (rows from the ring or the new tokens,
// token by token); otherwise every row comes from the new tokens, of input
// type DT (-1: any, as p.dtype says; pre-RoPE keys take that path).
template <int BV, bool WIN, int DT>
__global__ void __launch_bounds__(256, 4) quantize_append_kernel(QuantParams p) {
  __shared__ Plan s_plan;
  __shared__ float s_thr[KVQ_CB_N_THR];
  __shared__ float s_kz[kTile * kKzStride];
  __shared__ uint32_t s_words[kHeadDim * 16 + 1];  // + slack word for put_field
  __shared__ uint32_t s_flags;
  __shared__ double s_theta[64];
  __shared__ RotTables s_rot;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  for (int i = threadIdx.x; i < KVQ_CB_N_THR; i += blockDim.x) s_thr[i] = c_thr[i];
  for (int i = threadIdx.x; i < 64; i += blockDim.x) s_theta[i] = p.theta[i];
  if (threadIdx.x == 0) s_flags = 0;
  float tv[7];  // value thresholds in registers (widths <= 3)
#pragma unroll
  for (int i = 0; i < 7; ++i) tv[i] = c_thr[cb_t_off(BV) + min(i, (1 << BV) - 2)];
  uint32_t vsgn = 0;  // value signs of this lane's coordinates lane + 32 q
  int cur = -1;  // (b, h) whose plan is in shared memory
  bool plan_ok = false;
  const int n_items = p.batch * p.n_kv * p.tiles_max;
  for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
    const Item it = item_of<WIN>(p, item);
    const int b = it.b, h = it.h, bh = b * p.n_kv + h, tile = it.tile, len0 = it.len0;
    if (!it.fits) {
      if (threadIdx.x == 0 && item % p.tiles_max == 0 && h == 0)
        atomicOr(p.status, KVQ_FLAG_CAPACITY);
      continue;
    }
    if (!it.live) continue;
    uint8_t* rec = const_cast<uint8_t*>(page_base(p.cm, b, tile));
    if (!rec) {
      if (threadIdx.x == 0) atomicOr(p.status, KVQ_FLAG_BAD_PAGE);
      continue;
    }
    if ((reinterpret_cast<uintptr_t>(rec) & 15) != 0) {
      if (threadIdx.x == 0) atomicOr(p.status, KVQ_FLAG_BAD_PLAN);
      continue;
    }
    rec += ((size_t)(tile & page_mask(p.cm)) * p.n_kv + h) * p.tile_bytes;
    __syncthreads();  // the previous item is done with the shared buffers
    if (bh != cur) {
      const uint32_t* src = reinterpret_cast<const uint32_t*>(p.plans[b] + h);
      uint32_t* dst = reinterpret_cast<uint32_t*>(&s_plan);
      for (int i = threadIdx.x; i < KVQ_PLAN_BYTES / 4; i += blockDim.x) dst[i] = src[i];
      __syncthreads();
      cur = bh;
      plan_ok = s_plan.magic == KVQ_PLAN_MAGIC && s_plan.bits_k >= 1 && s_plan.bits_k <= 8 &&
                s_plan.bits_v == BV && p.tile_bytes == tile_bytes(s_plan.bits_k, BV) &&
                plan_sched_ok(s_plan, lane);
      if (plan_ok && s_plan.k_rot) rot_tables(s_plan, s_rot, threadIdx.x);
      vsgn = 0;
#pragma unroll
      for (int q = 0; q < 4; ++q) vsgn |= ((s_plan.v_sign[q] >> lane) & 1u) << q;
      __syncthreads();
    }
    if (!plan_ok) {
      if (threadIdx.x == 0) atomicOr(p.status, KVQ_FLAG_BAD_PLAN);
      continue;
    }
    const Plan& pl = s_plan;
    const int n_words = kHeadDim * (pl.bits_k + BV);
    const bool clear = len0 > tile * kTile;  // the tile already holds tokens
    uint32_t* gw = reinterpret_cast<uint32_t*>(rec);
    for (int i = threadIdx.x; i < n_words; i += blockDim.x) s_words[i] = clear ? gw[i] : 0u;
    __syncthreads();

    // ---- pass 1: one warp per new token
    const int p_lo = it.t_lo - tile * kTile, p_hi = it.t_hi - tile * kTile;
    uint32_t flags = 0;
    __half* norms = reinterpret_cast<__half*>(rec + 512 * (pl.bits_k + BV));
    for (int pp = p_lo + warp; pp < p_hi; pp += nw) {
      __half kn, vn;
      if (WIN) {
        const void *ks, *vs;
        size_t row;
        const int dt = token_source(p, it, tile * kTile + pp, ks, vs, row);
        warp_token_pass<BV>(pl, s_thr, ks, vs, dt, row, lane, pp, s_kz + pp * kKzStride,
                            s_words, clear, kn, vn, flags);
      } else {
        const size_t row =
            (((size_t)b * p.n_new + (tile * kTile + pp - len0)) * p.n_kv + h) * kHeadDim;
        if constexpr (DT >= 0)
          bulk_token_pass<BV, DT>(pl, s_thr, tv, vsgn, p.k, p.v, row, lane, pp,
                                  s_kz + pp * kKzStride, s_words, clear, kn, vn, flags);
        else
          warp_token_pass<BV>(pl, s_thr, p.k, p.v, p.dtype, row, lane, pp, s_kz + pp * kKzStride,
                              s_words, clear, kn, vn, flags, p.rope ? s_theta : nullptr,
                              (int64_t)tile * kTile + pp);
      }
      if (lane == 0) {
        norms[pp] = kn;
        norms[kTile + pp] = vn;
      }
    }
    if (flags) atomicOr(&s_flags, flags);
    __syncthreads();
    if (pl.k_rot) {  // ---- key rotation inside width groups, one warp per new token
      for (int pp = p_lo + warp; pp < p_hi; pp += nw)
        warp_rotate_row(s_kz + pp * kKzStride, pl, s_rot, pl.g, lane);
      __syncthreads();
    }
    // ---- pass 2: one warp per stored key block
    for (int r = warp; r < pl.n_ranks; r += nw)
      warp_block_pass(pl, s_thr, r, s_kz, p_lo, p_hi, lane, s_words, clear);
    __syncthreads();
    for (int i = threadIdx.x; i < n_words; i += blockDim.x) gw[i] = s_words[i];
  }
  __syncthreads();
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
  if (dtype == KVQ_BF16 || dtype == KVQ_FP16)
    energy_kernel<false><<<dim3((unsigned)nchunks, n_kv), 128, 0, st>>>(k, dtype, n_tokens, n_kv,
                                                                        chunk, acc, status);
  else
    energy_kernel<true><<<dim3((unsigned)nchunks, n_kv), 128, 0, st>>>(k, dtype, n_tokens, n_kv,
                                                                       chunk, acc, status);
  return cudaGetLastError();
}

template <int BV>
static void launch_quant_t(const QuantParams& p, bool win, unsigned grid, cudaStream_t st) {
  if (win) quantize_append_kernel<BV, true, -1><<<grid, 256, 0, st>>>(p);
  else if (p.rope) quantize_append_kernel<BV, false, -1><<<grid, 256, 0, st>>>(p);
  else if (p.dtype == KVQ_BF16) quantize_append_kernel<BV, false, KVQ_BF16><<<grid, 256, 0, st>>>(p);
  else if (p.dtype == KVQ_FP16) quantize_append_kernel<BV, false, KVQ_FP16><<<grid, 256, 0, st>>>(p);
  else quantize_append_kernel<BV, false, KVQ_FP32><<<grid, 256, 0, st>>>(p);
}

cudaError_t launch_quantize_append(const QuantParams& p_in, int bits_v, cudaStream_t st) {
  QuantParams p = p_in;
  p.tiles_max = (p.n_new + kTile - 1) / kTile + 1;
  const int64_t n_items = (int64_t)p.batch * p.n_kv * p.tiles_max;
  if (n_items > 0x7FFFFFFF) return cudaErrorInvalidValue;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    (void)cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  (void)cudaGetLastError();
  const unsigned grid = (unsigned)std::min<int64_t>(n_items, (int64_t)4 * sms);  // resident
  const bool win = p.wins != nullptr;
  switch (bits_v) {
    case 1: launch_quant_t<1>(p, win, grid, st); break;
    case 2: launch_quant_t<2>(p, win, grid, st); break;
    case 3: launch_quant_t<3>(p, win, grid, st); break;
    case 4: launch_quant_t<4>(p, win, grid, st); break;
    case 5: launch_quant_t<5>(p, win, grid, st); break;
    case 6: launch_quant_t<6>(p, win, grid, st); break;
    case 7: launch_quant_t<7>(p, win, grid, st); break;
    case 8: launch_quant_t<8>(p, win, grid, st); break;
    default: return cudaErrorInvalidValue;
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (p.wins) return cudaSuccess;  // the window's ring kernel updates the lengths
  bump_len_kernel<<<(p.batch + 255) / 256, 256, 0, st>>>(const_cast<int32_t*>(p.len), p.batch,
                                                          p.n_new, p.cap);
  return cudaGetLastError();
}

}  // namespace kvq
