// Packed-cache decode attention (split-K) and the split combine.
//
// "RoPE-Aware Bit Allocation for KV-Cache Quantization", abstract: the
// packed-cache serving path runs decode attention directly on the packed
// K/V cache (the pages report it faster than fp16 FlashAttention2 at 128K on
// H800). This is an sm_100a design of its own:
//
// * Work: CTA = (split, KV head, sequence), 4 warps; each warp owns every 4th
//   32-token tile of the CTA's range and streams its tiles into a private
//   3-stage shared-memory ring with 1-D bulk copies (cp.async.bulk +
//   mbarrier, no multicast).
// * Keys: the tile's codes are unpacked straight into the A fragments of
//   mma.sync m16n8k16 (16 tokens x 16 plan-ordered coordinates): each 32-bit
//   register is one RoPE block (codes of coordinates j and j + 64) of one
//   token, looked up as an fp16 pair. The B operand is the query group
//   (G <= 16 heads) pre-multiplied by the block scales a_hat_j, log2(e) and
//   1/sqrt(128), split into hi + lo fp16 parts so the logits keep fp32
//   accuracy. Width-uniform half k-steps (<= 4 blocks of one width) let the
//   unpack use compile-time shifts.
// * Softmax: base-2 online softmax per head on the fp32 accumulators, scaled
//   by the fp16 key norms; masked positions past the sequence length.
// * Values: P' = p * n^V (fp16) is transposed in registers (movmatrix) into
//   the B operand of O^T(128 x G) += Vhat^T(128 x 16 tokens) P'^T, where
//   Vhat^T's fragments (one rotated coordinate, two tokens) come from the
//   value tile's pair codes. Output stays in the rotated value domain.
// * Combine: merges the (m, l, o) partials of all splits, applies the inverse
//   randomised Hadamard transform and 1/l.
#include <algorithm>
#include <atomic>

#include "common.cuh"

namespace kvq {

__constant__ uint16_t c_c16[KVQ_CB_N_C16] = KVQ_CB_C16;

constexpr int kWarps = 4;
constexpr int kStages = 3;
constexpr int kMaxK = 12;       // k-steps of 16 coordinates (2 half-steps each)
constexpr int kPairLut = 340;   // pair tables of widths 1..4: 4 + 16 + 64 + 256
constexpr int kPartStride = 130;

__host__ __device__ constexpr int pair_off(int w) { return ((1 << (2 * w)) - 4) / 3; }

struct DecodeParams {
  const Plan* const* plans;
  const uint8_t* const* caches;
  const int32_t* len;
  const void* q;
  int q_dtype;
  int n_q, n_kv, G;
  int max_len;
  int n_splits, tiles_per_split;
  int tile_bytes;
  float* part;  // [batch][n_q][n_splits][130] = m, l, o[128]
  uint32_t* status;
};

struct alignas(128) Smem {
  Plan plan;
  uint32_t lut_pair[kPairLut];      // fp16 pairs (c[lo], c[hi]) for widths 1..4
  uint16_t lut1[KVQ_CB_N_C16];      // fp16 centroids, width w at 2^w - 2
  float inv_scale[16];              // 2^-sigma of each head's q' scaling
  uint32_t flags;
  uint4 qfrag[2][kMaxK][32];        // per (n-tile, k-step, lane): hi b0, hi b1, lo b0, lo b1
  unsigned long long bar[kWarps][kStages];
  float qp[16][kHeadDim];           // q' (fp32) of the head group
};

template <int W>
__device__ __forceinline__ uint32_t pair_lookup(const Smem& sm, uint32_t f) {
  if constexpr (W <= 4) {
    return sm.lut_pair[pair_off(W) + f];
  } else {
    const uint16_t* t = sm.lut1 + cb_c_off(W);
    return (uint32_t)t[f & ((1u << W) - 1u)] | ((uint32_t)t[f >> W] << 16);
  }
}

// Four 2W-bit pair fields at bits [8Wq, 8Wq + 8W) of a segment, as fp16 pairs.
template <int W>
__device__ __forceinline__ void fields4(const Smem& sm, const uint32_t* seg, int q,
                                        uint32_t (&out)[4]) {
  const int bit = 8 * W * q;
  const uint32_t* wp = seg + (bit >> 5);
  const uint32_t sh = bit & 31;
  constexpr uint32_t mask = (1u << (2 * W)) - 1u;
  if constexpr (W <= 4) {
    const uint32_t v = funnel_r(wp[0], wp[1], sh);
#pragma unroll
    for (int i = 0; i < 4; ++i) out[i] = pair_lookup<W>(sm, (v >> (2 * W * i)) & mask);
  } else {
    const uint32_t lo = funnel_r(wp[0], wp[1], sh), hi = funnel_r(wp[1], wp[2], sh);
    const unsigned long long v = ((unsigned long long)hi << 32) | lo;
#pragma unroll
    for (int i = 0; i < 4; ++i) out[i] = pair_lookup<W>(sm, (uint32_t)(v >> (2 * W * i)) & mask);
  }
}

// Key fragments of one half k-step: block (rank0 + c) of width w, tokens
// g, g + 8, g + 16, g + 24 (K slots 4g .. 4g + 3).
__device__ __forceinline__ void key_half(const Smem& sm, const uint32_t* kw, int hs, int g, int c,
                                         uint32_t (&o)[4]) {
  o[0] = o[1] = o[2] = o[3] = 0u;
  if (hs >= sm.plan.n_half || c >= sm.plan.hs_count[hs]) return;
  const uint32_t* seg = kw + sm.plan.seg_off[sm.plan.hs_rank0[hs] + c];
  switch (sm.plan.hs_width[hs]) {
    case 1: fields4<1>(sm, seg, g, o); break;
    case 2: fields4<2>(sm, seg, g, o); break;
    case 3: fields4<3>(sm, seg, g, o); break;
    case 4: fields4<4>(sm, seg, g, o); break;
    case 5: fields4<5>(sm, seg, g, o); break;
    case 6: fields4<6>(sm, seg, g, o); break;
    case 7: fields4<7>(sm, seg, g, o); break;
    default: fields4<8>(sm, seg, g, o); break;
  }
}

__device__ __forceinline__ void write_empty_partial(const DecodeParams& p, int b, int h, int split) {
  for (int head = 0; head < p.G; ++head) {
    float* dst = p.part + (((size_t)b * p.n_q + h * p.G + head) * p.n_splits + split) * kPartStride;
    for (int i = threadIdx.x; i < kPartStride; i += blockDim.x)
      dst[i] = i == 0 ? -INFINITY : 0.f;
  }
}

template <int BV, int NT>
__global__ void __launch_bounds__(kWarps * 32) decode_kernel(const DecodeParams p) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>(smem_raw);
  uint8_t* const stage_base = smem_raw + sizeof(Smem);

  const int split = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, c = lane & 3;

  // ---- plan and lookup tables
  {
    const uint4* src = reinterpret_cast<const uint4*>(p.plans[b] + h);
    uint4* dst = reinterpret_cast<uint4*>(&sm.plan);
    for (int i = tid; i < KVQ_PLAN_BYTES / 16; i += blockDim.x) dst[i] = src[i];
    for (int i = tid; i < KVQ_CB_N_C16; i += blockDim.x) sm.lut1[i] = c_c16[i];
    for (int i = tid; i < kPairLut; i += blockDim.x) {
      int w = 1;
      while (w < 4 && i >= pair_off(w + 1)) ++w;
      const int f = i - pair_off(w);
      const uint32_t lo = c_c16[cb_c_off(w) + (f & ((1 << w) - 1))];
      const uint32_t hi = c_c16[cb_c_off(w) + (f >> w)];
      sm.lut_pair[i] = lo | (hi << 16);
    }
    if (tid == 0) sm.flags = 0u;
  }
  __syncthreads();
  const uint8_t* cache = p.caches[b];
  const int bk = sm.plan.bits_k;
  if (sm.plan.magic != KVQ_PLAN_MAGIC || sm.plan.bits_v != BV || bk < 1 || bk > 8 ||
      p.tile_bytes != tile_bytes(bk, BV) || sm.plan.n_half > 2 * kMaxK ||
      (reinterpret_cast<uintptr_t>(cache) & 15) != 0) {
    if (tid == 0) atomicOr(p.status, KVQ_FLAG_BAD_PLAN);
    write_empty_partial(p, b, h, split);
    return;
  }
  int L = p.len[b];
  if (L > p.max_len) {
    if (tid == 0 && split == 0 && h == 0) atomicOr(p.status, KVQ_FLAG_CAPACITY);
    L = p.max_len;
  }
  L = max(L, 0);
  const int n_tiles = (L + kTile - 1) / kTile;
  const int tb = split * p.tiles_per_split;
  const int te = min(n_tiles, tb + p.tiles_per_split);
  if (tb >= te) {
    write_empty_partial(p, b, h, split);
    return;
  }

  // ---- query prologue: q' = q a_hat_j log2(e) / sqrt(128), per-head 2^sigma
  //      scaling into the fp16 range, hi/lo split into B fragments
  const int G = p.G;
  for (int i = tid; i < 16 * kHeadDim; i += blockDim.x) {
    const int head = i >> 7, x = i & 127;
    float v = 0.f;
    if (head < G) {
      const size_t qi = ((size_t)b * p.n_q + h * G + head) * kHeadDim + x;
      v = load_as_float(p.q, p.q_dtype, qi) * sm.plan.a_hat[x & 63] * 0.12751743074f;
    }
    sm.qp[head][x] = v;  // 0.12751743 = log2(e) / sqrt(128)
  }
  __syncthreads();
  for (int head = warp; head < 16; head += kWarps) {
    float mx = 0.f;
    for (int x = lane; x < kHeadDim; x += 32) mx = fmaxf(mx, fabsf(sm.qp[head][x]));
#pragma unroll
    for (int m = 16; m; m >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, m));
    const int sigma = (mx > 0.f && isfinite(mx)) ? 14 - ilogbf(mx) : 0;
    const float sc = ldexpf(1.f, sigma);
    for (int x = lane; x < kHeadDim; x += 32) sm.qp[head][x] *= sc;
    if (lane == 0) sm.inv_scale[head] = ldexpf(1.f, -sigma);
  }
  __syncthreads();
  const int n_half = sm.plan.n_half;
  const int n_k = (n_half + 1) >> 1;
  for (int e = tid; e < NT * n_k * 32; e += blockDim.x) {
    const int ln = e & 31, ks = (e >> 5) % n_k, nt = (e >> 5) / n_k;
    const int head = 8 * nt + (ln >> 2), cc = ln & 3;
    float x[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const int hs = 2 * ks + half;
      if (hs < n_half && cc < sm.plan.hs_count[hs]) {
        const int j = sm.plan.order[sm.plan.hs_rank0[hs] + cc];
        x[2 * half] = sm.qp[head][j];
        x[2 * half + 1] = sm.qp[head][j + 64];
      }
    }
    const uint32_t hi0 = pack_half2(x[0], x[1]), hi1 = pack_half2(x[2], x[3]);
    const __half2 h0 = *reinterpret_cast<const __half2*>(&hi0);
    const __half2 h1 = *reinterpret_cast<const __half2*>(&hi1);
    const uint32_t lo0 = pack_half2(x[0] - __low2float(h0), x[1] - __high2float(h0));
    const uint32_t lo1 = pack_half2(x[2] - __low2float(h1), x[3] - __high2float(h1));
    sm.qfrag[nt][ks][ln] = make_uint4(hi0, hi1, lo0, lo1);
  }
  if (tid < kWarps * kStages) mbar_init(&sm.bar[tid / kStages][tid % kStages], 1);
  fence_proxy_async();
  __syncthreads();

  // ---- per-warp pipeline over the warp's tiles
  const int tbytes = p.tile_bytes;
  uint8_t* const my_stages = stage_base + (size_t)warp * kStages * tbytes;
  const int n_mine = max(0, (te - tb - warp + kWarps - 1) / kWarps);
  auto tile_of = [&](int i) { return tb + warp + i * kWarps; };
  auto issue = [&](int i) {
    const int s = i % kStages;
    unsigned long long* bar = &sm.bar[warp][s];
    mbar_expect_tx(bar, (uint32_t)tbytes);
    bulk_g2s(my_stages + s * tbytes, cache + ((size_t)tile_of(i) * p.n_kv + h) * tbytes,
             (uint32_t)tbytes, bar);
  };
  if (lane == 0)
    for (int i = 0; i < min(kStages, n_mine); ++i) issue(i);
  __syncwarp();

  float o[8][NT][4];
  float m_run[NT][2], l_run[NT][2];
#pragma unroll
  for (int mu = 0; mu < 8; ++mu)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int r = 0; r < 4; ++r) o[mu][nt][r] = 0.f;
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      m_run[nt][e] = -INFINITY;
      l_run[nt][e] = 0.f;
    }

  int consumed = 0;
  bool timed_out = false;
  for (int i = 0; i < n_mine; ++i) {
    const int s = i % kStages;
    const bool ok = mbar_wait_bounded(&sm.bar[warp][s], (uint32_t)((i / kStages) & 1));
    if (!__all_sync(0xffffffffu, ok)) {
      timed_out = true;
      break;
    }
    consumed = i + 1;
    const int tile = tile_of(i);
    const int nvalid = min(kTile, L - tile * kTile);
    const uint32_t* kw = reinterpret_cast<const uint32_t*>(my_stages + s * tbytes);
    const uint32_t* vw = kw + 128 * bk;
    const __half* nrm = reinterpret_cast<const __half*>(vw + 128 * BV);

    // keys: S[32 tokens x 8 NT heads] on the tensor cores
    float sacc[2][NT][4];
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int r = 0; r < 4; ++r) sacc[mt][nt][r] = 0.f;
    for (int ks = 0; ks < n_k; ++ks) {
      uint32_t A0[4], A1[4];
      key_half(sm, kw, 2 * ks, g, c, A0);
      key_half(sm, kw, 2 * ks + 1, g, c, A1);
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const uint4 qf = sm.qfrag[nt][ks][lane];
        mma_16816(sacc[0][nt], A0[0], A0[1], A1[0], A1[1], qf.x, qf.y);
        mma_16816(sacc[0][nt], A0[0], A0[1], A1[0], A1[1], qf.z, qf.w);
        mma_16816(sacc[1][nt], A0[2], A0[3], A1[2], A1[3], qf.x, qf.y);
        mma_16816(sacc[1][nt], A0[2], A0[3], A1[2], A1[3], qf.z, qf.w);
      }
    }

    // online softmax (base 2); this thread's tokens are g + 8 r, r = 0..3
    float nk[4], nv[4];
    bool val[4];
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int tok = g + 8 * r;
      val[r] = tok < nvalid;
      nk[r] = val[r] ? __half2float(nrm[tok]) : 0.f;
      nv[r] = val[r] ? __half2float(nrm[kTile + tok]) : 0.f;
    }
    uint32_t pb0[2][NT], pb1[2][NT];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      float pe[2][4];
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const float isc = sm.inv_scale[8 * nt + 2 * c + e];
        float sv[4];
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const int mt = r >> 1, rr = r & 1;
          sv[r] = val[r] ? sacc[mt][nt][2 * rr + e] * nk[r] * isc : -INFINITY;
        }
        float mx = fmaxf(fmaxf(sv[0], sv[1]), fmaxf(sv[2], sv[3]));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
        const float m_new = fmaxf(m_run[nt][e], mx);
        float alpha = 1.f, lsum = 0.f;
        if (m_new != -INFINITY) {
          alpha = exp2f(m_run[nt][e] - m_new);
#pragma unroll
          for (int r = 0; r < 4; ++r) {
            const float pr = exp2f(sv[r] - m_new);
            lsum += pr;
            pe[e][r] = val[r] ? pr * nv[r] : 0.f;
          }
        } else {
#pragma unroll
          for (int r = 0; r < 4; ++r) pe[e][r] = 0.f;
        }
        l_run[nt][e] = l_run[nt][e] * alpha + lsum;
        m_run[nt][e] = m_new;
        if (alpha != 1.f) {
#pragma unroll
          for (int mu = 0; mu < 8; ++mu) {
            o[mu][nt][e] *= alpha;
            o[mu][nt][2 + e] *= alpha;
          }
        }
      }
#pragma unroll
      for (int mt = 0; mt < 2; ++mt) {
        pb0[mt][nt] = movmatrix_trans(pack_half2(pe[0][2 * mt], pe[1][2 * mt]));
        pb1[mt][nt] = movmatrix_trans(pack_half2(pe[0][2 * mt + 1], pe[1][2 * mt + 1]));
      }
    }

    // values: O^T[128 x 8 NT] += Vhat^T[128 x 32 tokens] P'^T
#pragma unroll
    for (int mu = 0; mu < 8; ++mu) {
      uint32_t F0[4], F1[4];
      fields4<BV>(sm, vw + (16 * mu + g) * BV, c, F0);
      fields4<BV>(sm, vw + (16 * mu + g + 8) * BV, c, F1);
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        mma_16816(o[mu][nt], F0[0], F1[0], F0[1], F1[1], pb0[0][nt], pb1[0][nt]);
        mma_16816(o[mu][nt], F0[2], F1[2], F0[3], F1[3], pb0[1][nt], pb1[1][nt]);
      }
    }
    __syncwarp();
    if (lane == 0 && i + kStages < n_mine) {
      fence_proxy_async();
      issue(i + kStages);
    }
  }
  if (timed_out) {
    if (lane == 0) atomicOr(p.status, KVQ_FLAG_TIMEOUT);
    // let the copies this warp still has in flight land before leaving
    for (int i = consumed; i < min(n_mine, consumed + kStages); ++i)
      (void)mbar_wait_bounded(&sm.bar[warp][i % kStages], (uint32_t)((i / kStages) & 1));
  }

  // ---- CTA merge of the 4 warps' (m, l, O), then one partial per head
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      float l = l_run[nt][e];
      l += __shfl_xor_sync(0xffffffffu, l, 4);
      l += __shfl_xor_sync(0xffffffffu, l, 8);
      l += __shfl_xor_sync(0xffffffffu, l, 16);
      l_run[nt][e] = l;
    }
  __syncthreads();
  float* mg = reinterpret_cast<float*>(stage_base);  // [warp][16 heads][130]
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      float* dst = mg + ((size_t)warp * 16 + 8 * nt + 2 * c + e) * kPartStride;
      if (g == 0) {
        dst[0] = m_run[nt][e];
        dst[1] = l_run[nt][e];
      }
#pragma unroll
      for (int mu = 0; mu < 8; ++mu) {
        dst[2 + 16 * mu + g] = o[mu][nt][e];
        dst[2 + 16 * mu + g + 8] = o[mu][nt][2 + e];
      }
    }
  __syncthreads();
  for (int head = 0; head < G; ++head) {
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) M = fmaxf(M, mg[((size_t)w * 16 + head) * kPartStride]);
    float Lsum = 0.f, O = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < kWarps; ++w) {
        const float* src = mg + ((size_t)w * 16 + head) * kPartStride;
        const float sc = exp2f(src[0] - M);
        Lsum += sc * src[1];
        O += sc * src[2 + tid];
      }
    }
    float* dst = p.part + (((size_t)b * p.n_q + h * G + head) * p.n_splits + split) * kPartStride;
    dst[2 + tid] = O;
    if (tid == 0) {
      dst[0] = M;
      dst[1] = Lsum;
    }
  }
}

// Merge split partials and undo the value rotation:
// o = (1 / (128 l)) s . (H sum_s 2^(m_s - m) o_s).
// One CTA of 512 threads per (sequence, query head): split weights in shared
// memory, then 4 groups of 128 threads (one per coordinate) sum interleaved
// splits with independent loads in flight.
constexpr int kCombineThreads = 512;

__device__ __forceinline__ float block_reduce(float v, bool is_max, float* red) {
#pragma unroll
  for (int m = 16; m; m >>= 1) {
    const float o = __shfl_xor_sync(0xffffffffu, v, m);
    v = is_max ? fmaxf(v, o) : v + o;
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  v = red[0];
  for (int w = 1; w < kCombineThreads / 32; ++w) v = is_max ? fmaxf(v, red[w]) : v + red[w];
  return v;
}

__global__ void __launch_bounds__(kCombineThreads) combine_kernel(
    const float* __restrict__ part, int n_splits, int n_q, int G, const Plan* const* plans,
    float* out) {
  const int bh = blockIdx.x, b = bh / n_q, head = bh % n_q;
  const int tid = threadIdx.x;
  const float* pp = part + (size_t)bh * n_splits * kPartStride;
  __shared__ float s_w[1024];
  __shared__ float s_red[kCombineThreads / 32];
  __shared__ float s_o[4][kHeadDim];
  float m = -INFINITY;
  for (int s = tid; s < n_splits; s += kCombineThreads) m = fmaxf(m, pp[(size_t)s * kPartStride]);
  const float M = block_reduce(m, true, s_red);
  float lsum = 0.f;
  for (int s = tid; s < n_splits; s += kCombineThreads) {
    const float w = M == -INFINITY ? 0.f : exp2f(pp[(size_t)s * kPartStride] - M);
    s_w[s] = w;
    lsum += w * pp[(size_t)s * kPartStride + 1];
  }
  const float Lsum = block_reduce(lsum, false, s_red);
  __syncthreads();
  const int coord = tid & (kHeadDim - 1), grp = tid >> 7;
  float o = 0.f;
#pragma unroll 8
  for (int s = grp; s < n_splits; s += 4) o += s_w[s] * pp[(size_t)s * kPartStride + 2 + coord];
  s_o[grp][coord] = o;
  __syncthreads();
  if (tid < 32) {
    float y[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int i = tid + 32 * q;
      y[q] = (s_o[0][i] + s_o[1][i]) + (s_o[2][i] + s_o[3][i]);
    }
#pragma unroll
    for (int hh = 1; hh < 32; hh <<= 1) {
      const bool upper = (tid & hh) != 0;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float x = __shfl_xor_sync(0xffffffffu, y[q], hh);
        y[q] = upper ? x - y[q] : y[q] + x;
      }
    }
    const float a0 = y[0] + y[1], a1 = y[0] - y[1], a2 = y[2] + y[3], a3 = y[2] - y[3];
    y[0] = a0 + a2;
    y[2] = a0 - a2;
    y[1] = a1 + a3;
    y[3] = a1 - a3;
    const Plan* pl = plans[b] + head / G;
    const float inv = Lsum > 0.f ? 1.f / (128.f * Lsum) : 0.f;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int i = tid + 32 * q;
      const float sgn = ((pl->v_sign[i >> 5] >> (i & 31)) & 1u) ? -1.f : 1.f;
      out[(size_t)bh * kHeadDim + i] = sgn * y[q] * inv;
    }
  }
}

// ------------------------------------------------------------- launchers
int decode_splits(int64_t max_len) {
  const int64_t tiles = (max_len + kTile - 1) / kTile;
  const int64_t target = 6 * kWarps;  // tiles per CTA
  int64_t s = (tiles + target - 1) / target;
  return (int)std::max<int64_t>(1, std::min<int64_t>(s, 1024));
}

size_t decode_smem_bytes(int tile_bytes) {
  const size_t stages = (size_t)kWarps * kStages * tile_bytes;
  const size_t merge = (size_t)kWarps * 16 * kPartStride * sizeof(float);
  return sizeof(Smem) + std::max(stages, merge);
}

// The dynamic shared-memory cap is raised once per device and instantiation
// (to the largest tile size), so calls made during stream capture only launch.
template <int BV, int NT>
static cudaError_t launch_decode_t(const DecodeParams& p, int batch, cudaStream_t st) {
  static std::atomic<unsigned long long> ready{0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const unsigned long long bit = 1ull << (dev & 63);
  if (!(ready.load() & bit)) {
    e = cudaFuncSetAttribute(decode_kernel<BV, NT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)decode_smem_bytes(tile_bytes(8, BV)));
    if (e != cudaSuccess) return e;
    ready.fetch_or(bit);
  }
  const size_t smem = decode_smem_bytes(p.tile_bytes);
  decode_kernel<BV, NT><<<dim3(p.n_splits, p.n_kv, batch), kWarps * 32, smem, st>>>(p);
  return cudaGetLastError();
}

template <int NT>
static cudaError_t launch_decode_nt(const DecodeParams& p, int bits_v, int batch, cudaStream_t st) {
  switch (bits_v) {
    case 1: return launch_decode_t<1, NT>(p, batch, st);
    case 2: return launch_decode_t<2, NT>(p, batch, st);
    case 3: return launch_decode_t<3, NT>(p, batch, st);
    case 4: return launch_decode_t<4, NT>(p, batch, st);
    case 5: return launch_decode_t<5, NT>(p, batch, st);
    case 6: return launch_decode_t<6, NT>(p, batch, st);
    case 7: return launch_decode_t<7, NT>(p, batch, st);
    case 8: return launch_decode_t<8, NT>(p, batch, st);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_decode(const Plan* const* plans, const uint8_t* const* caches, const int32_t* len,
                          int batch, int64_t max_len, const void* q, int q_dtype, int n_q, int n_kv,
                          int bits_k, int bits_v, float* out, float* part, uint32_t* status,
                          cudaStream_t st) {
  DecodeParams p;
  p.plans = plans;
  p.caches = caches;
  p.len = len;
  p.q = q;
  p.q_dtype = q_dtype;
  p.n_q = n_q;
  p.n_kv = n_kv;
  p.G = n_q / n_kv;
  p.max_len = (int)max_len;
  p.n_splits = decode_splits(max_len);
  const int tiles = (int)((max_len + kTile - 1) / kTile);
  p.tiles_per_split = std::max(1, (tiles + p.n_splits - 1) / p.n_splits);
  p.tile_bytes = tile_bytes(bits_k, bits_v);
  p.part = part;
  p.status = status;
  cudaError_t e = p.G <= 8 ? launch_decode_nt<1>(p, bits_v, batch, st)
                           : launch_decode_nt<2>(p, bits_v, batch, st);
  if (e != cudaSuccess) return e;
  combine_kernel<<<batch * n_q, kCombineThreads, 0, st>>>(part, p.n_splits, n_q, p.G, plans, out);
  return cudaGetLastError();
}

}  // namespace kvq
