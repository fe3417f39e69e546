// bf16 comparator: split-K decode attention over an unquantized bf16 KV
// cache, built like the packed-cache decode (one-wave grid, per-warp bulk-copy
// ring, mma.sync, base-2 online softmax, in-kernel two-level split merge), so
// that the packed path can be measured against the plain one on the same
// shapes and hardware. Not part of the method: "RoPE-Aware Bit Allocation for
// KV-Cache Quantization", abstract, compares its packed-cache decode with fp16
// FlashAttention2; this kernel stands in for that dense baseline.
//
// Cache layout: K and V each [batch][n_kv][cap][128] bf16 (the tokens of one
// head contiguous). Queries [batch][n_q][128] bf16; output fp32.
// Per warp and 32-token tile: S[32 tokens x 8 heads] = K Q^T by m16n8k16 bf16
// MMAs (A fragments by ldmatrix from rows padded to 272 B, conflict free; B =
// q as loaded), P = 2^(S - m) in bf16 moved to the B layout with movmatrix,
// O^T[128 x 8] += V^T P^T with A fragments by ldmatrix.trans.
#include <algorithm>
#include <atomic>

#include "splitk.cuh"

namespace kvq {

constexpr int kDWarps = 6;
constexpr int kDThreads = kDWarps * 32;
constexpr int kDStages = 2;
constexpr int kDRow = 272;                 // shared-memory row: 256 B of bf16 + 16 B pad
constexpr int kDTileBytes = kTile * kDRow;  // one tensor's tile
constexpr int kDStageBytes = 2 * kDTileBytes;

struct DenseParams {
  const __nv_bfloat16* k;  // [batch][n_kv][cap][128]
  const __nv_bfloat16* v;
  const int32_t* len;
  int64_t cap;
  int max_len;
  const __nv_bfloat16* q;  // [batch][n_q][128]
  int n_q, n_kv, G;
  int n_splits, tiles_per_split, n_groups;
  unsigned int* cnt_end;  // counters of pair k at cnt_end - (k + 1) * kCntStride
  float* part;            // [batch][n_kv][n_splits][G][132]
  float* gpart;           // [batch][n_kv][n_groups][G][132]
  float* out;             // [batch][n_q][128]
  uint32_t* status;
};

struct alignas(128) DSmem {
  unsigned long long bar[kDWarps][kDStages];
  int is_last;
};

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                               uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ uint32_t pack_bf162(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

template <int NT>
__global__ void __launch_bounds__(kDThreads, 1) dense_decode_kernel(const DenseParams p) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  DSmem& sm = *reinterpret_cast<DSmem*>(smem_raw);
  uint8_t* const stage_base = smem_raw + sizeof(DSmem);
  const int split = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, c = lane & 3;
  const int G = p.G;
  const size_t bh = (size_t)b * p.n_kv + h;
  unsigned int* const cnt = p.cnt_end - (bh + 1) * kCntStride;

  if (tid == 0) {
    for (int i = 0; i < kDWarps * kDStages; ++i)
      mbar_init(&sm.bar[i / kDStages][i % kDStages], 1);
    fence_proxy_async();
  }
  grid_dep_wait();
  __syncthreads();
  grid_dep_launch();
  int L = p.len[b];
  if (L > p.max_len || (int64_t)L > p.cap) {
    if (tid == 0 && split == 0 && h == 0) atomicOr(p.status, KVQ_FLAG_CAPACITY);
    L = (int)min((long long)p.max_len, (long long)p.cap);
  }
  L = max(L, 0);
  const int n_tiles = (L + kTile - 1) / kTile;
  const int tb = split * p.tiles_per_split;
  const int te = min(n_tiles, tb + p.tiles_per_split);
  const int n_mine = tb < te ? max(0, (te - tb - warp + kDWarps - 1) / kDWarps) : 0;
  auto tile_of = [&](int i) { return te - 1 - warp - i * kDWarps; };
  const __nv_bfloat16* kh = p.k + bh * p.cap * kHeadDim;
  const __nv_bfloat16* vh = p.v + bh * p.cap * kHeadDim;
  uint8_t* const my_stages = stage_base + (size_t)warp * kDStages * kDStageBytes;
  // rows of tile t that exist in the cache buffer (rows past the length are
  // masked; rows past the capacity are not read)
  auto rows_of = [&](int t) {
    return (int)min((long long)kTile, (long long)(p.cap - (int64_t)t * kTile));
  };
  auto issue = [&](int i) {  // whole warp
    const int t = tile_of(i), s = i % kDStages, nr = rows_of(t);
    unsigned long long* bar = &sm.bar[warp][s];
    if (lane == 0) mbar_expect_tx(bar, (uint32_t)(2 * nr * kHeadDim * 2));
    __syncwarp();
    if (lane < nr) {
      uint8_t* dst = my_stages + s * kDStageBytes + lane * kDRow;
      const size_t row = ((size_t)t * kTile + lane) * kHeadDim;
      bulk_g2s(dst, kh + row, kHeadDim * 2, bar);
      bulk_g2s(dst + kDTileBytes, vh + row, kHeadDim * 2, bar);
    }
  };
  for (int i = 0; i < min(kDStages, n_mine); ++i) issue(i);

  // query B fragments: b0 = q[head][16 ks + 2c, +1], b1 = q[head][16 ks + 2c + 8, +9]
  uint32_t qb[NT][8][2];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const int head = 8 * nt + g;
    const uint32_t* qrow = reinterpret_cast<const uint32_t*>(
        p.q + ((size_t)b * p.n_q + (size_t)h * G + min(head, G - 1)) * kHeadDim);
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      qb[nt][ks][0] = head < G ? qrow[(16 * ks + 2 * c) >> 1] : 0u;
      qb[nt][ks][1] = head < G ? qrow[(16 * ks + 2 * c + 8) >> 1] : 0u;
    }
  }

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
  constexpr float kC = 0.12751743074f;  // log2(e) / sqrt(128)
  // ldmatrix row addresses (lane part): K rows (tokens) for A = K, V rows
  // (tokens) for A = V^T with .trans
  const int k_row = (lane & 7) + 8 * ((lane >> 3) & 1), k_col = 8 * (lane >> 4);
  const int v_row = (lane & 7) + 8 * (lane >> 4), v_col = 8 * ((lane >> 3) & 1);

  int consumed = 0;
  bool timed_out = false;
  for (int i = 0; i < n_mine; ++i) {
    const int s = i % kDStages;
    const bool ok = mbar_wait_bounded(&sm.bar[warp][s], (uint32_t)((i / kDStages) & 1));
    if (!__all_sync(0xffffffffu, ok)) {
      timed_out = true;
      break;
    }
    consumed = i + 1;
    const int tile = tile_of(i);
    const int nvalid = min(kTile, L - tile * kTile);
    uint8_t* ks_ = my_stages + s * kDStageBytes;
    uint8_t* vs_ = ks_ + kDTileBytes;
    if (nvalid < kTile) {  // V rows past the length get weight 0: make them finite zeros
      for (int e = lane; e < (kTile - nvalid) * 16; e += 32)
        reinterpret_cast<uint4*>(vs_ + (nvalid + e / 16) * kDRow)[e % 16] =
            make_uint4(0u, 0u, 0u, 0u);
      __syncwarp();
    }
    const uint32_t ka = smem_addr(ks_), va = smem_addr(vs_);

    float sacc[2][NT][4];
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int r = 0; r < 4; ++r) sacc[mt][nt][r] = 0.f;
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        uint32_t A[4];
        ldsm_x4(ka + (16 * mt + k_row) * kDRow + (16 * kk + k_col) * 2, A);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
          mma_bf16_16816(sacc[mt][nt], A, qb[nt][kk][0], qb[nt][kk][1]);
      }

    // online softmax (base 2); this thread's tokens are g + 8 r, r = 0..3
    bool val[4];
#pragma unroll
    for (int r = 0; r < 4; ++r) val[r] = g + 8 * r < nvalid;
    uint32_t pb0[2][NT], pb1[2][NT];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      float pe[2][4];
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        float sv[4];
#pragma unroll
        for (int r = 0; r < 4; ++r)
          sv[r] = val[r] ? sacc[r >> 1][nt][2 * (r & 1) + e] * kC : -INFINITY;
        float mx = fmaxf(fmaxf(sv[0], sv[1]), fmaxf(sv[2], sv[3]));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
        const float m_new = fmaxf(m_run[nt][e], mx);
        float alpha = 1.f, lsum = 0.f;
        if (m_new != -INFINITY) {
          alpha = ex2(m_run[nt][e] - m_new);
#pragma unroll
          for (int r = 0; r < 4; ++r) {
            pe[e][r] = ex2(sv[r] - m_new);
            lsum += pe[e][r];
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
        pb0[mt][nt] = movmatrix_trans(pack_bf162(pe[0][2 * mt], pe[1][2 * mt]));
        pb1[mt][nt] = movmatrix_trans(pack_bf162(pe[0][2 * mt + 1], pe[1][2 * mt + 1]));
      }
    }

    // values: O^T[128 x 8 NT] += V^T[128 x 32 tokens] P^T
#pragma unroll
    for (int mu = 0; mu < 8; ++mu)
#pragma unroll
      for (int kt = 0; kt < 2; ++kt) {
        uint32_t A[4];
        ldsm_x4_t(va + (16 * kt + v_row) * kDRow + (16 * mu + v_col) * 2, A);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) mma_bf16_16816(o[mu][nt], A, pb0[kt][nt], pb1[kt][nt]);
      }
    __syncwarp();
    if (i + kDStages < n_mine) {
      fence_proxy_async();  // the zero fill above was a generic-proxy write
      issue(i + kDStages);
    }
  }
  if (timed_out) {
    if (lane == 0) atomicOr(p.status, KVQ_FLAG_TIMEOUT);
    for (int i = consumed; i < min(n_mine, consumed + kDStages); ++i)
      (void)mbar_wait_bounded(&sm.bar[warp][i % kDStages], (uint32_t)((i / kDStages) & 1));
  }

  // ---- warps -> records -> two-level split merge (as in the packed decode)
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
  float* mg = reinterpret_cast<float*>(stage_base);  // [warp][8 NT heads][132]
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      float* dst = mg + ((size_t)warp * 8 * NT + 8 * nt + 2 * c + e) * kPartStride;
      if (g == 0) {
        dst[0] = m_run[nt][e];
        dst[1] = l_run[nt][e];
      }
#pragma unroll
      for (int mu = 0; mu < 8; ++mu) {
        dst[kRecO + 16 * mu + g] = o[mu][nt][e];
        dst[kRecO + 16 * mu + g + 8] = o[mu][nt][2 + e];
      }
    }
  __syncthreads();
  float* const my_part = p.part + (bh * p.n_splits + split) * G * kPartStride;
  merge_records<kDThreads, 8>(mg, kDWarps, (size_t)8 * NT * kPartStride, G, my_part);

  const int grp = split / kGroup;
  const int g_lo = grp * kGroup, g_n = min(kGroup, p.n_splits - g_lo);
  __syncthreads();
  if (tid == 0) sm.is_last = arrive_last(&cnt[1 + grp], (unsigned int)g_n);
  __syncthreads();
  if (!sm.is_last) return;
  float* my_gpart = p.gpart + (bh * p.n_groups + grp) * G * kPartStride;
  merge_records<kDThreads>(p.part + (bh * p.n_splits + g_lo) * G * kPartStride, g_n,
                           (size_t)G * kPartStride, G, my_gpart);
  __syncthreads();
  if (tid == 0) sm.is_last = arrive_last(&cnt[0], (unsigned int)p.n_groups);
  __syncthreads();
  if (!sm.is_last) return;
  float* fin = reinterpret_cast<float*>(stage_base);  // [16][132]
  merge_records<kDThreads>(p.gpart + bh * p.n_groups * G * kPartStride, p.n_groups,
                           (size_t)G * kPartStride, G, fin);
  __syncthreads();
  for (int e = tid; e < G * kHeadDim; e += kDThreads) {
    const int head = e / kHeadDim, x = e % kHeadDim;
    const float* r = fin + (size_t)head * kPartStride;
    const float inv = r[1] > 0.f ? 1.f / r[1] : 0.f;
    p.out[((size_t)b * p.n_q + (size_t)h * G + head) * kHeadDim + x] = r[kRecO + x] * inv;
  }
}

// ------------------------------------------------------------- launchers
static size_t dense_smem_bytes(int nt) {
  const size_t stages = (size_t)kDWarps * kDStages * kDStageBytes;
  const size_t merge = (size_t)kDWarps * 8 * nt * kPartStride * sizeof(float);
  return sizeof(DSmem) + std::max(stages, merge);
}

template <int NT>
static int dense_ctas_per_sm(int dev, cudaError_t* err) {
  static std::atomic<int> cache[64];
  std::atomic<int>& slot = cache[dev & 63];
  int v = slot.load();
  if (v > 0) return v;
  cudaError_t e = cudaFuncSetAttribute(dense_decode_kernel<NT>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)dense_smem_bytes(NT));
  if (e == cudaSuccess)
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&v, dense_decode_kernel<NT>, kDThreads,
                                                      dense_smem_bytes(NT));
  if (e != cudaSuccess || v < 1) {
    *err = e != cudaSuccess ? e : cudaErrorInvalidConfiguration;
    return 0;
  }
  slot.store(v);
  return v;
}

struct DenseSplit {
  int n_splits, tiles_per_split, n_groups;
  int64_t slots;  // CTA slots the split count was sized for
};

static DenseSplit dense_split_plan(int batch, int n_kv, int G, int64_t max_len, bool allow_fallback,
                                   cudaError_t* err) {
  DenseSplit sp{1, 1, 1, 1024};
  int64_t slots = 1024;
  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  int per_sm = 0;
  if (e == cudaSuccess)
    per_sm = G <= 8 ? dense_ctas_per_sm<1>(dev, &e) : dense_ctas_per_sm<2>(dev, &e);
  if (e == cudaSuccess) {
    slots = (int64_t)sms * per_sm;
  } else if (!allow_fallback) {
    *err = e;
    return sp;
  } else {
    (void)cudaGetLastError();
  }
  *err = cudaSuccess;
  sp.slots = slots;
  const int64_t tiles = std::max<int64_t>(1, (max_len + kTile - 1) / kTile);
  int64_t s = std::max<int64_t>(1, slots / ((int64_t)batch * n_kv));
  s = std::min<int64_t>(s, std::max<int64_t>(1, (tiles + kDWarps - 1) / kDWarps));
  s = std::min<int64_t>(s, kMaxSplits);
  sp.tiles_per_split = (int)((tiles + s - 1) / s);
  sp.n_splits = (int)((tiles + sp.tiles_per_split - 1) / sp.tiles_per_split);
  sp.n_groups = (sp.n_splits + kGroup - 1) / kGroup;
  return sp;
}

static size_t dense_align256(size_t x) { return (x + 255) / 256 * 256; }

// Workspace: split records | group records | ... | counters of pair k at a
// fixed distance from the end (k + 1) * kCntStride words. The record regions
// are bounded by one record per CTA slot (or per pair, if there are more
// pairs) and 16 query heads, independently of max_len and G, so the records
// of any call with batch x n_kv <= that of the sizing call end before the
// counters of any such call (the counters are the only words that must be
// zero when a call starts; every completed call leaves them at zero).
static size_t dense_workspace_layout(size_t pairs, int64_t slots, size_t* gpart_off) {
  const size_t recs = (size_t)std::max<int64_t>(slots, (int64_t)pairs);
  const size_t rec_bytes = 16 * kPartStride * sizeof(float);
  const size_t part = dense_align256(recs * rec_bytes);
  const size_t gpart = dense_align256((recs / kGroup + pairs + 1) * rec_bytes);
  const size_t counters = dense_align256(pairs * kCntStride * sizeof(unsigned int));
  if (gpart_off) *gpart_off = part;
  return part + gpart + counters + 16;
}

size_t dense_workspace_bytes_for(int batch, int n_kv, int n_q, int64_t max_len) {
  cudaError_t err = cudaSuccess;
  const int G = n_q / n_kv;
  const DenseSplit sp = dense_split_plan(batch, n_kv, G, max_len, true, &err);
  return dense_workspace_layout((size_t)batch * n_kv, sp.slots, nullptr);
}

template <int NT>
static cudaError_t launch_dense_t(const DenseParams& p, int batch, cudaStream_t st) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.n_splits, p.n_kv, batch);
  cfg.blockDim = dim3(kDThreads);
  cfg.dynamicSmemBytes = dense_smem_bytes(NT);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, dense_decode_kernel<NT>, p);
}

cudaError_t launch_dense_decode(const void* k, const void* v, const int32_t* len, int batch,
                                int n_kv, int64_t cap, int64_t max_len, const void* q, int n_q,
                                float* out, void* ws, size_t ws_bytes, uint32_t* status,
                                cudaStream_t st) {
  cudaError_t err = cudaSuccess;
  const int G = n_q / n_kv;
  const DenseSplit sp = dense_split_plan(batch, n_kv, G, max_len, false, &err);
  if (err != cudaSuccess) return err;
  size_t gpart_off = 0;
  if (dense_workspace_layout((size_t)batch * n_kv, sp.slots, &gpart_off) > ws_bytes)
    return cudaErrorInvalidValue;
  DenseParams p;
  p.k = reinterpret_cast<const __nv_bfloat16*>(k);
  p.v = reinterpret_cast<const __nv_bfloat16*>(v);
  p.len = len;
  p.cap = cap;
  p.max_len = (int)max_len;
  p.q = reinterpret_cast<const __nv_bfloat16*>(q);
  p.n_q = n_q;
  p.n_kv = n_kv;
  p.G = G;
  p.n_splits = sp.n_splits;
  p.tiles_per_split = sp.tiles_per_split;
  p.n_groups = sp.n_groups;
  p.part = reinterpret_cast<float*>(ws);
  p.gpart = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(ws) + gpart_off);
  p.cnt_end = reinterpret_cast<unsigned int*>(
      (reinterpret_cast<uintptr_t>(ws) + ws_bytes) & ~static_cast<uintptr_t>(15));
  p.out = out;
  p.status = status;
  return G <= 8 ? launch_dense_t<1>(p, batch, st) : launch_dense_t<2>(p, batch, st);
}

}  // namespace kvq
