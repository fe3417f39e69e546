// Shared device definitions of libkvq: plan record, codebook constants,
// IEEE-exact helpers and the sm_100a inline-PTX primitives (bulk copies,
// mbarriers, mma.sync, movmatrix).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stddef.h>
#include <stdint.h>

#include "kvq.h"
#include "kvq_codebooks_gen.h"

namespace kvq {

constexpr int kHeadDim = 128;
constexpr int kBlocks = 64;
constexpr int kTile = 32;

// Plan record, byte layout documented in kvq.h.
struct Plan {
  uint32_t magic;
  int32_t bits_k, bits_v, n_ranks, layer, kv_head, words_k, words_v;
  float g[64];
  float a_hat[64];
  uint8_t width[64];
  uint8_t order[64];
  uint16_t seg_off[65];
  uint8_t n_half;
  uint8_t pad0;
  uint8_t hs_width[32];
  uint8_t hs_rank0[32];
  uint8_t hs_count[32];
  uint32_t v_sign[4];
  uint32_t pad1;
  double energy_sum;
  uint8_t n_class;         // runs of half steps of one width
  uint8_t pad2[7];
  uint8_t cls_w[8];
  uint8_t cls_hs0[8];
  uint8_t cls_nhs[8];
  uint8_t cls_last[8];     // blocks in the class's last half step
  uint16_t cls_seg0[8];    // first K word of the class in a tile record
  uint32_t k_sign[4];      // key rotation: bit P set <=> sign of plan position P is -1
  uint8_t k_rot;           // 1: keys rotated inside each width group
  uint8_t pad3[3];
  uint8_t tail[KVQ_PLAN_BYTES - 1004];
};
static_assert(sizeof(Plan) == KVQ_PLAN_BYTES, "plan size");
static_assert(offsetof(Plan, g) == 32 && offsetof(Plan, a_hat) == 288, "plan layout");
static_assert(offsetof(Plan, width) == 544 && offsetof(Plan, order) == 608, "plan layout");
static_assert(offsetof(Plan, seg_off) == 672 && offsetof(Plan, n_half) == 802, "plan layout");
static_assert(offsetof(Plan, hs_width) == 804 && offsetof(Plan, v_sign) == 900, "plan layout");
static_assert(offsetof(Plan, energy_sum) == 920, "plan layout");
static_assert(offsetof(Plan, n_class) == 928 && offsetof(Plan, cls_w) == 936, "plan layout");
static_assert(offsetof(Plan, cls_last) == 960 && offsetof(Plan, cls_seg0) == 968, "plan layout");
static_assert(offsetof(Plan, k_sign) == 984 && offsetof(Plan, k_rot) == 1000, "plan layout");

// Codebook offsets: width w centroids at 2^w - 2, thresholds at 2^w - w - 1.
__host__ __device__ constexpr int cb_c_off(int w) { return (1 << w) - 2; }
__host__ __device__ constexpr int cb_t_off(int w) { return (1 << w) - w - 1; }

__host__ __device__ inline int tile_bytes(int bits_k, int bits_v) { return 512 * (bits_k + bits_v) + 128; }

// Token position t of a tile -> bit slot (K segments, V segments) and back.
__host__ __device__ __forceinline__ int slot_k(int t) { return 4 * (t & 7) + (t >> 3); }
__host__ __device__ __forceinline__ int slot_v(int t) {
  return 8 * ((t & 7) >> 1) + 2 * (t >> 3) + (t & 1);
}
__host__ __device__ __forceinline__ int token_of_slot_k(int s) { return 8 * (s & 3) + (s >> 2); }
__host__ __device__ __forceinline__ int token_of_slot_v(int s) {
  return 8 * ((s & 7) >> 1) + 2 * (s >> 3) + (s & 1);
}

// Where the tiles of each sequence live (host and device side).
// Contiguous (table == nullptr): record of tile t, KV head h of sequence b at
// caches[b] + (t n_kv + h) tile_bytes. Paged: tile t is tile t mod P of page
// table[b][t / P] of the pool (P = 2^page_shift tiles per page, each page laid
// out like a contiguous cache of P tiles, page_bytes = P n_kv tile_bytes).
struct CacheMap {
  uint8_t* const* caches;  // contiguous: [batch] bases
  uint8_t* pool;           // paged: page g at pool + g page_bytes
  const int32_t* table;    // paged: [batch][max_pages] page ids
  int64_t n_pages;         // paged: ids outside [0, n_pages) are refused
  int64_t page_bytes;
  int max_pages;
  int page_shift;          // contiguous: 31 (one page)
};

inline CacheMap contiguous_map(const void* const* caches) {
  CacheMap m{};
  m.caches = reinterpret_cast<uint8_t* const*>(const_cast<void* const*>(caches));
  m.page_shift = 31;
  return m;
}

// Arguments of the quantize-append launch (host and device side).
struct QuantParams {
  const Plan* const* plans;  // [batch] -> [n_kv] plans
  const void* k;
  const void* v;
  int dtype;
  int batch, n_new, n_kv;
  CacheMap cm;
  const int32_t* len;
  int64_t cap;
  int tile_bytes;
  int tiles_max;  // work items per (sequence, KV head)
  uint32_t* status;
  int rope;           // keys are pre-RoPE: rotate each to its position first
  double theta[64];   // RoPE block frequencies base^(-2j/128)
  // recent-token window (wins != nullptr): per sequence, the oldest
  // max(0, wlen + n_new - R) tokens of window + new tokens are quantized
  // (window token at position t: fp32 rows in ring slot t mod R, keys then
  // values), and the lengths are left to the ring kernel
  const float* const* wins;
  const int32_t* wlen;
  int R;
};

// ------------------------------------------------------------------ device
#ifdef __CUDACC__

// Base of the page holding tile `tile` of sequence b (for a contiguous cache
// the sequence's base), or nullptr for a tile past the block table or a page
// id outside the pool. The record of (tile, h) is at base + tile_in_page
// offset: ((tile & page_mask(m)) n_kv + h) tile_bytes.
__device__ __forceinline__ const uint8_t* page_base(const CacheMap& m, int b, int tile) {
  if (!m.table) return m.caches[b];
  const int j = tile >> m.page_shift;
  if (j < 0 || j >= m.max_pages) return nullptr;
  const int g = m.table[(size_t)b * m.max_pages + j];
  if (g < 0 || (int64_t)g >= m.n_pages) return nullptr;
  return m.pool + (int64_t)g * m.page_bytes;
}
__device__ __forceinline__ int page_mask(const CacheMap& m) {
  return m.page_shift >= 31 ? 0x7FFFFFFF : (1 << m.page_shift) - 1;
}

__device__ __forceinline__ float load_as_float(const void* p, int dtype, size_t i) {
  if (dtype == KVQ_BF16) return __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(p)[i]);
  if (dtype == KVQ_FP16) return __half2float(reinterpret_cast<const __half*>(p)[i]);
  return reinterpret_cast<const float*>(p)[i];
}

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(unsigned long long* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count)
               : "memory");
}

__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_expect_tx(unsigned long long* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
               "r"(bytes)
               : "memory");
}

// 1-D bulk copy global -> shared, completion counted on `bar` (no multicast).
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes,
                                         unsigned long long* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(smem_addr(dst)),
      "l"(src), "r"(bytes), "r"(smem_addr(bar))
      : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(unsigned long long* bar, uint32_t phase) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_addr(bar)), "r"(phase)
      : "memory");
  return ok != 0;
}

// Bounded wait: gives up after `limit` clock cycles (default 2^31, about a
// second) and returns false.
constexpr long long kWaitCycles = 1ll << 31;
__device__ __forceinline__ bool mbar_wait_bounded(unsigned long long* bar, uint32_t phase,
                                                  long long limit = kWaitCycles) {
  if (mbar_try_wait(bar, phase)) return true;
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, phase)) {
    if (clock64() - t0 > limit) return false;
  }
  return true;
}

// D = A(16x16 f16, row) * B(16x8 f16, col) + D, fp32 accumulate.
__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                          uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Transpose of an 8x8 b16 matrix held one row per 4 lanes (2 elements each).
__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_half2(float lo, float hi) {
  __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ uint32_t funnel_r(uint32_t lo, uint32_t hi, uint32_t sh) {
  return __funnelshift_r(lo, hi, sh);
}

// Structural check of a plan (shared memory) by one whole warp; every lane
// gets the answer. True iff the plan order, the K segment offsets, the half
// steps and the width classes are exactly what the host's schedule builder
// makes of the widths: order = the blocks of nonzero width, width
// descending then block index ascending; seg_off[r + 1] = seg_off[r] + 2 W;
// 128 bits_k K words in all; half steps = runs of one width cut into groups
// of at most 4 ranks; classes = maximal runs of half steps of one width.
// Every index the kernels derive from these fields then stays inside the
// plan's arrays and the tile record, whatever the rest of the plan holds.
constexpr int kMaxHalfSteps = 24;  // <= 64 / 4 + one partial group per width
__device__ __forceinline__ bool plan_sched_ok(const Plan& pl, int lane) {
  // scalar fields as lane 0 read them, so that the early exit is uniform
  const int nr = __shfl_sync(0xffffffffu, pl.n_ranks, 0);
  const int nh = __shfl_sync(0xffffffffu, (int)pl.n_half, 0);
  const int nc = __shfl_sync(0xffffffffu, (int)pl.n_class, 0);
  const int bk = __shfl_sync(0xffffffffu, pl.bits_k, 0);
  if (nr < 1 || nr > 64 || bk < 1 || bk > 8 || nh < 1 || nh > kMaxHalfSteps || nc < 1 || nc > 8)
    return false;
  auto width_of_rank = [&](int r) { return (int)pl.width[pl.order[r] & 63]; };
  bool ok = true;
  uint32_t seen[2] = {0u, 0u};
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const int r = lane + 32 * i;
    if (r < nr) {
      const int o = pl.order[r], w = width_of_rank(r);
      ok &= o < 64 && w >= 1 && w <= 8;
      ok &= pl.seg_off[r + 1] == pl.seg_off[r] + 2 * w;
      if (r + 1 < nr) {
        const int o2 = pl.order[r + 1], w2 = width_of_rank(r + 1);
        ok &= w > w2 || (w == w2 && o < o2);
      }
      seen[(o >> 5) & 1] |= 1u << (o & 31);
    }
  }
  ok &= pl.seg_off[0] == 0 && pl.seg_off[nr] == 128 * bk;
  // the order holds each block of nonzero width once (with the strict
  // ordering above, no block twice)
  ok &= __reduce_or_sync(0xffffffffu, seen[0]) == __ballot_sync(0xffffffffu, pl.width[lane] != 0);
  ok &= __reduce_or_sync(0xffffffffu, seen[1]) ==
        __ballot_sync(0xffffffffu, pl.width[lane + 32] != 0);
  if (lane < nh) {
    const int r0 = pl.hs_rank0[lane], n = pl.hs_count[lane];
    ok &= n >= 1 && n <= 4 && r0 + n <= nr && (lane > 0 || r0 == 0);
    if (n >= 1 && r0 + n <= nr) {
      const int w = width_of_rank(r0);
      ok &= pl.hs_width[lane] == w && width_of_rank(r0 + n - 1) == w;
      if (n < 4 && r0 + n < nr) ok &= width_of_rank(r0 + n) != w;  // a short group ends its run
      ok &= lane + 1 < nh ? pl.hs_rank0[lane + 1] == r0 + n : r0 + n == nr;
    }
  }
  if (lane < nc) {
    const int h0 = pl.cls_hs0[lane], m = pl.cls_nhs[lane];
    ok &= m >= 1 && h0 + m <= nh && (lane > 0 || h0 == 0);
    if (m >= 1 && h0 + m <= nh) {
      const int w = pl.hs_width[h0], r0 = pl.hs_rank0[h0];
      ok &= pl.cls_w[lane] == w && pl.hs_width[h0 + m - 1] == w &&
            pl.cls_last[lane] == pl.hs_count[h0 + m - 1] && r0 < nr &&
            pl.cls_seg0[lane] == pl.seg_off[r0 & 63];
      ok &= lane + 1 < nc ? pl.cls_hs0[lane + 1] == h0 + m && pl.hs_width[h0 + m] != w
                          : h0 + m == nh;
    }
  }
  return __all_sync(0xffffffffu, ok);
}

#endif  // __CUDACC__

}  // namespace kvq
