// Packed-cache decode attention (optionally fused with the append of the
// step's new tokens): split-K over the context, the splits summed inside the
// same kernel (exponent buckets in L2, read by the last split).
//
// "RoPE-Aware Bit Allocation for KV-Cache Quantization", abstract: the
// packed-cache serving path runs decode attention directly on the packed
// K/V cache (the pages report it faster than fp16 FlashAttention2 at 128K on
// H800). This is an sm_100a design of its own:
//
// * Work: CTA = (split, KV head, sequence), 8 warps, grid sized to one wave.
//   Each warp owns every 8th 32-token tile of the CTA's range and streams its
//   tiles into a private 2-stage shared-memory ring with 1-D bulk copies
//   (cp.async.bulk + mbarrier, no multicast). The codebook lookup image
//   (pair tables, replicated per lane for widths <= 3 so lookups are free of
//   bank conflicts) and the plan also arrive by bulk copy. Launched with
//   programmatic dependent launch: everything up to griddepcontrol.wait does
//   not depend on the previous kernel.
// * Append (fused calls): the CTA that owns the tile of a new token
//   quantizes it and patches it into the streamed copy of the tile (the
//   first stage of one of its warps) and into the cache; the last CTA of the
//   sequence to read its length writes the new length.
// * Keys: logits S[32 tokens x 8 heads] by mma.sync m16n8k16, one MMA per
//   m-tile and "half step" of the plan (<= 4 RoPE blocks of one width W),
//   the A fragment repeated over k so that one MMA adds A q'_hi + A q'_lo
//   (split below). Each 32-bit A register is one block (codes of
//   coordinates j and j + 64) of one token,
//   looked up as an fp16 pair; the packed layout puts the 4 tokens a lane
//   needs (g, g + 8, g + 16, g + 24) in 8W contiguous bits. Half steps of one
//   width form a class compiled for its W. B = the query group times a_hat_j,
//   log2(e), 1/sqrt(128), scaled by 2^sigma per head and split hi + lo fp16.
// * Softmax: base-2 online softmax per head on the fp32 accumulators, scaled
//   by the fp16 key norms; positions past the sequence length masked. The
//   reference of a head moves only when a score passes it (then to the
//   tile's maximum plus a small headroom), so most tiles skip the maximum
//   reduction and the rescaling of o.
// * Values: P' = p * n^V (fp16) moves from the accumulator layout to the B
//   operand with movmatrix; O^T(128 x G) += Vhat^T(128 x 16 tokens) P'^T with
//   A registers holding one rotated coordinate of two tokens.
// * Merge: the 8 warps merge in shared memory into the split's record; per
//   query head the split adds 2^(m - 32 k) (l, o), k = floor(m / 32), to
//   exponent bucket k by L2 atomics (float, vector); the last of the pair's
//   splits to arrive (one acquire-release counter) sums the few buckets in
//   use with weights 2^(32 (k - k_max)), clears them, undoes the value
//   rotation (inverse Walsh-Hadamard, signs) and writes o / l. A split max
//   outside [-256, 256) makes the last split merge all records instead. The
//   sum order of the atomics varies, so outputs agree run to run to fp32
//   rounding, not bit for bit; a process-wide deterministic mode makes the
//   last split merge all records in split order instead.
#include <algorithm>
#include <cstddef>
#include <atomic>

#include "quant_dev.cuh"
#include "splitk.cuh"

namespace kvq {

// Lookup image (generated with the codebooks): byte offsets of its tables.
__device__ __align__(16) const uint32_t g_lut_image[KVQ_LUT_BYTES / 4] = KVQ_LUT_IMAGE;
static_assert(KVQ_LUT_BYTES >= 512 * 16 + 128, "placeholder source of a refused page's tile");
constexpr int kThrPad = (KVQ_CB_N_THR + 3) & ~3;  // thresholds, padded to 16 bytes
__device__ __align__(16) const float g_thr[kThrPad] = KVQ_CB_THR;
__host__ __device__ constexpr uint32_t lut_rep(int w) {  // widths 1..3, lane-replicated
  return w == 1 ? 0x4000u : w == 2 ? 0x2000u : 0x0000u;
}
constexpr uint32_t kLutPair4 = 0x2800u, kLutPair5 = 0x2C00u, kLutSingle = 0x3C00u;

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kStages = 2;
constexpr int kMaxHalf = kMaxHalfSteps;  // half steps of <= 4 blocks
constexpr int kBuckets = 16;  // split maxima m in [32 (k - 8), 32 (k - 7)), k = 0..15
// Per (sequence, KV head) "pair block" of the workspace, at a fixed distance
// from its end: 32 counter words (0: arrivals, 1: range flag, 2..17: bucket
// masks of the query heads, 31: sequence counter of KV head 0), then the
// exponent buckets of up to 16 query heads. Every completed call leaves the
// words and buckets it used at zero, and a pair block never overlaps the
// split records of any call whose batch x n_kv fits the workspace.
constexpr int kPairCntWords = 32;
constexpr size_t kPairBlockBytes =
    kPairCntWords * 4 + (size_t)16 * kBuckets * kPartStride * sizeof(float);
static_assert(kPairBlockBytes % 128 == 0, "pair blocks keep the buckets 16-byte aligned");
constexpr int kFallbackSlots = 1024;                  // CTA slots when no device answers
constexpr int kMaxNew = 64;                           // tokens appended by a fused call
constexpr float kHeadroom = 2.f;  // base-2 margin of a moved softmax reference
constexpr int kScratch = 16640;  // q' staging; append: kz [32][129] fp32 + 64 fp16 norms

struct DecodeParams {
  const Plan* const* plans;
  CacheMap cm;
  int32_t* len;
  const void* q;
  int q_dtype;
  int n_q, n_kv, G;
  int max_len;
  int n_splits, tiles_per_split;
  int tile_bytes;
  // fused append (n_new > 0)
  const void* k_new;
  const void* v_new;
  int kv_dtype, n_new;
  int64_t cap;
  int early;  // read lengths and stream tiles before waiting for the previous kernel
  int rope;   // appended keys are pre-RoPE: rotate each to its position first
  long long stall_cycles;  // test hook (> 0): each warp first waits that long in vain
  int deterministic;       // merge the split records in split order (no L2 atomics)
  // recent-token window step (window kernels only): per sequence a ring of R
  // fp32 rows (keys, then values; token t in slot t mod R) and its length
  float* const* wins;
  int32_t* wlen;
  int R;
  double theta[64];
  uint8_t* pb_end;        // pair block of pair k at pb_end - (k + 1) * kPairBlockBytes
  float* part;            // [batch][n_kv][n_splits][G][132] = m, l, -, -, o[128]
  float* out;             // [batch][n_q][128]
  float* rec_out;         // partial decode: merged records [batch][n_q][132], no out
  uint32_t* status;
};

struct alignas(128) Smem {
  Plan plan;
  uint8_t lut[KVQ_LUT_BYTES];
  uint2 qfrag[2][kMaxHalf][32];  // per (n-tile, half step, lane): hi, lo
  float inv_scale[16];           // 2^-sigma of each head's q' scaling
  unsigned long long bar[kWarps][kStages];
  unsigned long long setup_bar;
  unsigned long long stall_bar;  // nothing arrives on it (test hook of a wait that runs out)
  uint32_t cls_lane[8][32];      // per (class, lane): first K word << 8 | bit shift
  alignas(16) float thr[kThrPad];  // decision thresholds (fused append only)
  double theta[64];                // RoPE block frequencies (fused append of pre-RoPE keys)
  int8_t qj[kMaxHalf][4];        // per half step: block of MMA column c, or -1
  int len0, is_last;
  int w0;  // window step: the window's length before the step
  uint32_t flags;
  RotTables rot;                   // key rotation tables (plans with k_rot)
};

// Bulk-copy destinations start on 16-byte boundaries.
static_assert(offsetof(Smem, plan) % 16 == 0 && offsetof(Smem, lut) % 16 == 0 &&
                  offsetof(Smem, thr) % 16 == 0 && sizeof(Smem) % 128 == 0,
              "shared-memory layout");

// Loads from shared memory through pointers into the dynamic shared window,
// so constant table offsets fold into the load instruction.
__device__ __forceinline__ uint32_t ld32s(const uint8_t* p) {
  return *reinterpret_cast<const uint32_t*>(p);
}
__device__ __forceinline__ uint32_t ld16s(const uint8_t* p) {
  return *reinterpret_cast<const uint16_t*>(p);
}

// Vector float reduction in L2 (no return value).
__device__ __forceinline__ void red_add_v4(float* addr, float a, float b, float c, float d) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(addr), "f"(a), "f"(b),
               "f"(c), "f"(d)
               : "memory");
}

// Four fp16 pairs from the 4 pair fields (2W bits each) that start at bit
// `sh` of the word at `wp` (shared memory). lut: the lookup image; lane4 = 4 *
// lane. W is a compile-time width (the value width).
template <int W>
__device__ __forceinline__ void fields4(const uint8_t* lut, const uint8_t* wp, uint32_t sh,
                                        uint32_t lane4, uint32_t (&out)[4]) {
  if constexpr (W <= 3) {
    // replicated pair table: entry e of lane l at byte (e * 32 + l) * 4
    constexpr uint32_t m7 = ((1u << (2 * W)) - 1u) << 7;
    const uint32_t v7 = funnel_r(ld32s(wp), ld32s(wp + 4), sh) << 7;
    const uint32_t lb = lane4 | lut_rep(W);
#pragma unroll
    for (int i = 0; i < 4; ++i) out[i] = ld32s(lut + (((v7 >> (2 * W * i)) & m7) | lb));
  } else if constexpr (W == 4) {
    const uint32_t v = funnel_r(ld32s(wp), ld32s(wp + 4), sh);
    out[0] = ld32s(lut + kLutPair4 + ((v << 2) & 0x3FCu));
#pragma unroll
    for (int i = 1; i < 4; ++i) out[i] = ld32s(lut + kLutPair4 + ((v >> (8 * i - 2)) & 0x3FCu));
  } else if constexpr (W == 5) {
    const uint32_t w0 = ld32s(wp), w1 = ld32s(wp + 4), w2 = ld32s(wp + 8);
    const uint32_t lo = funnel_r(w0, w1, sh), hi = funnel_r(w1, w2, sh);
    out[0] = ld32s(lut + kLutPair5 + ((lo << 2) & 0xFFCu));
    out[1] = ld32s(lut + kLutPair5 + ((lo >> 8) & 0xFFCu));
    out[2] = ld32s(lut + kLutPair5 + ((lo >> 18) & 0xFFCu));
    out[3] = ld32s(lut + kLutPair5 + (funnel_r(lo, hi, 28) & 0xFFCu));
  } else {
    // widths 6..8: two single-code lookups per pair (fp16 table, 2 bytes each)
    const uint32_t w0 = ld32s(wp), w1 = ld32s(wp + 4), w2 = ld32s(wp + 8);
    const uint32_t lo = funnel_r(w0, w1, sh), hi = funnel_r(w1, w2, sh);
    const unsigned long long v = ((unsigned long long)hi << 32) | lo;
    constexpr uint32_t mw = ((1u << W) - 1u) << 1;
    const uint8_t* tab = lut + kLutSingle + 2u * (uint32_t)cb_c_off(W);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t a = (uint32_t)(v >> (2 * W * i)) << 1;
      out[i] = ld16s(tab + (a & mw)) | (ld16s(tab + ((a >> W) & mw)) << 16);
    }
  }
}

// Logits of one width class: its nhs half steps of <= 4 blocks of width W
// (runtime, warp-uniform: one code path per lookup kind keeps the kernel
// small). Lane (g, c) takes block c of every half step, tokens g, g + 8
// (m-tile 0) and g + 16, g + 24 (m-tile 1). In a class's last half step the
// lanes past its last block read other valid words of the tile: their q' is
// exactly 0, so those finite fp16 values add nothing.
template <int NT>
__device__ __forceinline__ void key_mma(float (&s)[2][NT][4], const uint32_t (&A)[4],
                                        const uint2* qp) {
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    // k16 with the A fragment repeated: A q'_hi + A q'_lo in one MMA
    const uint2 b = qp[nt * kMaxHalf * 32];
    mma_16816(s[0][nt], A[0], A[1], A[0], A[1], b.x, b.y);
    mma_16816(s[1][nt], A[2], A[3], A[2], A[3], b.x, b.y);
  }
}

template <int NT>
__device__ __forceinline__ void key_class(const Smem& sm, const uint8_t* kw, int ci, int lane,
                                          uint32_t lane4, float (&s)[2][NT][4]) {
  const int W = sm.plan.cls_w[ci];
  const int nhs = sm.plan.cls_nhs[ci];
  const uint32_t pk = sm.cls_lane[ci][lane];
  const uint8_t* wp = kw + 4u * (pk >> 8);
  const uint32_t sh = pk & 31u;
  const uint2* qp = &sm.qfrag[0][sm.plan.cls_hs0[ci]][lane];
  const uint32_t stride = 32u * (uint32_t)W;  // bytes per half step (8W words)
  const uint32_t w2 = 2u * (uint32_t)W;
  const uint8_t* lut = sm.lut;
  if (W <= 3) {
    const uint32_t m7 = ((1u << w2) - 1u) << 7;
    const uint32_t lb = lane4 | lut_rep(W);
#pragma unroll 2
    for (int i = 0; i < nhs; ++i, wp += stride, qp += 32) {
      const uint32_t v7 = funnel_r(ld32s(wp), ld32s(wp + 4), sh) << 7;
      uint32_t A[4];
      A[0] = ld32s(lut + ((v7 & m7) | lb));
      A[1] = ld32s(lut + (((v7 >> w2) & m7) | lb));
      A[2] = ld32s(lut + (((v7 >> (2u * w2)) & m7) | lb));
      A[3] = ld32s(lut + (((v7 >> (3u * w2)) & m7) | lb));
      key_mma<NT>(s, A, qp);
    }
  } else if (W == 4) {
#pragma unroll 2
    for (int i = 0; i < nhs; ++i, wp += stride, qp += 32) {
      uint32_t A[4];
      fields4<4>(lut, wp, sh, lane4, A);
      key_mma<NT>(s, A, qp);
    }
  } else if (W == 5) {
#pragma unroll 2
    for (int i = 0; i < nhs; ++i, wp += stride, qp += 32) {
      uint32_t A[4];
      fields4<5>(lut, wp, sh, lane4, A);
      key_mma<NT>(s, A, qp);
    }
  } else {
    // widths 6..8: two single-code lookups per pair (fp16 table, 2 bytes
    // each); window a holds the codes of tokens g, g + 8, window b of g + 16,
    // g + 24; code k of a window at byte 2 * code = (win >> (k W - 1)) & mw
    const uint8_t* tab = lut + kLutSingle + 2u * (uint32_t)((1 << W) - 2);
    const uint32_t mw = ((1u << W) - 1u) << 1;
    const uint32_t offb = 4u * ((sh + 4u * W) >> 5), shb = (sh + 4u * W) & 31u;
    const uint32_t s1 = (uint32_t)W - 1u, s2 = 2u * W - 1u, s3 = 3u * W - 1u;
#pragma unroll 2
    for (int i = 0; i < nhs; ++i, wp += stride, qp += 32) {
      const uint32_t ua = funnel_r(ld32s(wp), ld32s(wp + 4), sh);
      const uint32_t ub = funnel_r(ld32s(wp + offb), ld32s(wp + offb + 4), shb);
      uint32_t A[4];
      A[0] = ld16s(tab + ((ua << 1) & mw)) | (ld16s(tab + ((ua >> s1) & mw)) << 16);
      A[1] = ld16s(tab + ((ua >> s2) & mw)) | (ld16s(tab + ((ua >> s3) & mw)) << 16);
      A[2] = ld16s(tab + ((ub << 1) & mw)) | (ld16s(tab + ((ub >> s1) & mw)) << 16);
      A[3] = ld16s(tab + ((ub >> s2) & mw)) | (ld16s(tab + ((ub >> s3) & mw)) << 16);
      key_mma<NT>(s, A, qp);
    }
  }
}

// Inverse value rotation of one head held by a warp (o[128] in `src`),
// written as out[i] = s_i (H o)_i * inv.
__device__ __forceinline__ void warp_unrotate_store(const float* src, const Plan& pl, float inv,
                                                   float* out, int lane) {
  float y[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) y[q] = src[lane + 32 * q];
#pragma unroll
  for (int hh = 1; hh < 32; hh <<= 1) {
    const bool upper = (lane & hh) != 0;
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
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int i = lane + 32 * q;
    const float sgn = ((pl.v_sign[i >> 5] >> (i & 31)) & 1u) ? -1.f : 1.f;
    out[i] = sgn * y[q] * inv;
  }
}

// Window step (window kernels): the CTA's share of the window after the
// step, positions [w_lo, w_lo + w_n) of the sequence in chunks of 8 (chunk c
// to split c mod n_splits). A position below new_from is read from its ring
// slot; from new_from on it is a token of this step, read from the new rows
// (its ring slot is being written in this launch). Logits in fp32,
// s = (q . k) log2(e) / sqrt(128); values enter as H (s . v), the packed
// values' rotation. The CTA's record of its chunks (base-2 maximum, sum, o)
// goes to rec (8 NT records of kPartStride floats); returns whether it has
// chunks. qs: [G][128] floats; wsc: window scratch (kWinScratch floats).
constexpr int kWinTok = 8;  // window tokens staged at a time (one per warp)
constexpr int kWinScratch = kWinTok * (kHeadDim + 1) + kWinTok * kHeadDim + 16 * kWinTok + 48;

template <int NT>
__device__ __forceinline__ bool window_chunks(const DecodeParams& p, const Plan& pl, int b, int h,
                                           int split, int w_lo, int w_n, int64_t new_from,
                                           float* qs, float* wsc, float* rec, int tid) {
  if (split * kWinTok >= w_n) return false;  // CTA-uniform
  const int G = p.G, warp = tid >> 5, lane = tid & 31;
  float* ks = wsc;                            // [8][129]
  float* ys = ks + kWinTok * (kHeadDim + 1);  // [8][128]
  float* ps = ys + kWinTok * kHeadDim;        // [16][8]
  float* st = ps + 16 * kWinTok;              // max, sum, rescale per head
  for (int e = tid; e < G * kHeadDim; e += kThreads)
    qs[e] = load_as_float(p.q, p.q_dtype, ((size_t)b * p.n_q + (size_t)h * G) * kHeadDim + e) *
            0.12751743074f;  // log2(e) / sqrt(128)
  if (tid < 16) {
    st[tid] = -INFINITY;
    st[16 + tid] = 0.f;
  }
  uint32_t vsgn = 0;  // value signs of this lane's coordinates lane + 32 r
#pragma unroll
  for (int r = 0; r < 4; ++r) vsgn |= ((pl.v_sign[r] >> lane) & 1u) << r;
  const float* wk = p.wins[b];
  const float* wv = wk + (size_t)p.R * p.n_kv * kHeadDim;
  const int ci = tid & (kHeadDim - 1), cg = tid >> 7;  // o: coordinate, first head
  const int lt = tid & (kWinTok - 1), lg = tid >> 3;   // logit: token, head
  float o[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) o[k] = 0.f;
  __syncthreads();
  for (int c = split; c * kWinTok < w_n; c += p.n_splits) {
    const int c0 = w_lo + c * kWinTok, n = min(kWinTok, w_n - c * kWinTok);
    if (warp < n) {  // stage token `warp` of the chunk
      const int64_t pos = (int64_t)c0 + warp;
      float kx[4], y[4];
      if (pos >= new_from) {
        const size_t row = (((size_t)b * p.n_new + (size_t)(pos - new_from)) * p.n_kv + h) * kHeadDim;
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          kx[r] = load_as_float(p.k_new, p.kv_dtype, row + lane + 32 * r);
          const float x = load_as_float(p.v_new, p.kv_dtype, row + lane + 32 * r);
          y[r] = ((vsgn >> r) & 1u) ? -x : x;
        }
      } else {
        const size_t row = ((size_t)(pos % p.R) * p.n_kv + h) * kHeadDim;
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          kx[r] = wk[row + lane + 32 * r];
          const float x = wv[row + lane + 32 * r];
          y[r] = ((vsgn >> r) & 1u) ? -x : x;
        }
      }
#pragma unroll
      for (int r = 0; r < 4; ++r) ks[warp * (kHeadDim + 1) + lane + 32 * r] = kx[r];
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
      const float a0 = y[0] + y[1], a1 = y[0] - y[1], a2 = y[2] + y[3], a3 = y[2] - y[3];
      ys[warp * kHeadDim + lane] = a0 + a2;
      ys[warp * kHeadDim + lane + 32] = a1 + a3;
      ys[warp * kHeadDim + lane + 64] = a0 - a2;
      ys[warp * kHeadDim + lane + 96] = a1 - a3;
    }
    __syncthreads();
    if (lg < G) {  // logit of token lt for head lg (four partial sums)
      const float* kr = ks + lt * (kHeadDim + 1);
      const float* qr = qs + lg * kHeadDim;
      float a[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 8
      for (int i = 0; i < kHeadDim; i += 4) {
#pragma unroll
        for (int u = 0; u < 4; ++u) a[u] = fmaf(qr[i + u], kr[i + u], a[u]);
      }
      ps[lg * kWinTok + lt] = lt < n ? (a[0] + a[1]) + (a[2] + a[3]) : -INFINITY;
    }
    __syncthreads();
    for (int g = warp; g < G; g += kWarps) {  // running maximum, weights, sum
      const float sv = lane < kWinTok ? ps[g * kWinTok + lane] : -INFINITY;
      float mx = sv;
#pragma unroll
      for (int mm = 16; mm; mm >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, mm));
      const float m_old = st[g], m_new = fmaxf(m_old, mx);
      const bool none = m_new == -INFINITY;
      const float pr = none ? 0.f : ex2(sv - m_new);
      float sum = pr;
#pragma unroll
      for (int mm = 16; mm; mm >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, mm);
      if (lane < kWinTok) ps[g * kWinTok + lane] = pr;
      if (lane == 0) {
        const float alpha = none ? 1.f : ex2(m_old - m_new);  // 0 from -inf
        st[32 + g] = alpha;
        st[16 + g] = st[16 + g] * alpha + sum;
        st[g] = m_new;
      }
    }
    __syncthreads();
#pragma unroll
    for (int k = 0; k < 8; ++k) {  // o of coordinate ci for heads cg, cg + 2, ...
      const int g = cg + 2 * k;
      if (g < G) {
        const float* pg = ps + g * kWinTok;
        float acc = o[k] * st[32 + g];
#pragma unroll
        for (int t = 0; t < kWinTok; ++t)
          if (t < n) acc = fmaf(pg[t], ys[t * kHeadDim + ci], acc);
        o[k] = acc;
      }
    }
    __syncthreads();  // the next chunk overwrites the staged rows
  }
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const int g = cg + 2 * k;
    if (g < 8 * NT) rec[(size_t)g * kPartStride + kRecO + ci] = g < G ? o[k] : 0.f;
  }
  if (tid < 8 * NT) {
    rec[(size_t)tid * kPartStride] = tid < G ? st[tid] : -INFINITY;
    rec[(size_t)tid * kPartStride + 1] = tid < G ? st[16 + tid] : 0.f;
  }
  return true;
}

template <int BV, int NT, bool WIN>
__global__ void __launch_bounds__(kThreads, 2) decode_kernel(const DecodeParams p) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>(smem_raw);
  uint8_t* const scratch = smem_raw + sizeof(Smem);  // q' staging / append codes
  uint8_t* const stage_base = scratch + kScratch;

  const int split = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, c = lane & 3;
  const int G = p.G;
  const size_t bh = (size_t)b * p.n_kv + h;
  unsigned int* const cnt = reinterpret_cast<unsigned int*>(p.pb_end - (bh + 1) * kPairBlockBytes);
  unsigned int* const seq_cnt =
      reinterpret_cast<unsigned int*>(p.pb_end - ((size_t)b * p.n_kv + 1) * kPairBlockBytes) +
      (kPairCntWords - 1);


  // ---- independent of earlier kernels: barriers, plan and lookup image
  if (tid == 0) {
    mbar_init(&sm.setup_bar, 1);
    mbar_init(&sm.stall_bar, 1);
    for (int i = 0; i < kWarps * kStages; ++i) mbar_init(&sm.bar[i / kStages][i % kStages], 1);
    fence_proxy_async();
    const uint32_t thr_bytes = p.n_new > 0 ? (uint32_t)sizeof(g_thr) : 0u;
    mbar_expect_tx(&sm.setup_bar, KVQ_PLAN_BYTES + KVQ_LUT_BYTES + thr_bytes);
    bulk_g2s(&sm.plan, p.plans[b] + h, KVQ_PLAN_BYTES, &sm.setup_bar);
    bulk_g2s(sm.lut, g_lut_image, KVQ_LUT_BYTES, &sm.setup_bar);
    if (thr_bytes) bulk_g2s(sm.thr, g_thr, thr_bytes, &sm.setup_bar);
    sm.flags = 0u;
  }
  if (p.rope)
    for (int i = tid; i < 64; i += kThreads) sm.theta[i] = p.theta[i];
  {  // this CTA's query rows into L2 while the previous kernel finishes
    const size_t esz = (p.q_dtype == KVQ_BF16 || p.q_dtype == KVQ_FP16) ? 2 : 4;
    const uintptr_t q0 =
        reinterpret_cast<uintptr_t>(p.q) + ((size_t)b * p.n_q + (size_t)h * G) * kHeadDim * esz;
    const uintptr_t q1 = q0 + (size_t)G * kHeadDim * esz;
    for (uintptr_t a = (q0 & ~(uintptr_t)127) + (uintptr_t)tid * 128; a < q1; a += kThreads * 128)
      prefetch_l2(reinterpret_cast<const void*>(a < q0 ? q0 : a));
  }
  // ---- with `early` the caller guarantees that the previous kernel on the
  //      stream writes neither these caches nor these lengths: the length is
  //      read and the first tiles are streamed before waiting for it
  if (!p.early) grid_dep_wait();
  if (tid == 0) {
    const int l0 = p.len[b];
    sm.len0 = l0;
    int w0 = 0;
    if constexpr (WIN) {
      w0 = min(max(p.wlen[b], 0), p.R);
      sm.w0 = w0;
    }
    if (p.n_new > 0) {
      // the last CTA of the sequence to read its length writes the new one;
      // the counter wraps to zero in the same atomic, so a kernel that starts
      // before this one has ended finds it at zero
      __threadfence();
      const unsigned int total = (unsigned int)(p.n_kv * p.n_splits);
      if (atomicInc(seq_cnt, total - 1u) == total - 1u) {
        const int64_t lim = min((int64_t)p.max_len, p.cap);
        if constexpr (WIN) {  // the tokens leaving the window join the packed cache
          const int e = max(0, w0 + p.n_new - p.R);
          if (l0 >= 0 && (int64_t)l0 + e <= lim) {
            p.len[b] = l0 + e;
            p.wlen[b] = min(p.R, w0 + p.n_new);
          }
        } else {
          if (l0 >= 0 && (int64_t)l0 + p.n_new <= lim) p.len[b] = l0 + p.n_new;
        }
      }
    }
  }
  __syncthreads();
  const bool ok_setup = mbar_wait_bounded(&sm.setup_bar, 0u);
  const uint8_t* const cache0 = p.cm.table ? nullptr : p.cm.caches[b];  // contiguous base
  const int bk = sm.plan.bits_k;
  const int n_half = sm.plan.n_half;
  // Bounds that keep every index the kernel takes from the plan in range,
  // whatever its other bytes (the block pass of an append also masks its
  // word index); the full check of the schedule (plan_sched_ok) runs where
  // it costs no time, in split 0 during its arrival, and only flags
  bool bad = !ok_setup || sm.plan.magic != KVQ_PLAN_MAGIC || sm.plan.bits_v != BV ||
             bk < 1 || bk > 8 || p.tile_bytes != tile_bytes(bk, BV) || n_half < 1 ||
             n_half > kMaxHalf || sm.plan.n_class < 1 || sm.plan.n_class > 8 ||
             sm.plan.n_ranks < 1 || sm.plan.n_ranks > 64 ||
             (reinterpret_cast<uintptr_t>(cache0) & 15) != 0;
  // width classes: every word a class reads must lie in the tile's key words
  // plus the one half step of overrun a partial last half step allows
  for (int ci = 0; !bad && ci < sm.plan.n_class; ++ci) {
    const int W = sm.plan.cls_w[ci], hs0 = sm.plan.cls_hs0[ci], nhs = sm.plan.cls_nhs[ci];
    bad = W < 1 || W > 8 || nhs < 1 || hs0 + nhs > n_half ||
          sm.plan.cls_seg0[ci] + 8 * W * nhs > 128 * bk + 64;
  }
  if (bad && tid == 0) atomicOr(p.status, ok_setup ? KVQ_FLAG_BAD_PLAN : KVQ_FLAG_TIMEOUT);
  const int len0 = sm.len0;
  int n_add = 0;
  bool step_ok = false;  // the step's append fits (window: its evictions)
  if (p.n_new > 0) {
    const int64_t lim = min((int64_t)p.max_len, p.cap);
    int want = p.n_new;
    if constexpr (WIN) want = max(0, sm.w0 + p.n_new - p.R);
    if (len0 >= 0 && (int64_t)len0 + want <= lim) {
      n_add = want;
      step_ok = true;
    } else if (tid == 0 && split == 0 && h == 0) {
      atomicOr(p.status, KVQ_FLAG_CAPACITY);
    }
  }
  int L = bad ? 0 : len0 + n_add;
  if (L > p.max_len) {
    if (tid == 0 && split == 0 && h == 0) atomicOr(p.status, KVQ_FLAG_CAPACITY);
    L = p.max_len;
  }
  L = max(L, 0);
  const int n_tiles = (L + kTile - 1) / kTile;
  const int tb = split * p.tiles_per_split;
  const int te = min(n_tiles, tb + p.tiles_per_split);
  const bool has_work = tb < te;

  // ---- start streaming the warp's first tiles. Warp w takes tiles
  //      te - 1 - w - 8 i, so the tiles a fused append writes (the last tiles
  //      of the sequence) are the first tiles of warps 0..2.
  const int tbytes = p.tile_bytes;
  uint8_t* const my_stages = stage_base + (size_t)warp * kStages * tbytes;
  const int n_mine = has_work ? max(0, (te - tb - warp + kWarps - 1) / kWarps) : 0;
  const int pmask = page_mask(p.cm);
  auto tile_of = [&](int i) { return te - 1 - warp - i * kWarps; };
  // page base of the warp's i-th tile (a paged cache looks it up in the block
  // table; lane 0 does so one tile ahead of the copy that needs it)
  auto base_of = [&](int i) { return p.cm.table ? page_base(p.cm, b, tile_of(i)) : cache0; };
  auto issue = [&](int i, const uint8_t* base) {
    const int s = i % kStages;
    unsigned long long* bar = &sm.bar[warp][s];
    const uint8_t* src = reinterpret_cast<const uint8_t*>(g_lut_image);
    if (base)
      src = base + ((size_t)(tile_of(i) & pmask) * p.n_kv + h) * tbytes;
    else  // refused page: placeholder bytes are streamed, the output is flagged
      atomicOr(p.status, KVQ_FLAG_BAD_PAGE);
    mbar_expect_tx(bar, (uint32_t)tbytes);
    bulk_g2s(my_stages + s * tbytes, src, (uint32_t)tbytes, bar);
  };
  const uint8_t* next_base = nullptr;  // lane 0: base of tile kStages, kStages + 1, ...
  if (lane == 0) {
    for (int i = 0; i < min(kStages, n_mine); ++i) issue(i, base_of(i));
    if (kStages < n_mine) next_base = base_of(kStages);
  }
  // appended tiles of this CTA: [a_lo, a_hi] (CTA-uniform)
  const int a_lo = n_add > 0 ? max(len0 / kTile, tb) : 1;
  const int a_hi = n_add > 0 ? min((len0 + n_add - 1) / kTile, te - 1) : 0;
  const bool appends = has_work && a_lo <= a_hi;
  if (!WIN && appends) {  // the new tokens' rows into L2 (no value read before the wait)
    const size_t esz = (p.kv_dtype == KVQ_BF16 || p.kv_dtype == KVQ_FP16) ? 2 : 4;
    const int lines = (int)(kHeadDim * esz / 128);
    const int j0 = max(len0, a_lo * kTile) - len0, j1 = min(len0 + n_add, a_hi * kTile + kTile) - len0;
    for (int e = tid; e < (j1 - j0) * lines * 2; e += kThreads) {
      const int j = j0 + e / (2 * lines), l = e % lines;
      const void* src = (e / lines) % 2 ? p.v_new : p.k_new;
      prefetch_l2(reinterpret_cast<const uint8_t*>(src) +
                  ((((size_t)b * p.n_new + j) * p.n_kv + h) * kHeadDim) * esz + (size_t)l * 128);
    }
  }
  // plan-only part of the query prologue: MMA column -> RoPE block per half
  // step, and each width class's first word and bit shift per lane
  if (!bad) {
    for (int e = tid; e < n_half * 4; e += kThreads) {
      const int hs = e >> 2, cc = e & 3;
      sm.qj[hs][cc] = cc < sm.plan.hs_count[hs]
                          ? (int8_t)sm.plan.order[sm.plan.hs_rank0[hs] + cc] : (int8_t)-1;
    }
    for (int e = tid; e < sm.plan.n_class * 32; e += kThreads) {
      const int ci = e >> 5, ln = e & 31, W = sm.plan.cls_w[ci];
      const int off = sm.plan.cls_seg0[ci] + 2 * W * (ln & 3) + ((W * (ln >> 2)) >> 2);
      sm.cls_lane[ci][ln] = ((uint32_t)off << 8) | ((uint32_t)(8 * W * (ln >> 2)) & 31u);
    }
    if (sm.plan.k_rot) rot_tables(sm.plan, sm.rot, tid);
  }
  __syncthreads();  // the tables above are read by every warp
  if (p.early) grid_dep_wait();
  grid_dep_launch();

  // ---- fused append: quantize the new tokens of the appended tiles, then
  //      patch them into the streamed copy of each tile (stage 0 of warp
  //      te - 1 - tile) and into the cache
  if (appends) {
    float* kz = reinterpret_cast<float*>(scratch);                          // [32][129]
    __half* nrm_new = reinterpret_cast<__half*>(scratch + kTile * kKzStride * 4);  // [2][32]
    uint32_t flags = 0;
    for (int tile = a_lo; tile <= a_hi; ++tile) {
      const int t_lo = max(len0, tile * kTile), t_hi = min(len0 + n_add, tile * kTile + kTile);
      const int p_lo = t_lo - tile * kTile, p_hi = t_hi - tile * kTile;
      const int w_own = te - 1 - tile;
      const uint8_t* pb = page_base(p.cm, b, tile);
      uint8_t* rec = pb ? const_cast<uint8_t*>(pb) + ((size_t)(tile & pmask) * p.n_kv + h) * tbytes
                        : nullptr;
      uint8_t* st = stage_base + (size_t)w_own * kStages * tbytes;
      uint32_t* sw = reinterpret_cast<uint32_t*>(st);
      const int n_words = kHeadDim * (bk + BV);
      const bool clear = len0 > tile * kTile;  // the tile already holds tokens
      const bool ok = mbar_wait_bounded(&sm.bar[w_own][0], 0u);  // the old tile is in `st`
      if (!clear)
        for (int i = tid; i < n_words; i += kThreads) sw[i] = 0u;
      __syncthreads();
      // pass 1 (one warp per new token; the word after the packed words, the
      // first norm word of the copy, takes only no-op atomics), then pass 2
      for (int pp = p_lo + warp; pp < p_hi; pp += kWarps) {
        const int j = tile * kTile + pp - len0;  // j-th appended token
        size_t row = (((size_t)b * p.n_new + j) * p.n_kv + h) * kHeadDim;
        const void* ksrc = p.k_new;
        const void* vsrc = p.v_new;
        int dt = p.kv_dtype;
        if constexpr (WIN) {  // a token leaving the window: its ring row (fp32)
          row = ((size_t)(((int64_t)len0 + j) % p.R) * p.n_kv + h) * kHeadDim;
          ksrc = p.wins[b];
          vsrc = p.wins[b] + (size_t)p.R * p.n_kv * kHeadDim;
          dt = KVQ_FP32;
        }
        __half kn, vn;
        warp_token_pass<BV>(sm.plan, sm.thr, ksrc, vsrc, dt, row, lane, pp,
                            kz + pp * kKzStride, sw, clear, kn, vn, flags,
                            p.rope ? sm.theta : nullptr, (int64_t)tile * kTile + pp);
        if (lane == 0) {
          nrm_new[pp] = kn;
          nrm_new[kTile + pp] = vn;
        }
      }
      __syncthreads();
      if (sm.plan.k_rot) {  // key rotation inside width groups, one warp per new token
        for (int pp = p_lo + warp; pp < p_hi; pp += kWarps)
          warp_rotate_row(kz + pp * kKzStride, sm.plan, sm.rot, sm.plan.g, lane);
        __syncthreads();
      }
      for (int r = warp; r < sm.plan.n_ranks; r += kWarps)
        warp_block_pass(sm.plan, sm.thr, r, kz, p_lo, p_hi, lane, sw, clear);
      __syncthreads();
      if (ok && rec) {
        uint32_t* gw = reinterpret_cast<uint32_t*>(rec);
        for (int i = tid; i < n_words; i += kThreads) gw[i] = sw[i];
        for (int e = tid; e < 2 * (p_hi - p_lo); e += kThreads) {
          const int pp = p_lo + (e >> 1), off = (e & 1) * kTile + pp;
          reinterpret_cast<__half*>(rec + 512 * (bk + BV))[off] = nrm_new[off];
          reinterpret_cast<__half*>(st + 512 * (bk + BV))[off] = nrm_new[off];
        }
      } else {
        flags |= ok ? KVQ_FLAG_BAD_PAGE : KVQ_FLAG_TIMEOUT;
      }
      __syncthreads();
    }
    if (flags) atomicOr(&sm.flags, flags);
    fence_proxy_async();  // patched stages are later overwritten by bulk copies
    __syncthreads();
    if (tid == 0 && sm.flags) atomicOr(p.status, sm.flags);
  }
  if constexpr (WIN) {
    // the new tokens into their ring slots. New token j takes the slot of
    // position len0 + w0 + j - R: a token that left the window in this
    // launch (the CTA that appended it writes the slot, after reading it
    // above) or one that left before (a free slot, written by the CTA that
    // owns the last packed tile). No CTA reads those slots otherwise.
    if (step_ok && !bad) {
      const int ring_split = min(p.n_splits - 1, ((max(L, 1) - 1) / kTile) / p.tiles_per_split);
      float* wk = p.wins[b];
      float* wv = wk + (size_t)p.R * p.n_kv * kHeadDim;
      for (int e = tid; e < p.n_new * kHeadDim; e += kThreads) {
        const int j = e / kHeadDim, x = e % kHeadDim;
        const int64_t pos = (int64_t)len0 + sm.w0 + j - p.R;  // the slot's previous token
        const int owner = pos < len0 ? ring_split : (int)((pos / kTile) / p.tiles_per_split);
        if (owner != split) continue;
        const size_t dst = ((size_t)((pos + p.R) % p.R) * p.n_kv + h) * kHeadDim + x;
        const size_t src = (((size_t)b * p.n_new + j) * p.n_kv + h) * kHeadDim + x;
        wk[dst] = load_as_float(p.k_new, p.kv_dtype, src);
        wv[dst] = load_as_float(p.v_new, p.kv_dtype, src);
      }
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

  if (has_work) {
    // ---- query prologue (q' staged in the tile ring before it is used):
    //      q' = q a_hat_j log2(e) / sqrt(128); per-head 2^sigma scaling into
    //      the fp16 range; hi/lo split into the B fragments of each half step
    float* qp = reinterpret_cast<float*>(scratch);  // [8 NT][128]
    const bool krot = sm.plan.k_rot != 0;
    for (int head = warp; head < 8 * NT; head += kWarps) {  // warp-local: one head each
      float* row = qp + head * kHeadDim;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int x = lane + 32 * i;
        float v = 0.f;
        if (head < G) {
          const size_t qi = ((size_t)b * p.n_q + h * G + head) * kHeadDim + x;
          v = load_as_float(p.q, p.q_dtype, qi) * sm.plan.a_hat[x & 63] * 0.12751743074f;
        }  // 0.12751743 = log2(e) / sqrt(128)
        row[x] = v;
      }
      __syncwarp();
      // rotated plans: the same per-chunk rotation as the keys, so that
      // q'~ . y_hat = q' . z_hat; the row is then indexed by plan position
      if (krot) warp_rotate_row(row, sm.plan, sm.rot, nullptr, lane);
      float mx = 0.f;
#pragma unroll
      for (int i = 0; i < 4; ++i)
        if (!krot || lane + 32 * i < sm.rot.npos) mx = fmaxf(mx, fabsf(row[lane + 32 * i]));
#pragma unroll
      for (int m = 16; m; m >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, m));
      const int sigma = (mx > 0.f && isfinite(mx)) ? 14 - ilogbf(mx) : 0;
      const float sc = ldexpf(1.f, sigma);
      if (lane == 0) sm.inv_scale[head] = ldexpf(1.f, -sigma);
      // this head's B-fragment entries: lane 4 (head mod 8) + c of each half step
      const int nt = head >> 3, g8 = head & 7;
      for (int e = lane; e < n_half * 4; e += 32) {
        const int hs = e >> 2, cc = e & 3, j = sm.qj[hs][cc];
        float x0 = 0.f, x1 = 0.f;
        if (j >= 0) {
          const int i0 = krot ? 2 * (sm.plan.hs_rank0[hs] + cc) : j;
          x0 = row[i0] * sc;
          x1 = row[krot ? i0 + 1 : j + 64] * sc;
        }
        const uint32_t hi = pack_half2(x0, x1);
        const __half2 hh = *reinterpret_cast<const __half2*>(&hi);
        const uint32_t lo = pack_half2(x0 - __low2float(hh), x1 - __high2float(hh));
        sm.qfrag[nt][hs][4 * g8 + cc] = make_uint2(hi, lo);
      }
    }
    __syncthreads();

    // ---- per-warp pipeline over the warp's tiles
    __syncwarp();

    const uint32_t lane4 = (uint32_t)lane * 4u;
    const int n_class = sm.plan.n_class;
    const uint32_t v_sh = (uint32_t)(8 * BV * c) & 31u;
    const int v_off = 4 * (g * BV + ((BV * c) >> 2));  // row g of each m-tile, lane's slots
    int consumed = 0;
    bool timed_out = false;
    if (p.stall_cycles > 0)  // test hook: a wait that runs out, then the timeout path
      timed_out = !__all_sync(0xffffffffu, mbar_wait_bounded(&sm.stall_bar, 0u, p.stall_cycles));
    for (int i = 0; i < n_mine && !timed_out; ++i) {
      const int s = i % kStages;
      const bool ok = mbar_wait_bounded(&sm.bar[warp][s], (uint32_t)((i / kStages) & 1));
      if (!__all_sync(0xffffffffu, ok)) {
        timed_out = true;
        break;
      }
      consumed = i + 1;
      const int tile = tile_of(i);
      const int nvalid = min(kTile, L - tile * kTile);
      const uint8_t* kw = my_stages + s * tbytes;
      const uint8_t* vw = kw + 512 * bk + v_off;
      const __half* nrm = reinterpret_cast<const __half*>(kw + 512 * (bk + BV));

      // keys: S[32 tokens x 8 NT heads] on the tensor cores
      float sacc[2][NT][4];
#pragma unroll
      for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
          for (int r = 0; r < 4; ++r) sacc[mt][nt][r] = 0.f;
      for (int ci = 0; ci < n_class; ++ci) key_class<NT>(sm, kw, ci, lane, lane4, sacc);

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
      // scores in base 2; a head's reference m_run only moves when a score
      // passes it (lazy rescaling, warp-uniform test), and then to the
      // tile's maximum plus kHeadroom, so 2^(s - m_run) <= 1 always and most
      // tiles skip the maximum reduction and the rescale of o
      float sv[NT][2][4];
      bool up = false;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const float isc = sm.inv_scale[8 * nt + 2 * c + e];
#pragma unroll
          for (int r = 0; r < 4; ++r) {
            const int mt = r >> 1, rr = r & 1;
            sv[nt][e][r] = val[r] ? sacc[mt][nt][2 * rr + e] * (nk[r] * isc) : -INFINITY;
            up |= sv[nt][e][r] > m_run[nt][e];
          }
        }
      if (__any_sync(0xffffffffu, up)) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            float mx = fmaxf(fmaxf(sv[nt][e][0], sv[nt][e][1]), fmaxf(sv[nt][e][2], sv[nt][e][3]));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
            if (mx > m_run[nt][e]) {
              const float m_new = mx + kHeadroom;
              const float alpha = ex2(m_run[nt][e] - m_new);  // 0 from -inf
              l_run[nt][e] *= alpha;
#pragma unroll
              for (int mu = 0; mu < 8; ++mu) {
                o[mu][nt][e] *= alpha;
                o[mu][nt][2 + e] *= alpha;
              }
              m_run[nt][e] = m_new;
            }
          }
      }
      uint32_t pb0[2][NT], pb1[2][NT];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        float pe[2][4];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          // m_run is finite here: every processed tile holds a valid token
          float lsum = 0.f;
#pragma unroll
          for (int r = 0; r < 4; ++r) {
            const float pr = ex2(sv[nt][e][r] - m_run[nt][e]);  // 0 for masked tokens
            lsum += pr;
            pe[e][r] = pr * nv[r];
          }
          l_run[nt][e] += lsum;
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
        fields4<BV>(sm.lut, vw + 4 * (16 * mu * BV), v_sh, lane4, F0);
        fields4<BV>(sm.lut, vw + 4 * ((16 * mu + 8) * BV), v_sh, lane4, F1);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          mma_16816(o[mu][nt], F0[0], F1[0], F0[1], F1[1], pb0[0][nt], pb1[0][nt]);
          mma_16816(o[mu][nt], F0[2], F1[2], F0[3], F1[3], pb0[1][nt], pb1[1][nt]);
        }
      }
      __syncwarp();
      if (lane == 0 && i + kStages < n_mine) {
        fence_proxy_async();
        issue(i + kStages, next_base);
        if (i + kStages + 1 < n_mine) next_base = base_of(i + kStages + 1);
      }
    }
    if (timed_out) {
      if (lane == 0) atomicOr(p.status, KVQ_FLAG_TIMEOUT);
      // let the copies this warp still has in flight land before leaving
      for (int i = consumed; i < min(n_mine, consumed + kStages); ++i)
        (void)mbar_wait_bounded(&sm.bar[warp][i % kStages], (uint32_t)((i / kStages) & 1));
    }
  }

  // ---- warps -> one (m, l, o) per head in shared memory -> this split's record
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
  int n_rec = kWarps;  // records of the CTA merge
  if constexpr (WIN) {
    // the window after the step: [L, L + w_n) (the step's new token last)
    const int w_n = bad ? 0 : (step_ok ? min(p.R, sm.w0 + p.n_new) : sm.w0);
    if (window_chunks<NT>(p, sm.plan, b, h, split, L, w_n, (int64_t)len0 + sm.w0,
                          reinterpret_cast<float*>(scratch), mg + (kWarps + 1) * 8 * NT * kPartStride,
                          mg + kWarps * 8 * NT * kPartStride, tid))
      n_rec = kWarps + 1;
    __syncthreads();
  }
  // ---- this split's record, then its contribution to the exponent buckets:
  //      head hd with max m adds 2^(m - 32 kk) (l, o), kk = floor(m / 32), to
  //      bucket kk by L2 atomics, so the splits are summed in L2 without a
  //      merge tree; a max outside [-256, 256) flags the pair for a merge of
  //      all records instead
  float* const my_part = p.part + (bh * p.n_splits + split) * G * kPartStride;
  float* const crec = reinterpret_cast<float*>(scratch);  // [G][132]
  unsigned int* const ovf = cnt + 1;
  unsigned int* const bmask = cnt + 2;  // [G]: buckets in use
  float* const bkt = reinterpret_cast<float*>(cnt + kPairCntWords);  // [G][kBuckets][132]
  for (int item = tid; item < G * 32; item += kThreads) {
    const int hd = item >> 5, x4 = (item & 31) * 4;
    float m, l;
    float4 ov;
    merge_item<kWarps>(mg + hd * kPartStride, n_rec, (size_t)8 * NT * kPartStride, x4, m, l, ov);
    *reinterpret_cast<float4*>(crec + hd * kPartStride + kRecO + x4) = ov;
    *reinterpret_cast<float4*>(my_part + hd * kPartStride + kRecO + x4) = ov;
    if (x4 == 0) {
      crec[hd * kPartStride] = m;
      crec[hd * kPartStride + 1] = l;
      my_part[hd * kPartStride] = m;
      my_part[hd * kPartStride + 1] = l;
    }
    if (m == -INFINITY || p.deterministic) continue;  // no tokens, or merged in order
    const float kf = floorf(m * (1.f / 32.f));
    if (!(kf >= -8.f && kf < 8.f)) {
      if (x4 == 0) atomicOr(ovf, 1u);
      continue;
    }
    const int kk = (int)kf + 8;
    const float sc = ex2(m - 32.f * kf);  // in [1, 2^32)
    float* dst = bkt + (hd * kBuckets + kk) * kPartStride;
    red_add_v4(dst + kRecO + x4, ov.x * sc, ov.y * sc, ov.z * sc, ov.w * sc);
    if (x4 == 0) {
      atomicAdd(dst + 1, l * sc);
      atomicOr(bmask + hd, 1u << kk);
    }
  }
  __syncthreads();
  if (tid == 0) {
    sm.is_last = arrive_last(&cnt[0], (unsigned int)p.n_splits);
  } else if (warp == 1 && split == 0 && !bad) {
    // during the arrival's round trip: the full plan check (flag only; the
    // bounds checked up front keep every index of the decode in range)
    if (!plan_sched_ok(sm.plan, lane) && lane == 0) atomicOr(p.status, KVQ_FLAG_BAD_PLAN);
  }
  __syncthreads();
  if (!sm.is_last) return;

  // ---- the last split of the pair: sum the buckets (or merge all records),
  //      clear what this call used, undo the value rotation, write o / l.
  //      Reads go to L2 (ld.cg): the atomics were performed there.
  float* fin = reinterpret_cast<float*>(stage_base);  // [G][132]
  // one round of L2 loads (ld.cg: the atomics were performed there): the
  // overflow flag, each item's bucket mask, and the three buckets around this
  // split's own for the item's head (the usual ones)
  constexpr int kItems = (16 * 32 + kThreads - 1) / kThreads;  // items per thread
  const unsigned int ovf_v = __ldcg(ovf);
  unsigned int msk[kItems];
  int k0[kItems];
  float4 pre[kItems][3];
  float pl[kItems][3];
#pragma unroll
  for (int it = 0; it < kItems; ++it) {
    const int item = tid + it * kThreads;
    msk[it] = 0u;
    k0[it] = 0;
    if (item < G * 32) {
      const int hd = item >> 5, x4 = (item & 31) * 4;
      const float m_own = crec[hd * kPartStride];
      const int k_own = m_own == -INFINITY ? 8 : (int)floorf(m_own * (1.f / 32.f)) + 8;
      k0[it] = min(max(k_own - 1, 0), kBuckets - 3);
#pragma unroll
      for (int j = 0; j < 3; ++j) {
        const float* src = bkt + (hd * kBuckets + k0[it] + j) * kPartStride;
        pre[it][j] = __ldcg(reinterpret_cast<const float4*>(src + kRecO + x4));
        pl[it][j] = x4 == 0 ? __ldcg(src + 1) : 0.f;
      }
      msk[it] = __ldcg(bmask + hd);
    }
  }
  if (ovf_v == 0u && !p.deterministic) {
#pragma unroll
    for (int it = 0; it < kItems; ++it) {
      const int item = tid + it * kThreads;
      if (item >= G * 32) continue;
      const int hd = item >> 5, x4 = (item & 31) * 4;
      const unsigned int mask = msk[it];
      float L = 0.f;
      float4 O = make_float4(0.f, 0.f, 0.f, 0.f);
      if (mask) {
        const int kmax = 31 - __clz(mask);
        for (unsigned int mm = mask; mm; mm &= mm - 1u) {
          const int kk = __ffs(mm) - 1, d = kk - k0[it];
          const float w = ex2(32.f * (float)(kk - kmax));  // 2^(-32 j), exact
          float4 v;
          float lv;
          if (d >= 0 && d < 3) {
            v = d == 0 ? pre[it][0] : d == 1 ? pre[it][1] : pre[it][2];
            lv = d == 0 ? pl[it][0] : d == 1 ? pl[it][1] : pl[it][2];
          } else {
            const float* src = bkt + (hd * kBuckets + kk) * kPartStride;
            v = __ldcg(reinterpret_cast<const float4*>(src + kRecO + x4));
            lv = x4 == 0 ? __ldcg(src + 1) : 0.f;
          }
          O.x += w * v.x;
          O.y += w * v.y;
          O.z += w * v.z;
          O.w += w * v.w;
          L += w * lv;
        }
      }
      *reinterpret_cast<float4*>(fin + hd * kPartStride + kRecO + x4) = O;
      if (x4 == 0) {  // (L, O) are 2^-(32 (kmax - 8)) times the split sums
        fin[hd * kPartStride] = mask ? 32.f * (float)(31 - __clz(mask) - 8) : -INFINITY;
        fin[hd * kPartStride + 1] = L;
      }
    }
  } else {
    merge_records<kThreads>(p.part + bh * p.n_splits * G * kPartStride, p.n_splits,
                            (size_t)G * kPartStride, G, fin);
  }
  __syncthreads();
  // clear the buckets this call used (the masks were read with the sums)
#pragma unroll
  for (int it = 0; it < kItems; ++it) {
    const int item = tid + it * kThreads;
    if (item >= G * 32) continue;
    const int hd = item >> 5, x4 = (item & 31) * 4;
    for (unsigned int mm = msk[it]; mm; mm &= mm - 1u) {
      float* dst = bkt + (hd * kBuckets + __ffs(mm) - 1) * kPartStride;
      *reinterpret_cast<float4*>(dst + kRecO + x4) = make_float4(0.f, 0.f, 0.f, 0.f);
      if (x4 == 0) dst[1] = 0.f;
    }
  }
  __syncthreads();
  if (tid < G) bmask[tid] = 0u;
  if (tid == 0) *ovf = 0u;
  if (p.rec_out) {  // partial decode: the merged record, still rotated
    float* dst = p.rec_out + ((size_t)b * p.n_q + (size_t)h * G) * kPartStride;
    for (int i = tid; i < G * kPartStride / 4; i += kThreads)
      reinterpret_cast<float4*>(dst)[i] = reinterpret_cast<const float4*>(fin)[i];
    return;
  }
  for (int head = warp; head < G; head += kWarps) {
    const float* r = fin + (size_t)head * kPartStride;
    const float inv = r[1] > 0.f ? 1.f / (128.f * r[1]) : 0.f;
    warp_unrotate_store(r + kRecO, sm.plan, inv,
                        p.out + ((size_t)b * p.n_q + h * G + head) * kHeadDim, lane);
  }
}

// Merge of the records of n_parts partial decodes (context shards of the same
// sequences: part r's record of query head i at recs + (r * batch * n_q + i)
// * 132) and the inverse value rotation, o = s . H o_rot / (128 l). One CTA per
// (KV head, sequence).
__global__ void __launch_bounds__(kThreads) combine_kernel(const Plan* const* plans,
                                                           const float* recs, int n_parts,
                                                           int batch, int n_q, int n_kv,
                                                           float* out) {
  __shared__ __align__(16) float fin[16 * kPartStride];
  const int h = blockIdx.x, b = blockIdx.y, G = n_q / n_kv;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const size_t head0 = (size_t)b * n_q + (size_t)h * G;
  merge_records<kThreads>(recs + head0 * kPartStride, n_parts,
                          (size_t)batch * n_q * kPartStride, G, fin);
  __syncthreads();
  const Plan& pl = plans[b][h];
  for (int head = warp; head < G; head += kWarps) {
    const float* r = fin + (size_t)head * kPartStride;
    const float inv = r[1] > 0.f ? 1.f / (128.f * r[1]) : 0.f;
    warp_unrotate_store(r + kRecO, pl, inv, out + (head0 + head) * kHeadDim, lane);
  }
}

// ------------------------------------------------------------- launchers
size_t decode_smem_bytes(int tile_bytes, int nt, bool win = false) {
  const size_t stages = (size_t)kWarps * kStages * tile_bytes;
  const size_t merge = (size_t)kWarps * 8 * nt * kPartStride * sizeof(float);
  // window step: one more record (the window's) and the window scratch
  const size_t merge_win =
      ((size_t)(kWarps + 1) * 8 * nt * kPartStride + kWinScratch) * sizeof(float);
  return sizeof(Smem) + kScratch + std::max(stages, win ? merge_win : merge);
}
static_assert(16 * kHeadDim * sizeof(float) <= (size_t)kScratch, "window q' in the scratch");

// CTAs per SM of one instantiation for tiles of (bits_k, BV), queried once per
// device and bits_k. The first query also raises the dynamic shared-memory cap
// of the instantiation to its largest tile, so later calls (also under stream
// capture) only launch.
template <int BV, int NT>
static int ctas_per_sm(int dev, int bits_k, cudaError_t* err) {
  static std::atomic<int> cache[64][9];
  static std::atomic<unsigned long long> cap_set{0};
  std::atomic<int>& slot = cache[dev & 63][(bits_k & 7) ? bits_k : 8];
  int v = slot.load();
  if (v > 0) return v;
  cudaError_t e = cudaSuccess;
  const unsigned long long bit = 1ull << (dev & 63);
  if (!(cap_set.load() & bit)) {
    e = cudaFuncSetAttribute(decode_kernel<BV, NT, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)decode_smem_bytes(tile_bytes(8, BV), NT));
    if (e == cudaSuccess) cap_set.fetch_or(bit);
  }
  if (e == cudaSuccess)
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(
        &v, decode_kernel<BV, NT, false>, kThreads, decode_smem_bytes(tile_bytes(bits_k, BV), NT));
  if (e != cudaSuccess) {
    *err = e;
    return 0;
  }
  v = std::max(v, 1);
  slot.store(v);
  return v;
}

template <int NT>
static int ctas_per_sm_bv(int dev, int bits_k, int bv, cudaError_t* err) {
  switch (bv) {
    case 1: return ctas_per_sm<1, NT>(dev, bits_k, err);
    case 2: return ctas_per_sm<2, NT>(dev, bits_k, err);
    case 3: return ctas_per_sm<3, NT>(dev, bits_k, err);
    case 4: return ctas_per_sm<4, NT>(dev, bits_k, err);
    case 5: return ctas_per_sm<5, NT>(dev, bits_k, err);
    case 6: return ctas_per_sm<6, NT>(dev, bits_k, err);
    case 7: return ctas_per_sm<7, NT>(dev, bits_k, err);
    default: return ctas_per_sm<8, NT>(dev, bits_k, err);
  }
}

struct SplitPlan {
  int n_splits, tiles_per_split;
  int64_t slots;  // bound on the CTA slots of any decode launch on the device
};

constexpr int kMaxCtasPerSm = 2;  // the launch bounds' residency, also the grid's cap

// Splits per (sequence, KV head) so that the grid is about one wave of the
// current device, with at least one tile per warp. Without a device (size
// queries on a host without GPU) an upper bound of the CTA slots is used.
static SplitPlan decode_split_plan(int batch, int n_kv, int G, int bits_k, int bits_v,
                                   int64_t max_len, cudaError_t* err, bool allow_fallback) {
  SplitPlan sp{1, 1, kFallbackSlots};
  int64_t slots = kFallbackSlots;
  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  int per_sm = 0;
  if (e == cudaSuccess)
    per_sm = G <= 8 ? ctas_per_sm_bv<1>(dev, bits_k, bits_v, &e)
                    : ctas_per_sm_bv<2>(dev, bits_k, bits_v, &e);
  if (e == cudaSuccess) {
    slots = (int64_t)sms * std::min(per_sm, kMaxCtasPerSm);
    sp.slots = (int64_t)sms * kMaxCtasPerSm;  // the same for every bit budget
  } else if (!allow_fallback) {
    *err = e;
    return sp;
  } else {
    (void)cudaGetLastError();
  }
  *err = cudaSuccess;
  const int64_t tiles = std::max<int64_t>(1, (max_len + kTile - 1) / kTile);
  const int64_t pairs = (int64_t)batch * n_kv;
  int64_t s = std::max<int64_t>(1, slots / pairs);
  s = std::min<int64_t>(s, std::max<int64_t>(1, (tiles + kWarps - 1) / kWarps));
  s = std::min<int64_t>(s, kMaxSplits);
  sp.tiles_per_split = (int)((tiles + s - 1) / s);
  sp.n_splits = (int)((tiles + sp.tiles_per_split - 1) / sp.tiles_per_split);
  return sp;
}

static size_t align256(size_t x) { return (x + 255) / 256 * 256; }

// Workspace: split records from the start | ... | pair blocks at fixed
// distances from the end (pair k at end - (k + 1) * kPairBlockBytes, the end
// rounded down to 128 bytes). The split records of a call are bounded by one
// record per CTA slot of the device (or per pair, if there are more pairs)
// and 16 query heads, independently of max_len and G, so the records of any
// call with batch x n_kv <= that of the sizing call end before the pair
// blocks of any such call: one zero-filled workspace serves every sequence of
// calls of those shapes, whatever their max_len or query-head count.
static size_t decode_workspace_layout(size_t pairs, int64_t slots) {
  const size_t recs = (size_t)std::max<int64_t>(slots, (int64_t)pairs);
  const size_t part = align256(recs * 16 * kPartStride * sizeof(float));
  return part + pairs * kPairBlockBytes + 128;
}

// Workspace bytes of a decode call on the current device (an upper bound if
// no device answers).
size_t decode_workspace_bytes_for(int batch, int n_q, int n_kv, int bits_k, int bits_v,
                                  int64_t max_len) {
  cudaError_t err = cudaSuccess;
  const int G = n_q / n_kv;
  const SplitPlan sp = decode_split_plan(batch, n_kv, G, bits_k, bits_v, max_len, &err, true);
  return decode_workspace_layout((size_t)batch * n_kv, sp.slots);
}

template <int BV, int NT, bool WIN>
static cudaError_t launch_decode_t(const DecodeParams& p, int batch, cudaStream_t st) {
  if constexpr (WIN) {  // once per device: the window instantiation's cap, for its largest tile
    static std::atomic<unsigned long long> cap_set{0};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const unsigned long long bit = 1ull << (dev & 63);
    if (!(cap_set.load() & bit)) {
      e = cudaFuncSetAttribute(decode_kernel<BV, NT, true>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)decode_smem_bytes(tile_bytes(8, BV), NT, true));
      if (e != cudaSuccess) return e;
      cap_set.fetch_or(bit);
    }
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.n_splits, p.n_kv, batch);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = decode_smem_bytes(p.tile_bytes, NT, WIN);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, decode_kernel<BV, NT, WIN>, p);
}

template <int NT, bool WIN>
static cudaError_t launch_decode_nt(const DecodeParams& p, int bits_v, int batch, cudaStream_t st) {
  switch (bits_v) {
    case 1: return launch_decode_t<1, NT, WIN>(p, batch, st);
    case 2: return launch_decode_t<2, NT, WIN>(p, batch, st);
    case 3: return launch_decode_t<3, NT, WIN>(p, batch, st);
    case 4: return launch_decode_t<4, NT, WIN>(p, batch, st);
    case 5: return launch_decode_t<5, NT, WIN>(p, batch, st);
    case 6: return launch_decode_t<6, NT, WIN>(p, batch, st);
    case 7: return launch_decode_t<7, NT, WIN>(p, batch, st);
    case 8: return launch_decode_t<8, NT, WIN>(p, batch, st);
  }
  return cudaErrorInvalidValue;
}

// ws: >= decode_workspace_bytes_for(...) bytes, zero-filled before its first
// use; every completed call leaves its pair blocks (at the end of ws) zero.
// n_new > 0 fuses the append of k_new / v_new ([batch][n_new][n_kv][128]).
// Test hook: > 0 makes every later decode launch wait that many cycles on a
// barrier nothing arrives on before its tiles (the wait runs out, the launch
// flags TIMEOUT and skips its tiles).
static std::atomic<long long> g_stall_cycles{0};
void set_decode_stall(long long cycles) { g_stall_cycles.store(cycles > 0 ? cycles : 0); }
// Deterministic mode: the last split merges every split record in split
// order instead of summing exponent buckets filled by L2 atomics in arrival
// order, so outputs repeat bit for bit (slower: one CTA reads all records).
static std::atomic<int> g_deterministic{0};
void set_decode_deterministic(int on) { g_deterministic.store(on ? 1 : 0); }

static cudaError_t launch_decode_any(const Plan* const* plans, const CacheMap& cm, int32_t* len,
                                     int batch, int64_t max_len, const void* q, int q_dtype,
                                     int n_q, int n_kv, int bits_k, int bits_v, float* out,
                                     void* ws, size_t ws_bytes, uint32_t* status, cudaStream_t st,
                                     const void* k_new, const void* v_new, int kv_dtype,
                                     int n_new, int64_t cap, int early, const double* theta,
                                     float* rec_out, float* const* wins, int32_t* wlen, int R) {
  cudaError_t err = cudaSuccess;
  const int G = n_q / n_kv;
  const SplitPlan sp = decode_split_plan(batch, n_kv, G, bits_k, bits_v, max_len, &err, false);
  if (err != cudaSuccess) return err;
  if (decode_workspace_layout((size_t)batch * n_kv, sp.slots) > ws_bytes)
    return cudaErrorInvalidValue;
  if (n_new < 0 || n_new > kMaxNew) return cudaErrorInvalidValue;
  DecodeParams p;
  p.plans = plans;
  p.cm = cm;
  p.len = len;
  p.q = q;
  p.q_dtype = q_dtype;
  p.n_q = n_q;
  p.n_kv = n_kv;
  p.G = G;
  p.max_len = (int)max_len;
  p.n_splits = sp.n_splits;
  p.tiles_per_split = sp.tiles_per_split;
  p.tile_bytes = tile_bytes(bits_k, bits_v);
  p.k_new = k_new;
  p.v_new = v_new;
  p.kv_dtype = kv_dtype;
  p.n_new = n_new;
  p.cap = cap;
  p.early = early;
  p.stall_cycles = g_stall_cycles.load();
  p.deterministic = g_deterministic.load();
  p.rope = theta ? 1 : 0;
  for (int j = 0; j < 64; ++j) p.theta[j] = theta ? theta[j] : 0.0;
  p.part = reinterpret_cast<float*>(ws);
  p.pb_end = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(ws) + ws_bytes) & ~static_cast<uintptr_t>(127));
  p.out = out;
  p.rec_out = rec_out;
  p.status = status;
  p.wins = wins;
  p.wlen = wlen;
  p.R = R;
  if (wins)
    return G <= 8 ? launch_decode_nt<1, true>(p, bits_v, batch, st)
                  : launch_decode_nt<2, true>(p, bits_v, batch, st);
  return G <= 8 ? launch_decode_nt<1, false>(p, bits_v, batch, st)
                : launch_decode_nt<2, false>(p, bits_v, batch, st);
}

cudaError_t launch_decode(const Plan* const* plans, const CacheMap& cm, int32_t* len,
                          int batch, int64_t max_len, const void* q, int q_dtype, int n_q, int n_kv,
                          int bits_k, int bits_v, float* out, void* ws, size_t ws_bytes,
                          uint32_t* status, cudaStream_t st, const void* k_new,
                          const void* v_new, int kv_dtype, int n_new, int64_t cap, int early,
                          const double* theta, float* rec_out) {
  return launch_decode_any(plans, cm, len, batch, max_len, q, q_dtype, n_q, n_kv, bits_k, bits_v,
                           out, ws, ws_bytes, status, st, k_new, v_new, kv_dtype, n_new, cap,
                           early, theta, rec_out, nullptr, nullptr, 0);
}

// The window step in one launch: n_new (1..min(R, 64)) new tokens per
// sequence, the tokens leaving the window quantize-appended from their ring
// slots, the new tokens written to the ring, decode over the packed tokens
// and the window.
cudaError_t launch_decode_window(const Plan* const* plans, const CacheMap& cm, int32_t* len,
                                 int batch, int64_t max_len, const void* q, int q_dtype, int n_q,
                                 int n_kv, int bits_k, int bits_v, float* out, void* ws,
                                 size_t ws_bytes, uint32_t* status, cudaStream_t st,
                                 const void* k_new, const void* v_new, int kv_dtype,
                                 int n_new, int64_t cap, int early, float* const* wins,
                                 int32_t* wlen, int R) {
  if (!wins || !wlen || R < 1 || n_new < 1 || n_new > std::min(R, kMaxNew))
    return cudaErrorInvalidValue;
  return launch_decode_any(plans, cm, len, batch, max_len, q, q_dtype, n_q, n_kv, bits_k, bits_v,
                           out, ws, ws_bytes, status, st, k_new, v_new, kv_dtype, n_new, cap,
                           early, nullptr, nullptr, wins, wlen, R);
}

cudaError_t launch_combine(const Plan* const* plans, const float* recs, int n_parts, int batch,
                           int n_q, int n_kv, float* out, cudaStream_t st) {
  combine_kernel<<<dim3(n_kv, batch), kThreads, 0, st>>>(plans, recs, n_parts, batch, n_q, n_kv,
                                                         out);
  return cudaGetLastError();
}

}  // namespace kvq
