// Device code shared by the quantize-append kernel and the fused
// append + decode kernel: the TQ-MSE codes of a tile's new tokens (keys with
// per-block widths, values with a randomised Hadamard rotation) packed into
// the words of its tile record.
//
// "RoPE-Aware Bit Allocation for KV-Cache Quantization", abstract: keys are
// quantized with Block-GTQ's per-RoPE-block integer widths on top of
// TurboQuant-MSE, values with uniform TQ-MSE. All decisions use IEEE fp32
// in a fixed order with no product contracted into a sum (see kvq.h; an fma
// with a +-1 factor, whose product is exact, stands for an add or subtract),
// so codes are the same bit for bit on every run.
#pragma once

#include "common.cuh"

namespace kvq {

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

// Norm n (fp16 value), reciprocal r and flags of a warp-held 128-vector.
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

// ---------------------------------------------------------------------------
// Tile quantizer in two passes (one CTA per tile record):
//  1. one warp per new token: norms, kz[p][i] = k_i r (NaN for a token whose
//     key codes are all zero), the value rotation and the value codes, which
//     go straight into the packed words;
//  2. one warp per stored key block, lane = position: z = kz * g_j and the
//     codes of coordinates j and j + 64 with the block's width (uniform in
//     the warp), packed as one 2W-bit field.
// Fields enter the words by shared-memory atomics, so any number of warps
// can write one word; with `clear` a field's old bits are cleared first.

constexpr int kKzStride = kHeadDim + 1;  // padded rows: pass 2 reads a column

// Branch-free: the word after the field's first word is always touched (an
// OR of 0 / AND of all ones when the field does not reach it), so `words`
// needs one word of slack past the packed words. nbits <= 16. The first word
// is clamped to wmax, so a plan whose segments lie outside the key words
// (flagged by the plan checks) cannot send a write past word wmax + 1.
__device__ __forceinline__ void put_field(uint32_t* words, int bit, uint32_t val, int nbits,
                                          bool clear, int wmax) {
  const int wi = min(bit >> 5, wmax), off = bit & 31;
  const uint32_t mask = (1u << nbits) - 1u;
  // parts of the field in word wi and wi + 1 (64-bit shift: off may be 0)
  const unsigned long long v2 = (unsigned long long)val << off;
  const unsigned long long m2 = (unsigned long long)mask << off;
  if (clear) {
    atomicAnd(&words[wi], ~(uint32_t)m2);
    atomicAnd(&words[wi + 1], ~(uint32_t)(m2 >> 32));
  }
  atomicOr(&words[wi], (uint32_t)v2);
  atomicOr(&words[wi + 1], (uint32_t)(v2 >> 32));
}

// Number of width-W thresholds strictly below z (NaN -> 0): branch-free
// binary search over the sorted 2^W - 1 thresholds of width W (at
// thr + cb_t_off(W)), all steps unrolled.
template <int W>
__device__ __forceinline__ int code_of_w(const float* thr, float z) {
  const float* t = thr + cb_t_off(W);
  int c = 0;
#pragma unroll
  for (int step = 1 << (W - 1); step; step >>= 1) c += (t[c + step - 1] < z) ? step : 0;
  return c;
}

// RoPE of the key held as kx[q] = k[lane + 32 q] at position pos (theta:
// the 64 block frequencies, shared memory): angle pos theta_j in fp64, cos
// and sin rounded once to fp32, the 2-D rotation of (k_j, k_{j+64}) in fp32
// with every product and sum rounded. Block j = lane + 32 q pairs kx[q] with
// kx[q + 2], both held by this lane.
__device__ __forceinline__ void rope_f32(float (&kx)[4], const double* theta, int64_t pos,
                                         int lane) {
#pragma unroll
  for (int q = 0; q < 2; ++q) {
    double sd, cd;
    sincos((double)pos * theta[lane + 32 * q], &sd, &cd);
    const float c = (float)cd, s = (float)sd;
    const float a = kx[q], b = kx[q + 2];
    kx[q] = __fsub_rn(__fmul_rn(a, c), __fmul_rn(b, s));
    kx[q + 2] = __fadd_rn(__fmul_rn(a, s), __fmul_rn(b, c));
  }
}

// Pass 1 for the token at tile position p (row: element offset of its key /
// value in k / v), value width BV. With theta (not null) the key is pre-RoPE
// and is rotated to position pos first. Writes kz_row[128], the token's value
// fields into `words` and returns the fp16 norms.
template <int BV>
__device__ __forceinline__ void warp_token_pass(const Plan& pl, const float* thr, const void* k,
                                                const void* v, int dtype, size_t row, int lane,
                                                int p, float* kz_row, uint32_t* words, bool clear,
                                                __half& kn, __half& vn, uint32_t& flags,
                                                const double* theta = nullptr, int64_t pos = 0) {
  float kx[4], vx[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    kx[q] = load_as_float(k, dtype, row + lane + 32 * q);
    vx[q] = load_as_float(v, dtype, row + lane + 32 * q);
  }
  if (theta) rope_f32(kx, theta, pos, lane);
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
  // values: y = H (s . v) by the fixed fp32 butterfly graph, z = y r
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
  // butterflies h = 1..16 across lanes: lower y + o, upper o - y, each one
  // fma with a +-1 factor (exact product, one rounding: the same value)
#pragma unroll
  for (int hh = 1; hh < 32; hh <<= 1) {
    const float sg = (lane & hh) ? -1.f : 1.f;
#pragma unroll
    for (int q = 0; q < 4; ++q) y[q] = __fmaf_rn(y[q], sg, __shfl_xor_sync(0xffffffffu, y[q], hh));
  }
  {  // h = 32: (q0, q1), (q2, q3); h = 64: (q0, q2), (q1, q3)
    const float a0 = __fadd_rn(y[0], y[1]), a1 = __fsub_rn(y[0], y[1]);
    const float a2 = __fadd_rn(y[2], y[3]), a3 = __fsub_rn(y[2], y[3]);
    y[0] = __fadd_rn(a0, a2);
    y[2] = __fsub_rn(a0, a2);
    y[1] = __fadd_rn(a1, a3);
    y[3] = __fsub_rn(a1, a3);
  }
  // value fields: coordinate i at bit slot_v(p) BV of its BV-word segment;
  // the bit offset in the word is the same for every lane and q
  uint32_t* vwords = words + kHeadDim * pl.bits_k + ((slot_v(p) * BV) >> 5);
  const int off = (slot_v(p) * BV) & 31;
  const bool spill = off + BV > 32;  // uniform
  constexpr uint32_t mask = (1u << BV) - 1u;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint32_t* w = vwords + BV * (lane + 32 * q);
    const uint32_t c = vlive ? (uint32_t)code_of_w<BV>(thr, __fmul_rn(y[q], vr)) : 0u;
    if (clear) atomicAnd(w, ~(mask << off));
    atomicOr(w, c << off);
    if (spill) {
      if (clear) atomicAnd(w + 1, ~(mask >> (32 - off)));
      atomicOr(w + 1, c >> (32 - off));
    }
  }
}

// ---- key rotation inside width groups (plan.k_rot)
// Plan position P = 2 r + e is coordinate order[r] + 64 e. A width group (the
// ranks of one width) holds 2 n positions, cut into chunks by the binary
// expansion of 2 n, largest first. Tables (shared memory): rank of each block
// (0xFF for width 0); first position and log2 size of each position's chunk.
struct RotTables {
  uint8_t rank_of[64];
  uint8_t base[128];
  uint8_t lg[128];
  int npos;
};

// Built by the threads of a CTA in one parallel step (a barrier must follow):
// thread x < 128 fills position x from the plan's classes (a class is the
// run of ranks of one width), thread x < 64 block x's rank entry.
__device__ __forceinline__ void rot_tables(const Plan& pl, RotTables& t, int x) {
  if (x < 64) {
    if (pl.width[x] == 0) t.rank_of[x] = 0xFF;          // not stored
    if (x < pl.n_ranks) t.rank_of[pl.order[x] & 63] = (uint8_t)x;  // blocks of width > 0
  }
  if (x == 0) t.npos = 2 * pl.n_ranks;
  if (x >= 2 * pl.n_ranks || x >= 128) return;
  const int r = x >> 1;
  int ci = 0;
  while (ci + 1 < pl.n_class && ci + 1 < 8 && pl.hs_rank0[pl.cls_hs0[ci + 1] & 31] <= r) ++ci;
  const int r0 = pl.hs_rank0[pl.cls_hs0[ci] & 31];
  const int m = 2 * (4 * (pl.cls_nhs[ci] - 1) + pl.cls_last[ci]);  // positions of the group
  const int local = x - 2 * r0;
  int off = 0;
  for (int e = 7; e >= 0; --e)
    if (m & (1 << e)) {
      if (local < off + (1 << e)) {
        t.base[x] = (uint8_t)(2 * r0 + off);
        t.lg[x] = (uint8_t)e;
        return;
      }
      off += 1 << e;
    }
}

// Chunk factor c(2^e) = 2^-floor(e/2), times fp32(sqrt(1/2)) for odd e.
__device__ __forceinline__ float rot_scale(int e) {
  const float base = (e & 1) ? 0.70710678118654752f : 1.f;
  return __fmul_rn(base, __int_as_float((127 - (e >> 1)) << 23));
}

// One warp rotates one row in place: in, 128 values in coordinate order (times
// gs[j] when gs is given, one fp32 product); out, positions [0, npos):
// u_P = s_P x, the fp32 butterflies h = 1, 2, ... inside each chunk, then
// y_P = fp32(h_P c(size)).
__device__ __forceinline__ void warp_rotate_row(float* row, const Plan& pl, const RotTables& t,
                                                const float* gs, int lane) {
  float v[4];
  int P[4], sz[4], loc[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int i = lane + 32 * q, j = i & 63, rk = t.rank_of[j];
    P[q] = rk == 0xFF ? -1 : 2 * rk + (i >> 6);
    float x = row[i];
    if (gs) x = __fmul_rn(x, gs[j]);
    if (P[q] >= 0 && ((pl.k_sign[P[q] >> 5] >> (P[q] & 31)) & 1u)) x = -x;
    v[q] = x;
    // this lane's butterfly positions p = lane + 32 q: chunk size and offset
    const int p = lane + 32 * q;
    sz[q] = p < t.npos ? 1 << (t.lg[p] & 7) : 0;
    loc[q] = p < t.npos ? p - t.base[p] : 0;
  }
  __syncwarp();
#pragma unroll
  for (int q = 0; q < 4; ++q)
    if (P[q] >= 0) row[P[q]] = v[q];
  __syncwarp();
#pragma unroll
  for (int q = 0; q < 4; ++q) v[q] = row[lane + 32 * q];  // position order
  // butterflies h < 32 across lanes: the partner of position p is p + h
  // (lower element) or p - h (upper), in this or the neighbouring register
#pragma unroll
  for (int h = 1; h < 32; h <<= 1) {
    float nv[4];
    const int s_lo = (lane + h) & 31, s_up = (lane - h) & 31;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float a0 = __shfl_sync(0xffffffffu, v[q], s_lo);
      const float a1 = __shfl_sync(0xffffffffu, v[q < 3 ? q + 1 : q], s_lo);
      const float b0 = __shfl_sync(0xffffffffu, v[q], s_up);
      const float b1 = __shfl_sync(0xffffffffu, v[q > 0 ? q - 1 : q], s_up);
      const float lo_partner = lane + h < 32 ? a0 : a1;
      const float up_partner = lane >= h ? b0 : b1;
      nv[q] = v[q];
      if (sz[q] > h)
        nv[q] = (loc[q] & h) == 0 ? __fadd_rn(v[q], lo_partner) : __fsub_rn(up_partner, v[q]);
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) v[q] = nv[q];
  }
  // h = 32, 64: the partner is in this lane, register q +- h / 32
#pragma unroll
  for (int k = 1; k <= 2; k <<= 1) {
    const int h = 32 * k;
    float nv[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      nv[q] = v[q];
      if (sz[q] > h) {
        if ((loc[q] & h) == 0) {
          if (q + k < 4) nv[q] = __fadd_rn(v[q], v[q + k]);
        } else {
          if (q - k >= 0) nv[q] = __fsub_rn(v[q - k], v[q]);
        }
      }
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) v[q] = nv[q];
  }
#pragma unroll
  for (int q = 0; q < 4; ++q)
    if (sz[q]) row[lane + 32 * q] = __fmul_rn(v[q], rot_scale(31 - __clz(sz[q])));
  __syncwarp();
}

// Pass 2 for stored block rank r, positions [p_lo, p_hi) (lane = position).
// Without rotation the row holds k r by coordinate (z = (k r) g_j); with it,
// the rotated y by plan position (2 r, 2 r + 1).
template <int W>
__device__ __forceinline__ void block_field(const Plan& pl, const float* thr, int r, int j,
                                            const float* row, int lane, uint32_t* words,
                                            bool clear, bool rot) {
  const float g = pl.g[j & 63];
  const float z0 = rot ? row[2 * r] : __fmul_rn(row[j & 63], g);
  const float z1 = rot ? row[2 * r + 1] : __fmul_rn(row[(j & 63) + 64], g);
  const uint32_t c0 = (uint32_t)code_of_w<W>(thr, z0);
  const uint32_t c1 = (uint32_t)code_of_w<W>(thr, z1);
  put_field(words, 32 * pl.seg_off[r] + slot_k(lane) * 2 * W, c0 | (c1 << W), 2 * W, clear,
            128 * pl.bits_k - 1);
}

__device__ __forceinline__ void warp_block_pass(const Plan& pl, const float* thr, int r,
                                                const float* kz, int p_lo, int p_hi, int lane,
                                                uint32_t* words, bool clear) {
  const int j = pl.order[r], w = pl.width[j];
  const bool rot = pl.k_rot != 0;
  if (lane < p_lo || lane >= p_hi) return;
  const float* row = kz + lane * kKzStride;
  switch (w) {  // uniform in the warp
    case 1: block_field<1>(pl, thr, r, j, row, lane, words, clear, rot); break;
    case 2: block_field<2>(pl, thr, r, j, row, lane, words, clear, rot); break;
    case 3: block_field<3>(pl, thr, r, j, row, lane, words, clear, rot); break;
    case 4: block_field<4>(pl, thr, r, j, row, lane, words, clear, rot); break;
    case 5: block_field<5>(pl, thr, r, j, row, lane, words, clear, rot); break;
    case 6: block_field<6>(pl, thr, r, j, row, lane, words, clear, rot); break;
    case 7: block_field<7>(pl, thr, r, j, row, lane, words, clear, rot); break;
    default: block_field<8>(pl, thr, r, j, row, lane, words, clear, rot); break;
  }
}

}  // namespace kvq
