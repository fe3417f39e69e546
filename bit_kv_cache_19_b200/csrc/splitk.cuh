// Split-K decode plumbing shared by the packed-cache decode kernel and the
// bf16 comparator: split records, their merge, arrival counters, and the
// programmatic-dependent-launch and L2-prefetch primitives.
//
// A split's partial result per query head is a record of 132 fp32 (m, l, 2
// unused, o[128], o 16-byte aligned): base-2 running max m, sum l of
// 2^(s - m), and o = sum 2^(s - m) v. Records merge exactly like the
// online-softmax update (flash-decoding's split-K combine).
#pragma once

#include "common.cuh"

namespace kvq {

constexpr int kPartStride = 132;  // split record: m, l, 2 unused, o[128]
constexpr int kRecO = 4;          // o at float 4 (16-byte aligned)
constexpr int kGroup = 16;        // splits merged per first-level group
constexpr int kMergeChunk = 16;   // records whose loads a merge issues together
constexpr int kMaxSplits = 1024;
constexpr int kCntStride = 2 + kMaxSplits / kGroup;  // merge-tree counters per (sequence, KV head)

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ void grid_dep_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}
// Arrival on a counter that wraps to zero after n arrivals, by one thread of
// a CTA after a CTA barrier; true for the last arriver. The atomic is
// acquire-release at GPU scope: the CTA's earlier writes (ordered before it
// by the barrier) are visible to the last arriver, whose CTA reads after a
// barrier that follows see the writes of every arriver.
__device__ __forceinline__ bool arrive_last(unsigned int* c, unsigned int n) {
  unsigned int old;
  asm volatile("atom.acq_rel.gpu.global.inc.u32 %0, [%1], %2;"
               : "=r"(old)
               : "l"(c), "r"(n - 1u)
               : "memory");
  return old == n - 1u;
}

// L2 prefetch (a hint: no value is read, so it may precede the wait for the
// kernel that writes the line).
__device__ __forceinline__ void prefetch_l2(const void* p) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}
__device__ __forceinline__ void grid_dep_launch() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}


// Merge of n records of one head at coordinates x4..x4+3 (record s at
// r + s * rec_stride): one pass with online rescaling over chunks of CHUNK
// records whose loads are issued together (about n / CHUNK load round trips).
// Every thread of the head gets the same M and L.
template <int CHUNK>
__device__ __forceinline__ void merge_item(const float* r, int n, size_t rec_stride, int x4,
                                           float& M, float& L, float4& O) {
  M = -INFINITY;
  L = 0.f;
  O = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int s0 = 0; s0 < n; s0 += CHUNK) {
    float2 ml[CHUNK];
    float4 oo[CHUNK];
#pragma unroll
    for (int k = 0; k < CHUNK; ++k) {
      const bool v = s0 + k < n;
      const float* q = r + (size_t)(v ? s0 + k : 0) * rec_stride;
      ml[k] = *reinterpret_cast<const float2*>(q);
      oo[k] = *reinterpret_cast<const float4*>(q + kRecO + x4);
      if (!v) ml[k].x = -INFINITY;
    }
    float cm = M;
#pragma unroll
    for (int k = 0; k < CHUNK; ++k) cm = fmaxf(cm, ml[k].x);
    if (cm != -INFINITY) {
      const float a = ex2(M - cm);
      L *= a;
      O.x *= a;
      O.y *= a;
      O.z *= a;
      O.w *= a;
#pragma unroll
      for (int k = 0; k < CHUNK; ++k) {
        const float w = ex2(ml[k].x - cm);  // 0 for records past n
        L += w * ml[k].y;
        O.x += w * oo[k].x;
        O.y += w * oo[k].y;
        O.z += w * oo[k].z;
        O.w += w * oo[k].w;
      }
      M = cm;
    }
  }
}

// Merge n records per head (record s of head h at src + s * rec_stride +
// h * kPartStride) into dst (record h at dst + h * kPartStride), for G heads,
// 32 threads per head, 4 coordinates each.
template <int NTHREADS, int CHUNK = kMergeChunk>
__device__ __forceinline__ void merge_records(const float* src, int n, size_t rec_stride, int G,
                                              float* dst) {
  for (int item = threadIdx.x; item < G * 32; item += NTHREADS) {
    const int head = item >> 5, x4 = (item & 31) * 4;
    float M, L;
    float4 O;
    merge_item<CHUNK>(src + (size_t)head * kPartStride, n, rec_stride, x4, M, L, O);
    float* d = dst + (size_t)head * kPartStride;
    *reinterpret_cast<float4*>(d + kRecO + x4) = O;
    if (x4 == 0) {
      d[0] = M;
      d[1] = L;
    }
  }
}

}  // namespace kvq
