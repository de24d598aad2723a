// Exact merge of KV-chunk partials (sm_100a, bandwidth-bound).
//
// For every (row s, head h) with chunk partials (o_p, lse_p), p < P:
//   L   = max_p lse_p
//   lse = L + ln(sum_p exp(lse_p - L))
//   o   = sum_p exp(lse_p - lse) * o_p
// This is the combine step of ring attention's online softmax (TensorRT 11.0
// multi-device article, Ring Attention) and the split-reduction the accuracy
// table of "TensorRT Multi-Device (multi-GPU) support" (Validation) refers
// to.  Chunks with lse_p = -inf (no keys) get weight 0.
//
// One block owns 256 consecutive (s, h) pairs.  Phase 1: thread t computes
// the P weights of pair t into shared memory and writes lse.  Phase 2: the
// block streams the pairs' o_p rows, which are contiguous in the
// [P][S][H][D] layout, as float4 loads (8 chunks in flight per thread),
// accumulates in fp32 and stores fp16.
#pragma once

#include <cmath>

#include "ptx.cuh"

namespace b2a {

constexpr int kMergePairs = 256;     // (s, h) pairs per block = threads per block
constexpr int kMergeMaxP = 64;       // shared weights: P x 256 floats

template <int D>
__global__ void __launch_bounds__(kMergePairs)
    attn_merge_kernel(const float* __restrict__ o_parts, const float* __restrict__ lse_parts, int P,
                      int S, int H, uint16_t* __restrict__ out, float* __restrict__ lse_out) {
  extern __shared__ float w_s[];  // [P][kMergePairs]
  const long long npairs = static_cast<long long>(S) * H;
  const long long pair0 = static_cast<long long>(blockIdx.x) * kMergePairs;
  const int t = threadIdx.x;

  {
    const long long pr = pair0 + t;
    if (pr < npairs) {
      const int s = static_cast<int>(pr / H);
      const int h = static_cast<int>(pr - static_cast<long long>(s) * H);
      const size_t plane = static_cast<size_t>(H) * S;
      const float* lp = lse_parts + static_cast<size_t>(h) * S + s;
      float L = -INFINITY;
      for (int q = 0; q < P; ++q) L = fmaxf(L, __ldg(lp + q * plane));
      float lse;
      if (L == -INFINITY) {
        lse = -INFINITY;
        for (int q = 0; q < P; ++q) w_s[q * kMergePairs + t] = 0.f;
      } else {
        float tot = 0.f;
        for (int q = 0; q < P; ++q) tot += expf(__ldg(lp + q * plane) - L);
        lse = L + logf(tot);
        for (int q = 0; q < P; ++q) {
          const float lq = __ldg(lp + q * plane);
          w_s[q * kMergePairs + t] = (lq == -INFINITY) ? 0.f : expf(lq - lse);
        }
      }
      if (lse_out) lse_out[static_cast<size_t>(h) * S + s] = lse;
    }
  }
  __syncthreads();

  constexpr int U = D / 4;  // float4 units per pair
  const long long pairs_here = (npairs - pair0 < kMergePairs) ? (npairs - pair0) : kMergePairs;
  const int units = static_cast<int>(pairs_here) * U;
  const float4* src = reinterpret_cast<const float4*>(o_parts) + pair0 * U;
  const size_t plane4 = static_cast<size_t>(npairs) * U;  // float4 per chunk
  uint2* dst = reinterpret_cast<uint2*>(out) + pair0 * U;

  for (int u = t; u < units; u += kMergePairs) {
    const int pi = u / U;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int q0 = 0; q0 < P; q0 += 8) {
      float4 x[8];
#pragma unroll
      for (int i = 0; i < 8; ++i)
        if (q0 + i < P) x[i] = __ldcs(src + (q0 + i) * plane4 + u);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        if (q0 + i < P) {
          const float w = w_s[(q0 + i) * kMergePairs + pi];
          acc.x = fmaf(w, x[i].x, acc.x);
          acc.y = fmaf(w, x[i].y, acc.y);
          acc.z = fmaf(w, x[i].z, acc.z);
          acc.w = fmaf(w, x[i].w, acc.w);
        }
      }
    }
    dst[u] = make_uint2(pack_half2(acc.x, acc.y), pack_half2(acc.z, acc.w));
  }
}

}  // namespace b2a
