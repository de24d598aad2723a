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

  // Two units per thread per pass, all their chunk loads issued before use,
  // so each thread keeps up to 16 independent 16-byte loads in flight.
  for (int u0 = t; u0 < units; u0 += 2 * kMergePairs) {
    const int u1 = u0 + kMergePairs;
    const bool has1 = u1 < units;
    const int pi0 = u0 / U;
    const int pi1 = has1 ? u1 / U : pi0;
    float4 acc0 = make_float4(0.f, 0.f, 0.f, 0.f);
    float4 acc1 = acc0;
    for (int q0 = 0; q0 < P; q0 += 8) {
      float4 x0[8], x1[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        if (q0 + i < P) {
          x0[i] = __ldcs(src + (q0 + i) * plane4 + u0);
          if (has1) x1[i] = __ldcs(src + (q0 + i) * plane4 + u1);
        }
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        if (q0 + i < P) {
          const float w0 = w_s[(q0 + i) * kMergePairs + pi0];
          acc0.x = fmaf(w0, x0[i].x, acc0.x);
          acc0.y = fmaf(w0, x0[i].y, acc0.y);
          acc0.z = fmaf(w0, x0[i].z, acc0.z);
          acc0.w = fmaf(w0, x0[i].w, acc0.w);
          if (has1) {
            const float w1 = w_s[(q0 + i) * kMergePairs + pi1];
            acc1.x = fmaf(w1, x1[i].x, acc1.x);
            acc1.y = fmaf(w1, x1[i].y, acc1.y);
            acc1.z = fmaf(w1, x1[i].z, acc1.z);
            acc1.w = fmaf(w1, x1[i].w, acc1.w);
          }
        }
      }
    }
    dst[u0] = make_uint2(pack_half2(acc0.x, acc0.y), pack_half2(acc0.z, acc0.w));
    if (has1) dst[u1] = make_uint2(pack_half2(acc1.x, acc1.y), pack_half2(acc1.z, acc1.w));
  }
}

}  // namespace b2a
