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
// [P][S][H][D] layout, as 16-byte loads (4 fp32 or 8 fp16 partial values;
// 8 chunks in flight per thread), accumulates in fp32 and stores fp16.  The
// fp16 form reads the partials the FP16 split-reduction stores: half the
// bytes of the dominant term.
#pragma once

#include <cmath>

#include "ptx.cuh"

#include <cuda_fp16.h>

namespace b2a {

constexpr int kMergePairs = 256;     // (s, h) pairs per block = threads per block
constexpr int kMergeMaxP = 64;       // shared weights: P x 256 floats

// Widens one 16-byte unit of partial values to fp32.
template <typename T>
__device__ __forceinline__ void unpack_unit(const uint4& x, float (&v)[16 / sizeof(T)]) {
  if constexpr (sizeof(T) == 4) {
    v[0] = __uint_as_float(x.x);
    v[1] = __uint_as_float(x.y);
    v[2] = __uint_as_float(x.z);
    v[3] = __uint_as_float(x.w);
  } else {
    const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      __half2 h;
      memcpy(&h, &w[i], 4);
      const float2 f = __half22float2(h);
      v[2 * i] = f.x;
      v[2 * i + 1] = f.y;
    }
  }
}

// Phase 2 of a group of kMergePairs (s, h) pairs starting at pair0: the
// weighted sum of the pairs' chunk partials with the weights w_s[q * wstride
// + pair - pair0], stored as fp16.
template <int D, typename T>
__device__ __forceinline__ void merge_stream_group(const T* __restrict__ o_parts, int P, long long npairs,
                                                   long long pair0, const float* w_s, int wstride,
                                                   uint16_t* __restrict__ out) {
  const int t = threadIdx.x;
  constexpr int E = 16 / static_cast<int>(sizeof(T));  // partial values per 16-byte unit
  constexpr int U = D / E;                              // units per pair
  const long long pairs_here = (npairs - pair0 < kMergePairs) ? (npairs - pair0) : kMergePairs;
  const int units = static_cast<int>(pairs_here) * U;
  const uint4* src = reinterpret_cast<const uint4*>(o_parts) + pair0 * U;
  const size_t plane16 = static_cast<size_t>(npairs) * U;  // units per chunk
  uint16_t* dst = out + pair0 * D;

  // Two units per thread per pass, all their chunk loads issued before use,
  // so each thread keeps up to 16 independent 16-byte loads in flight.
  for (int u0 = t; u0 < units; u0 += 2 * kMergePairs) {
    const int u1 = u0 + kMergePairs;
    const bool has1 = u1 < units;
    const int pi0 = u0 / U;
    const int pi1 = has1 ? u1 / U : pi0;
    float acc0[E], acc1[E];
#pragma unroll
    for (int e = 0; e < E; ++e) acc0[e] = acc1[e] = 0.f;
    for (int q0 = 0; q0 < P; q0 += 8) {
      uint4 x0[8], x1[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        if (q0 + i < P) {
          x0[i] = __ldcs(src + (q0 + i) * plane16 + u0);
          if (has1) x1[i] = __ldcs(src + (q0 + i) * plane16 + u1);
        }
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        if (q0 + i < P) {
          float v[E];
          const float w0 = w_s[(q0 + i) * wstride + pi0];
          unpack_unit<T>(x0[i], v);
#pragma unroll
          for (int e = 0; e < E; ++e) acc0[e] = fmaf(w0, v[e], acc0[e]);
          if (has1) {
            const float w1 = w_s[(q0 + i) * wstride + pi1];
            unpack_unit<T>(x1[i], v);
#pragma unroll
            for (int e = 0; e < E; ++e) acc1[e] = fmaf(w1, v[e], acc1[e]);
          }
        }
      }
    }
    if constexpr (E == 4) {
      reinterpret_cast<uint2*>(dst)[u0] = make_uint2(pack_half2(acc0[0], acc0[1]), pack_half2(acc0[2], acc0[3]));
      if (has1)
        reinterpret_cast<uint2*>(dst)[u1] = make_uint2(pack_half2(acc1[0], acc1[1]), pack_half2(acc1[2], acc1[3]));
    } else {
      reinterpret_cast<uint4*>(dst)[u0] = make_uint4(pack_half2(acc0[0], acc0[1]), pack_half2(acc0[2], acc0[3]),
                                                     pack_half2(acc0[4], acc0[5]), pack_half2(acc0[6], acc0[7]));
      if (has1)
        reinterpret_cast<uint4*>(dst)[u1] = make_uint4(pack_half2(acc1[0], acc1[1]), pack_half2(acc1[2], acc1[3]),
                                                       pack_half2(acc1[4], acc1[5]), pack_half2(acc1[6], acc1[7]));
    }
  }
}

// T: float (fp32 partials) or uint16_t (fp16 partials).
template <int D, typename T>
__global__ void __launch_bounds__(kMergePairs)
    attn_merge_kernel(const T* __restrict__ o_parts, const float* __restrict__ lse_parts, int P,
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

  merge_stream_group<D, T>(o_parts, P, npairs, pair0, w_s, kMergePairs, out);
}

// Pair-group weights of the pipelined merge: thread t's pair (pair0 + t)
// from its P lse values ``lv``; writes the weights into w_s[q * kMergePairs
// + t] and the merged lse.
template <int PMAX>
__device__ __forceinline__ void merge_weights(const float (&lv)[PMAX], int P, long long npairs, long long pair0,
                                              int S, int H, float* w_s, float* __restrict__ lse_out) {
  const int t = threadIdx.x;
  const long long pr = pair0 + t;
  if (pr >= npairs) return;
  float L = -INFINITY;
#pragma unroll
  for (int q = 0; q < PMAX; ++q)
    if (q < P) L = fmaxf(L, lv[q]);
  float lse;
  if (L == -INFINITY) {
    lse = -INFINITY;
#pragma unroll
    for (int q = 0; q < PMAX; ++q)
      if (q < P) w_s[q * kMergePairs + t] = 0.f;
  } else {
    float tot = 0.f;
#pragma unroll
    for (int q = 0; q < PMAX; ++q)
      if (q < P) tot += expf(lv[q] - L);
    lse = L + logf(tot);
#pragma unroll
    for (int q = 0; q < PMAX; ++q)
      if (q < P) w_s[q * kMergePairs + t] = (lv[q] == -INFINITY) ? 0.f : expf(lv[q] - lse);
  }
  if (lse_out) {
    const int s = static_cast<int>(pr / H);
    const int h = static_cast<int>(pr - static_cast<long long>(s) * H);
    lse_out[static_cast<size_t>(h) * S + s] = lse;
  }
}

// Pipelined form for P <= kMergePipeMaxP, same arithmetic as
// attn_merge_kernel: a persistent grid whose blocks walk groups of
// kMergePairs pairs.  The lse loads of a block's next group are issued before
// the current group streams and its weights are computed after, into the
// other half of a double buffer, so the weight phase (P dependent loads and
// exponentials per pair) hides behind the streaming instead of stalling it.
constexpr int kMergePipeMaxP = 16;

template <int D, typename T>
__global__ void __launch_bounds__(kMergePairs, 2)
    attn_merge_pipe_kernel(const T* __restrict__ o_parts, const float* __restrict__ lse_parts, int P, int S,
                           int H, uint16_t* __restrict__ out, float* __restrict__ lse_out) {
  __shared__ float w_s[2][kMergePipeMaxP * kMergePairs];
  const long long npairs = static_cast<long long>(S) * H;
  const long long ngroups = (npairs + kMergePairs - 1) / kMergePairs;
  const size_t plane = static_cast<size_t>(H) * S;
  const int t = threadIdx.x;
  float lv[kMergePipeMaxP];
  auto load_lse = [&](long long g) {
    const long long pr = g * kMergePairs + t;
    if (g < ngroups && pr < npairs) {
      const int s = static_cast<int>(pr / H);
      const int h = static_cast<int>(pr - static_cast<long long>(s) * H);
      const float* lp = lse_parts + static_cast<size_t>(h) * S + s;
#pragma unroll
      for (int q = 0; q < kMergePipeMaxP; ++q)
        if (q < P) lv[q] = __ldg(lp + q * plane);
    }
  };
  long long g = blockIdx.x;
  load_lse(g);
  merge_weights(lv, P, npairs, g * kMergePairs, S, H, w_s[0], lse_out);
  int buf = 0;
  for (; g < ngroups; g += gridDim.x) {
    const long long gn = g + gridDim.x;
    load_lse(gn);  // in flight while this group streams
    __syncthreads();  // w_s[buf] complete; every thread is done with w_s[buf ^ 1]
    merge_stream_group<D, T>(o_parts, P, npairs, g * kMergePairs, w_s[buf], kMergePairs, out);
    if (gn < ngroups) merge_weights(lv, P, npairs, gn * kMergePairs, S, H, w_s[buf ^ 1], lse_out);
    buf ^= 1;
  }
}

}  // namespace b2a
