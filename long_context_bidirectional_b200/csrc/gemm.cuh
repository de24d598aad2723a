// Projection GEMM for sm_100a: C[M,N] = A[M,K] * W[N,K]^T (+ R[M,N]).
//
// The fused QKV projection and the output projection of the self-attention
// block ("Tensor Parallelism: Sharding Weights for Parallel Layer
// Execution", section 3: Q = X W_Q, K = X W_K, V = X W_V and
// Z = Concat(heads) W_O; "Multi-Device Attention Inference with TensorRT",
// Generating the ONNX Models: Q/K/V and output projections), with weights in
// the [out, in] layout.  fp16 operands, fp32 accumulation in TMEM, one fp16
// rounding of (acc + residual) in the epilogue.  A second instantiation
// applies a per-head RMSNorm to the q and k columns of the fused QKV output
// in the epilogue (the sample block lists Q/K/V projections, then RMSNorm,
// then attention: "Multi-Device Attention Inference with TensorRT",
// Generating the ONNX Models).
//
// Persistent kernel on CTA pairs: a cluster of two CTAs (two SMs) owns a
// 256x256 output tile, 128 rows per CTA.  Every MMA is one M = 256
// tcgen05.mma.cta_group::2 issued by the leader CTA: each CTA supplies its
// 128 rows of A and half (128 rows) of W from its own shared memory and
// keeps its 128 rows of the result in its own TMEM.  Per 64 columns of K
// each SM loads 32 KB (A 16 KB + W half 16 KB) for 4 MMAs of 128 cycles,
// instead of 48 KB for a 128x256 tile on one SM: the tensor core reads 64
// instead of 96 bytes of shared memory per clock and W's L2 traffic halves.
// K in steps of 128 through a 3-stage TMA ring (two 128-byte-swizzled
// blocks of 64 columns per operand and stage); the loads
// of both CTAs complete on the leader's barriers.  Warp roles per CTA:
//   warp 0     TMA producer (its CTA's A rows and W half)
//   warp 1     TMEM allocator and (leader only) single-thread MMA issuer
//   warps 2-5  epilogue of the CTA's 128 rows (TMEM -> registers ->
//              +residual or q/k RMSNorm -> fp16 -> global)
// The accumulator is double-buffered in TMEM (2 x 256 columns) so the
// epilogue of tile i overlaps the main loop of tile i+1; each epilogue warp
// releases a buffer with one relaxed arrival on the leader's barrier after
// its TMEM loads have completed.
#pragma once

#include "ptx.cuh"

namespace b2a {

struct GemmParams {
  int M, N, K;
  int tiles_m, tiles_n, num_tiles;  // tiles of 256 x 256 (one per CTA pair)
  uint16_t* c;          // [M, N] fp16
  const uint16_t* r;    // [M, N] fp16 residual (nullable, may alias c)
  unsigned int* status;
  // q/k RMSNorm epilogue (gemm_tn_kernel<true>): columns [0, hsec) are q and
  // [hsec, 2*hsec) are k, in heads of dh columns; each head segment of a row
  // is scaled by rsqrt(mean of its squares + eps) and by g_q / g_k [dh].
  const uint16_t* g_q;
  const uint16_t* g_k;
  int hsec, dh;
  float eps;
};

struct GemmShape {
  static constexpr int BM = 128, BN = 256, BK = 128;  // per CTA: 128 rows; per pair: 256 x 256
  static constexpr int PAIR_M = 2 * BM;
  static constexpr int STAGES = 3;
  static constexpr int KSUB = 64;                    // K columns per 128-byte swizzled block
  static constexpr int A_SUB = BM * KSUB * 2;        // 16 KB: [128 rows x 128 B]
  static constexpr int B_SUB = (BN / 2) * KSUB * 2;  // 16 KB
  static constexpr int A_BYTES = BM * BK * 2;        // 32 KB
  static constexpr int B_BYTES = (BN / 2) * BK * 2;  // 32 KB: this CTA's half of the W tile
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int OFF_BAR = STAGES * STAGE_BYTES;
  // barriers: full[STAGES] (leader), empty[STAGES], acc_full[2],
  //           acc_empty[2] (leader), drain
  static constexpr int B_FULL = 0;
  static constexpr int B_EMPTY = STAGES;
  static constexpr int B_ACCF = 2 * STAGES;
  static constexpr int B_ACCE = 2 * STAGES + 2;
  static constexpr int B_DRAIN = 2 * STAGES + 4;
  static constexpr int NBAR = B_DRAIN + 1;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;
  static constexpr int TM_COLS = 512;
  static constexpr int THREADS = 192;
  static constexpr int ACCE_ARRIVALS = 8;            // 4 epilogue warps x 2 CTAs
  static constexpr int GROUP_M = 8;    // raster: 8 pair m-blocks share each n sweep
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory per CTA");
  static_assert(A_SUB == B_SUB, "one K offset for both operands");
};

__device__ __forceinline__ void gemm_tile_coords(const GemmParams& p, int tile, int& mb, int& nb) {
  constexpr int G = GemmShape::GROUP_M;
  const int per_group = G * p.tiles_n;
  const int g = tile / per_group;
  const int first_m = g * G;
  const int gsize = min(G, p.tiles_m - first_m);
  const int in = tile - g * per_group;
  mb = first_m + in % gsize;
  nb = in / gsize;
}

// Epilogue of one output row of a tile: its 256 accumulator columns from
// TMEM (``t_base``: this thread's lane, the buffer's first column), plus the
// residual or the q/k RMSNorm, rounded once to fp16.  Every lane runs the
// TMEM loads (warp-collective); only live rows store.
template <bool NORM>
__device__ __forceinline__ void gemm_epilogue_row(const GemmParams& p, int row, bool live, int nb,
                                                  uint32_t t_base) {
  using C = GemmShape;
  if constexpr (NORM) {
    // Head segments of dh columns: q and k heads are normalised from the
    // fp32 accumulator (read twice from TMEM: sum of squares, then scale),
    // v heads are stored as they are.  Segments never straddle q|k|v.
    for (int s0 = 0; s0 < C::BN; s0 += p.dh) {
      const int cseg = nb * C::BN + s0;
      if (cseg >= p.N) break;
      const int sec = cseg / p.hsec;
      float mul = 1.f;
      if (sec < 2) {
        float ss = 0.f;
        for (int cb = 0; cb < p.dh; cb += 32) {
          uint32_t v[32];
          tmem_ld32(t_base + s0 + cb, v);
          tmem_wait_ld(v);
#pragma unroll
          for (int c = 0; c < 32; ++c) ss = fmaf(__uint_as_float(v[c]), __uint_as_float(v[c]), ss);
        }
        mul = rsqrtf(ss / static_cast<float>(p.dh) + p.eps);
      }
      const uint16_t* g = sec == 0 ? p.g_q : p.g_k;
      for (int cb = 0; cb < p.dh; cb += 32) {
        uint32_t v[32];
        tmem_ld32(t_base + s0 + cb, v);
        tmem_wait_ld(v);
        if (!live) continue;
        float y[32];
#pragma unroll
        for (int c = 0; c < 32; ++c) y[c] = __uint_as_float(v[c]);
        if (sec < 2) {
          const uint4* gv = reinterpret_cast<const uint4*>(g + cb);
#pragma unroll
          for (int q8 = 0; q8 < 4; ++q8) {
            const uint4 gw = gv[q8];
            const __half2* gh = reinterpret_cast<const __half2*>(&gw);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float2 gf = __half22float2(gh[e]);
              y[q8 * 8 + 2 * e] *= mul * gf.x;
              y[q8 * 8 + 2 * e + 1] *= mul * gf.y;
            }
          }
        }
        uint4* dst = reinterpret_cast<uint4*>(p.c + static_cast<size_t>(row) * p.N + cseg + cb);
#pragma unroll
        for (int q8 = 0; q8 < 4; ++q8)
          dst[q8] = make_uint4(pack_half2(y[q8 * 8], y[q8 * 8 + 1]), pack_half2(y[q8 * 8 + 2], y[q8 * 8 + 3]),
                               pack_half2(y[q8 * 8 + 4], y[q8 * 8 + 5]),
                               pack_half2(y[q8 * 8 + 6], y[q8 * 8 + 7]));
      }
    }
  } else {
#pragma unroll 1
    for (int cb = 0; cb < C::BN; cb += 32) {
      uint32_t v[32];
      tmem_ld32(t_base + cb, v);
      tmem_wait_ld(v);
      const int col0 = nb * C::BN + cb;
      if (live) {
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          const int col = col0 + g * 8;
          if (col < p.N) {
            const size_t off = static_cast<size_t>(row) * p.N + col;
            float add[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
            if (p.r) {
              const uint4 rv = *reinterpret_cast<const uint4*>(p.r + off);
              const __half2* rh = reinterpret_cast<const __half2*>(&rv);
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const float2 f = __half22float2(rh[e]);
                add[2 * e] = f.x;
                add[2 * e + 1] = f.y;
              }
            }
            uint4 o;
            o.x = pack_half2(__uint_as_float(v[g * 8 + 0]) + add[0], __uint_as_float(v[g * 8 + 1]) + add[1]);
            o.y = pack_half2(__uint_as_float(v[g * 8 + 2]) + add[2], __uint_as_float(v[g * 8 + 3]) + add[3]);
            o.z = pack_half2(__uint_as_float(v[g * 8 + 4]) + add[4], __uint_as_float(v[g * 8 + 5]) + add[5]);
            o.w = pack_half2(__uint_as_float(v[g * 8 + 6]) + add[6], __uint_as_float(v[g * 8 + 7]) + add[7]);
            *reinterpret_cast<uint4*>(p.c + off) = o;
          }
        }
      }
    }
  }
}

template <bool NORM>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(192, 1)
    gemm_tn_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                   const GemmParams p) {
  using C = GemmShape;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_u32 = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_u32 & 1023u)) & 1023u);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int cluster = static_cast<int>(blockIdx.x >> 1);
  const int nclusters = static_cast<int>(gridDim.x >> 1);
  const uint32_t sBase = smem_u32(smem);
  const uint32_t sBar = smem_u32(smem + C::OFF_BAR);
  auto bar = [&](int i) -> uint32_t { return sBar + 8u * static_cast<uint32_t>(i); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);
  // [rank]: K steps each CTA's producer issued (meaningful in the leader)
  volatile uint32_t* issued_by = reinterpret_cast<volatile uint32_t*>(smem + C::OFF_MISC + 8);
  const int nk = (p.K + C::BK - 1) / C::BK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(bar(C::B_FULL + s), 1);
      mbar_init(bar(C::B_EMPTY + s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar(C::B_ACCF + b), 1);
      mbar_init(bar(C::B_ACCE + b), C::ACCE_ARRIVALS);
    }
    mbar_init(bar(C::B_DRAIN), 1);
    // A CTA launched after an earlier one timed out gives up at its first
    // wait that does not complete at once.
    *abort_flag = (*reinterpret_cast<volatile unsigned int*>(p.status) != 0u) ? 1 : 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(tmem_slot), C::TM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  // both CTAs' barriers initialised and TMEM allocated before any cross-CTA use
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ---------------------------------------------------------- TMA producer --
    if (lane == 0) {
      prefetch_tmap(&tm_a);
      prefetch_tmap(&tm_b);
      // ends of the K columns and of the A / W rows the tiles cover
      // (debug-build bounds)
      const int k_end = nk * C::BK;
      const int m_end = p.tiles_m * C::PAIR_M, n_end = p.tiles_n * C::BN;
      int it = 0;
      bool ok = true;
      for (int tile = cluster; tile < p.num_tiles && ok; tile += nclusters) {
        int mb, nb;
        gemm_tile_coords(p, tile, mb, nb);
        const int arow = mb * C::PAIR_M + static_cast<int>(rank) * C::BM;
        const int brow = nb * C::BN + static_cast<int>(rank) * (C::BN / 2);
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const int st = it % C::STAGES;
          if (!mbar_wait(bar(C::B_EMPTY + st), ((it / C::STAGES) & 1) ^ 1, abort_flag, p.status)) {
            ok = false;
            break;
          }
          // the leader posts both CTAs' bytes on its own full barrier
          if (leader) mbar_arrive_expect_tx(bar(C::B_FULL + st), 2 * C::STAGE_BYTES);
          const uint32_t lf = map_to_rank(bar(C::B_FULL + st), 0);
          const uint32_t sa = sBase + st * C::STAGE_BYTES;
#pragma unroll
          for (int sb = 0; sb < C::BK / C::KSUB; ++sb) {
            tma_load_2d_pair_chk(sa + sb * C::A_SUB, C::A_SUB, raw_u32, &tm_a, lf, kb * C::BK + sb * C::KSUB, arow,
                                 k_end, m_end);
            tma_load_2d_pair_chk(sa + C::A_BYTES + sb * C::B_SUB, C::B_SUB, raw_u32, &tm_b, lf,
                                 kb * C::BK + sb * C::KSUB, brow, k_end, n_end);
          }
        }
      }
      st_cluster_u32(map_to_rank(smem_u32(const_cast<uint32_t*>(issued_by + rank)), 0),
                     static_cast<uint32_t>(it));
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------- MMA issuer (leader) --
    if (leader && lane == 0) {
      constexpr uint32_t idesc = idesc_f16_f32(C::PAIR_M, C::BN, false, false);
      int it = 0, lt = 0;
      bool ok = true;
      for (int tile = cluster; tile < p.num_tiles && ok; tile += nclusters, ++lt) {
        const int buf = lt & 1;
        // both CTAs' epilogues have read this accumulator buffer
        if (!(ok = mbar_wait(bar(C::B_ACCE + buf), ((lt >> 1) & 1) ^ 1, abort_flag, p.status))) break;
        tc_fence_after();
        const uint32_t d_t = tmem + buf * C::BN;
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const int st = it % C::STAGES;
          if (!(ok = mbar_wait(bar(C::B_FULL + st), (it / C::STAGES) & 1, abort_flag, p.status))) break;
          tc_fence_after();
          const uint32_t sa = sBase + st * C::STAGE_BYTES;
#pragma unroll
          for (int kk = 0; kk < C::BK / 16; ++kk) {
            const uint32_t ko = (kk >> 2) * C::A_SUB + (kk & 3) * 32;   // A_SUB == B_SUB
            mma_ss_pair(d_t, sw128_desc(sa + ko, 16, 1024), sw128_desc(sa + C::A_BYTES + ko, 16, 1024), idesc,
                        (kb > 0 || kk > 0) ? 1u : 0u);
          }
          tc_commit_pair(bar(C::B_EMPTY + st));
        }
        if (!ok) break;
        tc_commit_pair(bar(C::B_ACCF + buf));
      }
      // every MMA issued above must finish before TMEM is released
      tc_commit_pair(bar(C::B_DRAIN));
      mbar_drain(bar(C::B_DRAIN), 0);
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------- epilogue --
    // Warps 2..5 cover TMEM lane quarters 2,3,0,1 of this CTA's 128 rows.
    const int quarter = warp & 3;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t lacc = map_to_rank(bar(C::B_ACCE), 0);  // the leader's acc_empty barriers
    int lt = 0;
    for (int tile = cluster; tile < p.num_tiles; tile += nclusters, ++lt) {
      const int buf = lt & 1;
      if (!mbar_wait_warp(bar(C::B_ACCF + buf), (lt >> 1) & 1, abort_flag, p.status)) break;
      tc_fence_after();
      int mb, nb;
      gemm_tile_coords(p, tile, mb, nb);
      const int row = mb * C::PAIR_M + static_cast<int>(rank) * C::BM + quarter * 32 + lane;
      gemm_epilogue_row<NORM>(p, row, row < p.M, nb, tmem + lane_off + buf * C::BN);
      // this warp's TMEM loads have completed (tcgen05.wait::ld in each load)
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster_relaxed(lacc + 8u * static_cast<uint32_t>(buf));
    }
  }

  tc_fence_before();
  __syncthreads();
  // the drain commit also lands in the peer: wait for it there before exiting
  if (!leader && warp == 1 && lane == 0) mbar_drain(bar(C::B_DRAIN), 0);
  cluster_sync();
  if (leader && warp == 0 && lane == 0 &&
      (*abort_flag || *reinterpret_cast<volatile unsigned int*>(p.status) != 0u)) {
    // loads still in flight land before either CTA can exit
    const int n = static_cast<int>(issued_by[0] > issued_by[1] ? issued_by[0] : issued_by[1]);
    for (int i = n - C::STAGES; i < n; ++i) {
      if (i < 0) continue;
      mbar_drain(bar(C::B_FULL + i % C::STAGES), (i / C::STAGES) & 1);
    }
  }
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, C::TM_COLS);
  }
}

}  // namespace b2a
