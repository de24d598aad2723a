// Non-causal flash-style attention forward for sm_100a (tcgen05 + TMEM + TMA).
//
// Computes, per head h and query row i, o_i = sum_j softmax_j(scale*q_i.k_j) v_j
// and the natural-log log-sum-exp of the scaled logits ("Multi-Device
// Attention Inference with TensorRT", Introduction: every token attends to
// every token; "Tensor Parallelism: Sharding Weights for Parallel Layer
// Execution", section 3, step 3: attention per head).  Keys are visited in
// 128-wide tiles with an online (running-max) softmax, the form ring
// attention relies on (TensorRT 11.0 multi-device article, Ring Attention).
//
// Used for head dim 64, and for head dim 128 when a call has fewer than 48
// key tiles (longer key ranges run on CTA pairs, attn_pair.cuh: this kernel's
// pipeline fills and drains in fewer SM-cycles per row).  Both write their
// results through attn_epilogue below, in the monolithic, partial or
// accumulate (ring step) form.
// One CTA owns two 128-row query tiles of one head and one key range: the
// call's keys, or one of its P key chunks when a launch computes every
// chunk's partial (CTA x = row block * P + chunk).  Warp roles (18 warps):
//   warps 0-7   softmax for query tile 0, warps 8-15 for query tile 1.  Each
//               row is shared by two threads (warps w and w+4 of a group, the
//               same TMEM lane quarter), each owning 64 of the tile's 128
//               score columns; the two exchange their row max through shared
//               memory with a 64-thread named barrier.
//   warp  16    TMA producer (Q once, then K_j, V_j through a smem ring;
//               it also prefetches the next wave's Q tile into L2)
//   warp  17    TMEM allocator and single-thread tcgen05.mma issuer
// TMEM (512 columns x 128 lanes, fp32): S0 | S1 | O0 | O1.  The softmax
// writes P (fp16, two per column) over the first half of its S block and the
// PV MMA reads it from there as the A operand.  MMA issue order per key tile
// j interleaves the two query tiles so that one softmax group works while
// the tensor core runs the other group's MMAs:
//   QK0(0) QK1(0) | PV0(0) QK0(1) PV1(0) QK1(1) | PV0(1) QK0(2) ...
// A commit after every PV_q(j) (o_done of the query tile) lets the softmax
// rescale its O row in place once PV_q(j-1) has landed (done lazily, only
// when the running max grows by more than 2^14, which keeps every P value
// <= 16384).
//
// The tile stays 128 keys wide on purpose: QK^T MMAs of N = 128 read their
// shared-memory operands at exactly the 128 B/clk the tensor core's
// shared-memory path delivers; narrower tiles oversubscribe it, and then
// every mbarrier operation issued meanwhile stalls behind the MMA reads.
#pragma once

#include <cmath>

#include "ptx.cuh"

namespace b2a {

struct AttnParams {
  int Sq;             // query rows
  int Skv;            // key/value rows
  int H;              // heads
  int lse_ld;         // row stride of lse / lse_part ([H, lse_ld]); Sq unless a row block
  float scale_log2;   // scale * log2(e)
  uint16_t* out;      // monolithic: fp16 [Sq, ld_o], head h at column h*D;
                      // accumulate: fp16 [Sq, H, D] (ld_o = H*D) or null
  int ld_o;
  float* lse;         // monolithic: fp32 [H, Sq] (nullable)
  float* o_part;      // partial: fp32 [Sq, H, D]; accumulate: running o_acc (in place)
  float* lse_part;    // partial: fp32 [H, Sq]; accumulate: running lse_acc (in place)
  unsigned int* status;
  int wave;           // CTAs resident at once (one per SM); 0: no L2 prefetch of Q
  // Key chunks in one launch (single-CTA kernel): with nchunks = P > 1, chunk
  // c = keys [c*Skv/P, (c+1)*Skv/P) and its outputs sit at out / o_part +
  // c * out_chunk_stride and lse / lse_part + c * lse_chunk_stride
  // (elements); grid.x = row blocks * P with the chunk varying fastest.
  int nchunks;
  long long out_chunk_stride;
  long long lse_chunk_stride;
};

template <int D>
struct AttnShape {
  static_assert(D == 64 || D == 128, "head dim 64 or 128");
  static constexpr int BM = 128;                  // query rows per tile
  static constexpr int BN = 128;                  // keys per tile
  static constexpr int QT = 2;                    // query tiles per CTA
  static constexpr int HALF = BN / 2;             // score columns per softmax thread
  static constexpr int OH = D / 2;                // output columns per softmax thread
  static constexpr int SUB = D / 64;              // 128-byte column blocks per row
  static constexpr int SUB_BYTES = 128 * 128;     // one [128 rows x 128 B] block
  static constexpr int Q_BYTES = BM * D * 2;
  static constexpr int KV_BYTES = BN * D * 2;
  static constexpr int STAGES = D == 128 ? 4 : 8;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_KV = QT * Q_BYTES;
  static constexpr int OFF_BAR = OFF_KV + STAGES * KV_BYTES;
  // barriers: q_full, kv_full[STAGES], kv_empty[STAGES], s_full[2], p_full[2],
  //           o_full[2], drain
  static constexpr int B_Q = 0;
  static constexpr int B_KVF = 1;
  static constexpr int B_KVE = 1 + STAGES;
  static constexpr int B_S = 1 + 2 * STAGES;
  static constexpr int B_P = B_S + 2;
  static constexpr int B_O = B_P + 2;
  static constexpr int B_DRAIN = B_O + 2;
  static constexpr int NBAR = B_DRAIN + 1;
  // row-max exchange: [tile][parity][half][row] floats, then the final row
  // sums: [tile][row] floats
  static constexpr int OFF_RED = OFF_BAR + NBAR * 8;
  static constexpr int OFF_LSUM = OFF_RED + QT * 2 * 2 * BM * 4;
  static constexpr int OFF_MISC = OFF_LSUM + QT * BM * 4;
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;  // + slack for 1 KB alignment
  static constexpr int TM_S0 = 0, TM_S1 = 128, TM_O0 = 256, TM_O1 = 256 + D;
  static constexpr int TM_COLS = 512;
  static constexpr int SOFTMAX_WARPS = 16;
  static constexpr int WARP_TMA = 16, WARP_MMA = 17;
  static constexpr int THREADS = 18 * 32;
  static constexpr int ROWS_PER_CTA = QT * BM;
};

// Running max is kept in units of log2-scaled logits; P = 2^(t - m) <= 2^14
// (fp16 holds it with its usual 11-bit precision, 4x below its largest
// finite value).  On the 32k workload (Q ~ N(0, 4^2)) a threshold of 8 made
// a softmax warp rescale in 21% of the key tiles of a 4096-key chunk (7%
// over 32768 keys), each one waiting for the previous PV; 12 brings that to
// 2% (1.4%), 14 to 0.5% (0.3%).
constexpr float kRescaleThreshold = 14.0f;
constexpr float kLn2 = 0.69314718055994530942f;

// Optional per-tile event trace (build with -DB2A_TRACE): one CTA records
// SM clock stamps of each role's events into g_attn_trace[event][tile].
enum AttnTraceEvent : int {
  kTrSReady0 = 0, kTrLdDone0, kTrMaxDone0, kTrPDone0,    // softmax, query tile 0
  kTrSReady1, kTrLdDone1, kTrMaxDone1, kTrPDone1,        // softmax, query tile 1
  kTrPv0Issue, kTrQk0Issue, kTrPv1Issue, kTrQk1Issue,    // MMA issuer
  kTrKLoad, kTrVLoad,                                    // TMA producer
  kTrPv0Done, kTrPv1Done,                                // MMA issuer, PV issued
  kTrSlotWait, kTrSlotReady,                             // MMA issuer, K/V slot wait
  kTrEvents
};
constexpr int kTraceTiles = 512;
#ifdef B2A_TRACE
__device__ unsigned long long g_attn_trace[kTrEvents][kTraceTiles];
__device__ unsigned long long g_attn_trace_ns[kTrEvents][kTraceTiles];  // %globaltimer
__device__ int g_attn_trace_cta[2];
#define B2A_TR(ev, j)                                                                   \
  do {                                                                                  \
    if (tracing && (j) < kTraceTiles) {                                                 \
      g_attn_trace[(ev)][(j)] = clock64();                                              \
      g_attn_trace_ns[(ev)][(j)] = global_timer_ns();                                   \
    }                                                                                   \
  } while (0)
#else
#define B2A_TR(ev, j) \
  do {                \
  } while (0)
#endif

__device__ __forceinline__ float lg2_approx(float x) {
  float y;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// 2^x on the FMA/ALU pipes, for x <= 14 (Cody-Waite range reduction, then a
// degree-3 polynomial for 2^f on [-1/2, 1/2] whose coefficients come from
// the Remez fit in fit_exp2_poly.py; max relative error 7.5e-5, below the
// fp16 rounding that P receives).  x is clamped at -126 so that the exponent
// arithmetic stays in range; 2^-126 rounds to 0 in fp16.
__device__ __forceinline__ float exp2_poly(float x) {
  x = fmaxf(x, -126.f);
  const float t = x + 12582912.f;              // 1.5 * 2^23: rounds x to an integer n
  const float n = t - 12582912.f;
  const float f = x - n;                       // f in [-1/2, 1/2]
  float p = 0.0551716685295105f;
  p = fmaf(p, f, 0.2426111251115799f);
  p = fmaf(p, f, 0.6932609677314758f);
  p = fmaf(p, f, 0.9999280571937561f);
  // low bits of t hold n; shifting them into the exponent field scales by 2^n
  return __int_as_float(__float_as_int(p) + (__float_as_int(t) << 23));
}

// What a launch writes.  kModeFwd: fp16 out + optional lse (attn_fwd);
// kModePartial: fp32 o_part + lse_part of one key chunk (attn_fwd_partial);
// kModeAccum: one ring step in place -- the chunk's result is merged into
// the running fp32 o_acc / lse_acc held in o_part / lse_part (the exact
// log-sum-exp combine of ring attention's online softmax), optionally also
// writing the fp16 rounding of the merged output to out.
enum AttnMode : int { kModeFwd = 0, kModePartial = 1, kModeAccum = 2 };

constexpr float kLog2eF = 1.4426950408889634f;

// The running log-sum-exp of one row in log2 units (accumulate mode only;
// -inf when no keys have been folded in yet).  Read by every thread of the
// row before the row-sum exchange, which orders it before the update.
template <int MODE>
__device__ __forceinline__ float accum_lse2(const AttnParams& p, int row, int head) {
  if constexpr (MODE == kModeAccum) {
    if (row < p.Sq) return p.lse_part[static_cast<size_t>(head) * p.lse_ld + row] * kLog2eF;
  }
  return -INFINITY;
}

// Named barriers over ``n`` threads (a multiple of 32): plain, and returning
// the AND of every thread's ``v``.
__device__ __forceinline__ void named_bar_sync(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}
__device__ __forceinline__ bool named_bar_and(int id, int n, bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred pi, po;\n\t"
      "setp.ne.u32 pi, %1, 0;\n\t"
      "bar.red.and.pred po, %2, %3, pi;\n\t"
      "selp.u32 %0, 1, 0, po;\n\t}\n"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(v)), "r"(id), "r"(n)
      : "memory");
  return r != 0;
}

// Epilogue of a 128-row tile, staged through shared memory.  Values: O
// scaled by 1/l in fp32, then fp16 (monolithic) or fp32 (partial); in
// accumulate mode the merge wa * o_acc + wc * O with the row's running lse
// (the exact log-sum-exp combine), optionally also rounded to fp16.  Each
// thread writes its NC columns into ``stage`` ([128 rows x D] in the output
// type, fp32 in accumulate mode; 16-byte chunks XOR-swizzled by row so that
// neither these writes nor the reads below conflict on banks); after a
// barrier of the tile's 256 threads each warp stores whole output rows, so
// a store instruction covers 256-512 contiguous bytes instead of 16 bytes in
// each of 32 rows (measured: 8-tile partial pass 662 -> 758 TFLOP/s).  ``stage`` must
// be shared memory no MMA or copy touches any more; ``wa_s`` (accumulate
// mode) 128 floats of free shared memory for the rows' o_acc weights; ``la``
// the row's running lse (log2 units, accumulate mode).  All 256 threads call
// this with the same ``ok``; with ok false nothing is written.
template <int D, int MODE, int NC>
__device__ __forceinline__ void attn_epilogue(const AttnParams& p, int row0, int row_in_tile, int head,
                                                     int col, bool write_lse, uint32_t tO, float m, float l,
                                                     float la, uint8_t* stage, float* wa_s, int bar_id, int wt,
                                                     int lane, bool ok) {
  static_assert(NC % 32 == 0, "whole 32-column TMEM loads");
  constexpr int EB = MODE == kModeFwd ? 2 : 4;  // bytes per staged element
  constexpr int PITCH = D * EB;                 // staging bytes per row
  constexpr int CHUNKS = PITCH / 16;            // 16-byte chunks per row
  static_assert(CHUNKS >= 8, "the swizzle permutes 8 chunks");
  if (!named_bar_and(bar_id, 256, ok)) return;
  // this CTA's key chunk (0 unless one launch covers several)
  const size_t chunk = p.nchunks > 1 ? static_cast<size_t>(blockIdx.x % p.nchunks) : 0;
  const float lse2 = m + lg2_approx(l);  // this launch's keys, log2 units
  float wc = 1.f / l;                    // weight of the TMEM accumulator
  float lse_new2 = lse2;
  if constexpr (MODE == kModeAccum) {
    float wa = 0.f;                      // weight of the running output
    if (la > -INFINITY) {
      const float mx = fmaxf(la, lse2);
      const float ea = ex2_approx(la - mx), ec = ex2_approx(lse2 - mx);
      const float inv = 1.f / (ea + ec);
      lse_new2 = mx + lg2_approx(ea + ec);
      wa = ea * inv;
      wc = ec * inv / l;
    }
    if (write_lse) wa_s[row_in_tile] = wa;
  }
  const int sw = row_in_tile & 7;
  uint8_t* srow = stage + row_in_tile * PITCH;
#pragma unroll
  for (int cb = 0; cb < NC; cb += 32) {
    uint32_t o[32];
    tmem_ld32(tO + cb, o);
    tmem_wait_ld(o);
    if constexpr (EB == 2) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int c = (col + cb) / 8 + i;
        const uint32_t* a = o + 8 * i;
        *reinterpret_cast<uint4*>(srow + ((c ^ sw) << 4)) =
            make_uint4(pack_half2(__uint_as_float(a[0]) * wc, __uint_as_float(a[1]) * wc),
                       pack_half2(__uint_as_float(a[2]) * wc, __uint_as_float(a[3]) * wc),
                       pack_half2(__uint_as_float(a[4]) * wc, __uint_as_float(a[5]) * wc),
                       pack_half2(__uint_as_float(a[6]) * wc, __uint_as_float(a[7]) * wc));
      }
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int c = (col + cb) / 4 + i;
        const uint32_t* a = o + 4 * i;
        *reinterpret_cast<float4*>(srow + ((c ^ sw) << 4)) =
            make_float4(__uint_as_float(a[0]) * wc, __uint_as_float(a[1]) * wc, __uint_as_float(a[2]) * wc,
                        __uint_as_float(a[3]) * wc);
      }
    }
  }
  const int row = row0 + row_in_tile;
  if (write_lse && row < p.Sq) {
    const size_t li = chunk * p.lse_chunk_stride + static_cast<size_t>(head) * p.lse_ld + row;
    if constexpr (MODE == kModeFwd) {
      if (p.lse) p.lse[li] = lse2 * kLn2;
    } else {
      p.lse_part[li] = lse_new2 * kLn2;
    }
  }
  named_bar_sync(bar_id, 256);
  uint8_t* dst;
  size_t row_bytes;
  if constexpr (MODE == kModeFwd) {
    dst = reinterpret_cast<uint8_t*>(p.out + chunk * p.out_chunk_stride) + static_cast<size_t>(head) * D * 2;
    row_bytes = static_cast<size_t>(p.ld_o) * 2;
  } else {
    dst = reinterpret_cast<uint8_t*>(p.o_part + chunk * p.out_chunk_stride) + static_cast<size_t>(head) * D * 4;
    row_bytes = static_cast<size_t>(p.H) * D * 4;
  }
  const int rows = p.Sq - row0 < 128 ? p.Sq - row0 : 128;
#pragma unroll 4
  for (int i = wt * 32 + lane; i < rows * CHUNKS; i += 256) {
    const int r = i / CHUNKS, c = i - r * CHUNKS;
    uint4 v = *reinterpret_cast<const uint4*>(stage + r * PITCH + ((c ^ (r & 7)) << 4));
    uint8_t* g = dst + static_cast<size_t>(row0 + r) * row_bytes + (c << 4);
    if constexpr (MODE == kModeAccum) {
      float4 f = make_float4(__uint_as_float(v.x), __uint_as_float(v.y), __uint_as_float(v.z),
                             __uint_as_float(v.w));
      const float wa = wa_s[r];
      if (wa > 0.f) {
        const float4 a = *reinterpret_cast<const float4*>(g);
        f.x = fmaf(wa, a.x, f.x);
        f.y = fmaf(wa, a.y, f.y);
        f.z = fmaf(wa, a.z, f.z);
        f.w = fmaf(wa, a.w, f.w);
      }
      *reinterpret_cast<float4*>(g) = f;
      if (p.out) {
        uint16_t* o16 = p.out + (static_cast<size_t>(row0 + r) * p.H + head) * D + 4 * c;
        *reinterpret_cast<uint2*>(o16) = make_uint2(pack_half2(f.x, f.y), pack_half2(f.z, f.w));
      }
    } else {
      *reinterpret_cast<uint4*>(g) = v;
    }
  }
}


// 64-thread named barrier for the two warps that share rows (ids 1..8).
__device__ __forceinline__ void pair_barrier(int id) {
  asm volatile("bar.sync %0, 64;" ::"r"(id) : "memory");
}

// Same barrier, returning the AND of both warps' ``v``: the pair agrees on
// whether to go on, so neither can be left waiting in bar.sync alone.
__device__ __forceinline__ bool pair_barrier_and(int id, bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred pi, po;\n\t"
      "setp.ne.u32 pi, %1, 0;\n\t"
      "bar.red.and.pred po, %2, 64, pi;\n\t"
      "selp.u32 %0, 1, 0, po;\n\t}\n"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(v)), "r"(id)
      : "memory");
  return r != 0;
}

// EMU: of every 16 score columns, how many take exp2_poly instead of MUFU.
template <int D, int MODE, int EMU>
__global__ void __launch_bounds__(576, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q,
                    const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const AttnParams p) {
  using C = AttnShape<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_u32 = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_u32 & 1023u)) & 1023u);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int head = blockIdx.y;
  // key chunk of this CTA (the whole key range unless the launch covers
  // several chunks; then the chunk varies fastest, so the CTAs running at
  // once share their Q tiles and the head's K/V in L2)
  const int nch = p.nchunks > 1 ? p.nchunks : 1;
  const int chunk = static_cast<int>(blockIdx.x) % nch;
  const int q0 = (static_cast<int>(blockIdx.x) / nch) * C::ROWS_PER_CTA;
  const int key0 = static_cast<int>(static_cast<long long>(chunk) * p.Skv / nch);
  const int klen = static_cast<int>(static_cast<long long>(chunk + 1) * p.Skv / nch) - key0;
  const int nkv = (klen + C::BN - 1) / C::BN;  // >= 1: the host never launches an empty chunk
#ifdef B2A_TRACE
  const bool tracing = blockIdx.x == g_attn_trace_cta[0] && blockIdx.y == g_attn_trace_cta[1];
#endif

  const uint32_t sQ = smem_u32(smem + C::OFF_Q);
  const uint32_t sKV = smem_u32(smem + C::OFF_KV);
  const uint32_t sBar = smem_u32(smem + C::OFF_BAR);
  auto bar = [&](int i) -> uint32_t { return sBar + 8u * static_cast<uint32_t>(i); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);

  if (threadIdx.x == 0) {
    mbar_init(bar(C::B_Q), 1);
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(bar(C::B_KVF + s), 1);
      mbar_init(bar(C::B_KVE + s), 1);
    }
    for (int q = 0; q < 2; ++q) {
      mbar_init(bar(C::B_S + q), 1);
      mbar_init(bar(C::B_P + q), 8);  // one elected arrival per softmax warp of the tile
      mbar_init(bar(C::B_O + q), 1);
    }
    mbar_init(bar(C::B_DRAIN), 1);
    // A CTA launched after an earlier one timed out gives up at its first
    // wait that does not complete at once.
    *abort_flag = (*reinterpret_cast<volatile unsigned int*>(p.status) != 0u) ? 1 : 0;
    fence_mbar_init();
  }
  if (warp == C::WARP_MMA) {
    tmem_alloc(smem_u32(tmem_slot), C::TM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == C::WARP_TMA) {
    // ------------------------------------------------------ TMA producer --
    if (lane == 0) {
      prefetch_tmap(&tm_q);
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_v);
      // end of the query rows this grid covers (debug-build bounds)
      const int q_rows_end = (p.Sq + C::ROWS_PER_CTA - 1) / C::ROWS_PER_CTA * C::ROWS_PER_CTA;
      mbar_arrive_expect_tx(bar(C::B_Q), C::QT * C::Q_BYTES);
#pragma unroll
      for (int qt = 0; qt < C::QT; ++qt)
#pragma unroll
        for (int sb = 0; sb < C::SUB; ++sb)
          tma_load_3d_chk(sQ + qt * C::Q_BYTES + sb * C::SUB_BYTES, C::SUB_BYTES, raw_u32, &tm_q, bar(C::B_Q),
                          sb * 64, head, q0 + qt * C::BM, D, p.H, q_rows_end);
      int issued = 0;
      bool ok = true;
      for (int j = 0; j < nkv && ok; ++j) {
        for (int kind = 0; kind < 2; ++kind) {
          const int idx = 2 * j + kind;
          const int st = idx % C::STAGES;
          const uint32_t par = ((idx / C::STAGES) & 1) ^ 1;
          if (!mbar_wait(bar(C::B_KVE + st), par, abort_flag, p.status)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(bar(C::B_KVF + st), C::KV_BYTES);
          B2A_TR(kind ? kTrVLoad : kTrKLoad, j);
          const CUtensorMap* m = kind ? &tm_v : &tm_k;
#pragma unroll
          for (int sb = 0; sb < C::SUB; ++sb)
            tma_load_3d_chk(sKV + st * C::KV_BYTES + sb * C::SUB_BYTES, C::SUB_BYTES, raw_u32, m,
                            bar(C::B_KVF + st), sb * 64, head, key0 + j * C::BN, D, p.H, key0 + klen);
          ++issued;
        }
        if (j == 0 && p.wave > 0) {
          // Q of the CTA that takes this SM about one wave later: start its
          // DRAM read now so that CTA finds it in L2 (its K/V tiles are
          // shared by the head's CTAs and usually there already).
          const int next = blockIdx.y * gridDim.x + blockIdx.x + p.wave;
          const int nx = (next % gridDim.x) / nch, ny = next / gridDim.x;
          if (ny < static_cast<int>(gridDim.y)) {
#pragma unroll
            for (int qt = 0; qt < C::QT; ++qt) {
              const int row = nx * C::ROWS_PER_CTA + qt * C::BM;
              if (row >= p.Sq) break;
#pragma unroll
              for (int sb = 0; sb < C::SUB; ++sb) tma_prefetch_l2_3d(&tm_q, sb * 64, ny, row);
            }
          }
        }
      }
      if (!ok) {
        // Let every copy still in flight land before the CTA can exit.
        mbar_drain(bar(C::B_Q), 0);
        for (int idx = issued - C::STAGES; idx < issued; ++idx) {
          if (idx < 0) continue;
          mbar_drain(bar(C::B_KVF + idx % C::STAGES), (idx / C::STAGES) & 1);
        }
      }
    }
    __syncwarp();
  } else if (warp == C::WARP_MMA) {
    // ------------------------------------------------------- MMA issuer --
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_f16_f32(128, 128, false, false);
      constexpr uint32_t idesc_pv = idesc_f16_f32(128, D, false, true);
      const uint64_t dq = sw128_desc(sQ, 16, 1024);                 // Q, K-major
      const uint64_t dk = sw128_desc(sKV, 16, 1024);                // K, K-major
      const uint64_t dv = sw128_desc(sKV, C::SUB_BYTES, 1024);      // V, MN-major
      auto issue_qk = [&](int qt, int st) {
        const uint32_t d_t = tmem + (qt ? C::TM_S1 : C::TM_S0);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * C::SUB_BYTES + (kk & 3) * 32;
          mma_ss(d_t, dq + ((qt * C::Q_BYTES + off) >> 4), dk + ((st * C::KV_BYTES + off) >> 4), idesc_qk,
                 kk > 0);
        }
      };
      auto issue_pv = [&](int qt, int st, bool acc) {
        const uint32_t d_t = tmem + (qt ? C::TM_O1 : C::TM_O0);
        const uint32_t a_t = tmem + (qt ? C::TM_S1 : C::TM_S0);
#pragma unroll
        for (int kk = 0; kk < C::BN / 16; ++kk) {
          // V tile is MN-major (d contiguous): 16 keys = 16 rows of 128 B.
          mma_ts(d_t, a_t + kk * 8, dv + ((st * C::KV_BYTES + kk * 2048) >> 4), idesc_pv,
                 (acc || kk > 0) ? 1u : 0u);
        }
      };
      auto wait_kv = [&](int idx, int& st) -> bool {
        st = idx % C::STAGES;
        return mbar_wait(bar(C::B_KVF + st), (idx / C::STAGES) & 1, abort_flag, p.status);
      };
      bool ok = mbar_wait(bar(C::B_Q), 0, abort_flag, p.status);
      int stk = 0, stv = 0;
      if (ok) ok = wait_kv(0, stk);
      if (ok) {
        tc_fence_after();
        issue_qk(0, stk);
        tc_commit(bar(C::B_S + 0));
        issue_qk(1, stk);
        tc_commit(bar(C::B_S + 1));
        tc_commit(bar(C::B_KVE + stk));
      }
      for (int j = 0; j < nkv && ok; ++j) {
        const bool more = (j + 1 < nkv);
        if (!(ok = wait_kv(2 * j + 1, stv))) break;
        if (!(ok = mbar_wait(bar(C::B_P + 0), j & 1, abort_flag, p.status))) break;
        tc_fence_after();
        B2A_TR(kTrPv0Issue, j);
        issue_pv(0, stv, j > 0);
        tc_commit(bar(C::B_O + 0));  // O_0 holds PV0(0..j)
        B2A_TR(kTrPv0Done, j);
        if (more) {
          if (!(ok = wait_kv(2 * j + 2, stk))) break;
          tc_fence_after();
          issue_qk(0, stk);
          tc_commit(bar(C::B_S + 0));
          B2A_TR(kTrQk0Issue, j);
        }
        if (!(ok = mbar_wait(bar(C::B_P + 1), j & 1, abort_flag, p.status))) break;
        tc_fence_after();
        B2A_TR(kTrPv1Issue, j);
        issue_pv(1, stv, j > 0);
        tc_commit(bar(C::B_KVE + stv));
        tc_commit(bar(C::B_O + 1));  // O_1 holds PV1(0..j)
        B2A_TR(kTrPv1Done, j);
        if (more) {
          issue_qk(1, stk);
          tc_commit(bar(C::B_S + 1));
          tc_commit(bar(C::B_KVE + stk));
          B2A_TR(kTrQk1Issue, j);
        }
      }
      // Every MMA issued above must finish before TMEM is released.
      tc_commit(bar(C::B_DRAIN));
      mbar_drain(bar(C::B_DRAIN), 0);
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------- softmax --
    const int qt = warp >> 3;               // query tile
    const int half = (warp >> 2) & 1;       // which 64 of the 128 score columns
    const int quarter = warp & 3;           // TMEM lane quarter
    const int row_in_tile = quarter * 32 + lane;
    const int pair_id = 1 + qt * 4 + quarter;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t tS = tmem + lane_off + (qt ? C::TM_S1 : C::TM_S0);
    const uint32_t tO = tmem + lane_off + (qt ? C::TM_O1 : C::TM_O0) + half * C::OH;
    float* red = reinterpret_cast<float*>(smem + C::OFF_RED) + qt * (2 * 2 * C::BM);
    float* lsum = reinterpret_cast<float*>(smem + C::OFF_LSUM) + qt * C::BM;
    const float sl2 = p.scale_log2;
    float m_used = -INFINITY;  // running max, log2-scaled units (same in both halves)
    float l = 0.f;             // this half's running sum of 2^(t - m_used)
    bool ok = true;
    const bool tr_me = (quarter == 0 && half == 0 && lane == 0);
    (void)tr_me;

    for (int j = 0; j < nkv; ++j) {
      // A failed wait still runs the (harmless) TMEM reads below so that the
      // pair reaches its barrier together; the barrier then stops both.
      const bool got = mbar_wait_warp(bar(C::B_S + qt), j & 1, abort_flag, p.status);
      tc_fence_after();
      if (tr_me) B2A_TR(qt ? kTrSReady1 : kTrSReady0, j);
      uint32_t r0[32], r1[32];
      tmem_ld32(tS + half * C::HALF + 0, r0);
      tmem_ld32(tS + half * C::HALF + 32, r1);
      tmem_wait_ld(r0);
      tmem_wait_ld(r1);
      if (tr_me) B2A_TR(qt ? kTrLdDone1 : kTrLdDone0, j);
      float s[64];
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        s[c] = __uint_as_float(r0[c]);
        s[32 + c] = __uint_as_float(r1[c]);
      }
      if (j + 1 == nkv) {
        // the chunk's last tile: keys past its end are masked (the key count
        // is recomputed here rather than kept live through the loop)
        const int ch = static_cast<int>(blockIdx.x) % nch;
        const int kl = static_cast<int>(static_cast<long long>(ch + 1) * p.Skv / nch) -
                       static_cast<int>(static_cast<long long>(ch) * p.Skv / nch);
        const int valid = kl - j * C::BN - half * C::HALF;
        if (valid < C::HALF) {
#pragma unroll
          for (int c = 0; c < 64; ++c)
            if (c >= valid) s[c] = -INFINITY;
        }
      }
      // this half's row max: four independent 3-input max chains
      float ma = s[0], mb = s[1], mc = s[2], md = s[3];
#pragma unroll
      for (int c = 4; c < 60; c += 8) {
        ma = fmax3(ma, s[c], s[c + 1]);
        mb = fmax3(mb, s[c + 2], s[c + 3]);
        mc = fmax3(mc, s[c + 4], s[c + 5]);
        md = fmax3(md, s[c + 6], s[c + 7]);
      }
      ma = fmax3(ma, s[60], s[61]);
      mb = fmax3(mb, s[62], s[63]);
      const float mx_half = fmax3(ma, mb, fmaxf(mc, md));
      // exchange with the partner thread of the same row; the slot alternates
      // with the tile so a fast partner cannot overwrite an unread value
      float* slot = red + (j & 1) * (2 * C::BM);
      slot[half * C::BM + row_in_tile] = mx_half;
      // The barrier also orders both threads' S loads before any P store
      // below: P of the upper half lands in columns the lower half read.
      // ``ok`` carries a failed O wait of the previous tile into the AND,
      // so a pair always leaves the loop together.
      tc_fence_before();
      if (!pair_barrier_and(pair_id, got && ok)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const float mx = fmaxf(mx_half, slot[(half ^ 1) * C::BM + row_in_tile]);
      if (tr_me) B2A_TR(qt ? kTrMaxDone1 : kTrMaxDone0, j);
      const float m_tile = mx * sl2;
      const float m_new = fmaxf(m_used, m_tile);
      const bool need = m_new > m_used + kRescaleThreshold;
      const float factor = need ? ex2_approx(m_used - m_new) : 1.f;
      if (need) {
        l *= factor;
        m_used = m_new;
      }
      const float neg_m = -m_used;
      float sum[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int cb = 0; cb < 64; cb += 32) {
        // 32 scores -> 16 packed fp16x2 words -> P columns (half*64 + cb)/2 ..
        uint32_t pk[16];
#pragma unroll
        for (int c = 0; c < 32; c += 2) {
          const float x0 = fmaf(s[cb + c], sl2, neg_m);
          const float x1 = fmaf(s[cb + c + 1], sl2, neg_m);
          const float a0 = ((c & 15) >= 16 - EMU) ? exp2_poly(x0) : ex2_approx(x0);
          const float a1 = ((c & 15) + 1 >= 16 - EMU) ? exp2_poly(x1) : ex2_approx(x1);
          sum[(c >> 1) & 3] += a0 + a1;
          pk[c >> 1] = pack_half2(a0, a1);
        }
        tmem_st16(tS + ((half * C::HALF + cb) >> 1), pk);
      }
      l += (sum[0] + sum[1]) + (sum[2] + sum[3]);
      if (j > 0 && __any_sync(0xffffffffu, need)) {
        // Wait for PV_q(j-1) through the commit issued right behind it (o_done
        // of this query tile, one phase per key tile: it cannot be a phase
        // ahead, as PV_q(j) needs this warp's p_full arrival below, nor two
        // behind, as its commit for PV_q(j-2) precedes that of S_q(j)), then
        // rescale O_q in place.
        if (!mbar_wait_warp(bar(C::B_O + qt), (j - 1) & 1, abort_flag, p.status)) {
          ok = false;  // the pair stops at the next exchange (or after the loop)
        } else {
          tc_fence_after();
#pragma unroll
          for (int cb = 0; cb < C::OH; cb += 32) {
            uint32_t o[32];
            tmem_ld32(tO + cb, o);
            tmem_wait_ld(o);
#pragma unroll
            for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * factor);
            tmem_st32(tO + cb, o);
          }
        }
      }
      tmem_wait_st();
      if (tr_me) B2A_TR(qt ? kTrPDone1 : kTrPDone0, j);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(C::B_P + qt));
    }

    const int row = q0 + qt * C::BM + row_in_tile;
    // accumulate mode: both halves read the running lse before the exchange
    // below, which orders the reads before half 0's update in the epilogue
    const float la = accum_lse2<MODE>(p, row, head);
    // combine the two halves' row sums
    if (half == 1) lsum[row_in_tile] = l;
    pair_barrier(pair_id);
    if (half == 0) l += lsum[row_in_tile];
    pair_barrier(pair_id);
    if (half == 0) lsum[row_in_tile] = l;
    pair_barrier(pair_id);
    l = lsum[row_in_tile];

    if (ok) ok = mbar_wait_warp(bar(C::B_O + qt), (nkv - 1) & 1, abort_flag, p.status);
    {
      tc_fence_after();
      // Staging: query tile 0 over Q (its final o_done commit follows every
      // QK), tile 1 over the K/V ring (its final o_done commit follows the
      // kernel's last MMA, and every K/V load has been consumed by then).
      uint8_t* stage = smem + (qt ? C::OFF_KV : C::OFF_Q);
      static_assert(C::QT * C::Q_BYTES >= C::BM * D * 4 && C::STAGES * C::KV_BYTES >= C::BM * D * 4,
                    "an fp32 output tile fits either staging area");
      // the row-max exchange slots are free once both halves have read them
      attn_epilogue<D, MODE, C::OH>(p, q0 + qt * C::BM, row_in_tile, head, half * C::OH, half == 0, tO,
                                           m_used, l, la, stage, red, 9 + qt, warp & 7, lane, ok);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == C::WARP_MMA) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TM_COLS);
  }
}

// Accumulate step with an empty key chunk: the running state is unchanged;
// only the optional fp16 output is written (0 for rows that have seen no key).
__global__ void attn_accum_empty_kernel(const float* o_acc, const float* lse_acc, uint16_t* out, int Sq,
                                        int H, int D) {
  const size_t n = static_cast<size_t>(Sq) * H * D;
  const size_t stride = static_cast<size_t>(gridDim.x) * blockDim.x;
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n; i += stride) {
    const size_t rh = i / D;  // row * H + head
    const int row = static_cast<int>(rh / H), head = static_cast<int>(rh % H);
    const bool seen = lse_acc[static_cast<size_t>(head) * Sq + row] > -INFINITY;
    out[i] = static_cast<uint16_t>(pack_half2(seen ? o_acc[i] : 0.f, 0.f) & 0xffffu);
  }
}

// Fill for an empty key chunk: o = 0, lse = -inf (the empty sum).
template <typename T>  // float or uint16_t (fp16 zero is all-zero bits)
__global__ void attn_empty_partial_kernel(T* o_part, float* lse_part, size_t n_o, size_t n_lse) {
  const size_t stride = static_cast<size_t>(gridDim.x) * blockDim.x;
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n_o; i += stride)
    o_part[i] = T(0);
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n_lse; i += stride)
    lse_part[i] = -INFINITY;
}

}  // namespace b2a
