// Non-causal attention forward on CTA pairs (sm_100a, head dim 128, calls
// with at least 48 key tiles unless chosen explicitly).
//
// Same result as attn_fwd_kernel, bit for bit (per head and query row: the softmax of the
// scaled logits against every key, times V, and the natural-log LSE: "Multi-
// Device Attention Inference with TensorRT", Introduction; "Tensor
// Parallelism: Sharding Weights for Parallel Layer Execution", section 3),
// visiting keys in 128-wide tiles with an online softmax (TensorRT 11.0
// multi-device article, Ring Attention).
//
// A cluster of two CTAs on two SMs owns 256 query rows of one head; each CTA
// holds 128 of them.  Every tensor-core MMA is one M = 256 operation issued
// by the leader CTA (cluster rank 0): each CTA supplies its 128 rows of the A
// operand and half of the B operand from its own shared memory (or TMEM), and
// keeps its 128 rows of the result in its own TMEM.  So each SM loads only
// half of every K tile (64 keys) and half of every V tile (64 of the 128 head
// columns), and the tensor core reads 6 KB of shared memory per 64-cycle
// QK^T step instead of 8 KB.
//
// Per CTA, TMEM holds three score buffers and the output: S[0] | S[1] | S[2]
// | O (4 x 128 columns).  The softmax writes P(j) (fp16) over S[j%3] and PV(j)
// reads it there; in-order tcgen05 execution keeps P(j) alive until PV(j)
// has read it, so the leader issues S(j+3) = Q K(j+3)^T into the same buffer
// once PV(j) has completed:
//   QK(0) QK(1) QK(2) | PV(0) -> QK(3) | PV(1) -> QK(4) | ...
// (PVs and QKs come from two issuing threads; see the PV issuer below).
// Each CTA's softmax therefore finds the scores of its next two tiles
// already computed and runs tile after tile; the P-ready -> PV -> QK -> S
// chain has two softmax periods to complete instead of one.
// Warp roles per CTA (12 warps): warps 0-7 softmax (each row shared by two
// threads, 64 score columns each, row max exchanged through shared memory),
// warp 8 TMA producer, warp 9 TMEM allocator and (leader only) PV issuer,
// warp 10 (leader only) waits for P on the PV issuer's behalf, warp 11
// (leader only) QK issuer.
// Barriers the MMAs depend on (Q and K/V arrival, P ready) live in the
// leader; barriers the MMAs signal (score ready, slot free = PV done) are
// signalled in both CTAs by multicast commits.  The P-ready arrivals that
// cross to the leader are relaxed: each softmax warp has already waited for
// its TMEM stores to complete (tcgen05.wait::st) before arriving, and a
// cluster-scope release costs about a microsecond per arrival on B200.
#pragma once

#include "attn_fwd.cuh"
#include "ptx.cuh"

namespace b2a {


struct AttnPairShape {
  static constexpr int D = 128;
  static constexpr int BM = 128;                  // query rows per CTA (256 per pair)
  static constexpr int BN = 128;                  // keys per tile
  static constexpr int HALF = 64;                 // score / output columns per softmax thread
  static constexpr int NSB = 3;                   // score buffers
  static constexpr int Q_BYTES = BM * D * 2;      // [128 rows x 256 B] as two 128-byte blocks
  static constexpr int QSUB = BM * 128;
  static constexpr int KH_BYTES = 64 * D * 2;     // this CTA's 64 keys of a K tile
  static constexpr int KSUB = 64 * 128;
  static constexpr int VH_BYTES = BN * 64 * 2;    // this CTA's 64 columns of a V tile
  static constexpr int STAGE_BYTES = KH_BYTES + VH_BYTES;
  static constexpr int STAGES = 5;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_KV = Q_BYTES;
  static constexpr int OFF_BAR = OFF_KV + STAGES * STAGE_BYTES;
  // barriers: q_full, kv_full[STAGES], kv_empty[STAGES] (= PV of the
  //           stage's tile done), s_full[NSB], p_full[NSB], o_final, drain
  static constexpr int B_Q = 0;
  static constexpr int B_KVF = 1;
  static constexpr int B_KVE = 1 + STAGES;
  static constexpr int B_S = 1 + 2 * STAGES;
  static constexpr int B_P = B_S + NSB;
  static constexpr int B_OF = B_P + NSB;
  static constexpr int B_DRAIN = B_OF + 1;    // the PV issuer's last commit
  static constexpr int B_DRAIN2 = B_DRAIN + 1;  // the QK issuer's last commit
  static constexpr int NBAR = B_DRAIN2 + 1;
  static constexpr int OFF_RED = OFF_BAR + NBAR * 8;           // [parity][half][row] floats
  static constexpr int OFF_LSUM = OFF_RED + 2 * 2 * BM * 4;    // [row] floats
  static constexpr int OFF_MISC = OFF_LSUM + BM * 4;
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;
  static constexpr int TM_O = NSB * 128;
  static constexpr int TM_COLS = 512;
  static constexpr int THREADS = 384;
  static constexpr int WARP_TMA = 8, WARP_MMA = 9, WARP_SYNC = 10, WARP_QK = 11;
  static constexpr int BAR_HANDOFF = 5;    // named barrier: MMA warp + helper warp
  static constexpr int BAR_EPI = 6;        // named barrier: the 8 softmax warps (epilogue)
  static constexpr int P_ARRIVALS = 16;                        // 8 softmax warps x 2 CTAs
  static constexpr int ROWS_PER_PAIR = 2 * BM;
  __host__ __device__ static constexpr int tm_s(int buf) { return 128 * buf; }
  static_assert(TM_O + D <= TM_COLS, "score buffers and O must fit in TMEM");
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory per CTA");
};

template <int MODE>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(384, 1)
    attn_pair_kernel(const __grid_constant__ CUtensorMap tm_q,
                     const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, const AttnParams p) {
  using C = AttnPairShape;
  constexpr int D = C::D;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_u32 = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_u32 & 1023u)) & 1023u);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = (rank == 0);
  const int head = blockIdx.y;
  const int q0 = (blockIdx.x >> 1) * C::ROWS_PER_PAIR + static_cast<int>(rank) * C::BM;
  const int nkv = (p.Skv + C::BN - 1) / C::BN;
#ifdef B2A_TRACE
  // the traced pair: leader events in the tile-0 slots, peer in the tile-1 slots
  const bool tracing = (blockIdx.x >> 1) == g_attn_trace_cta[0] && blockIdx.y == g_attn_trace_cta[1];
  const int tr_off = rank ? (kTrSReady1 - kTrSReady0) : 0;
#endif

  const uint32_t sQ = smem_u32(smem + C::OFF_Q);
  const uint32_t sKV = smem_u32(smem + C::OFF_KV);
  const uint32_t sBar = smem_u32(smem + C::OFF_BAR);
  auto bar = [&](int i) -> uint32_t { return sBar + 8u * static_cast<uint32_t>(i); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);
  // [rank]: K/V stages each CTA's producer issued (meaningful in the leader)
  volatile uint32_t* issued_by = reinterpret_cast<volatile uint32_t*>(smem + C::OFF_MISC + 8);

  if (threadIdx.x == 0) {
    mbar_init(bar(C::B_Q), 1);
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(bar(C::B_KVF + s), 1);
      mbar_init(bar(C::B_KVE + s), 1);
    }
    for (int b = 0; b < C::NSB; ++b) {
      mbar_init(bar(C::B_S + b), 1);
      mbar_init(bar(C::B_P + b), C::P_ARRIVALS);
    }
    mbar_init(bar(C::B_OF), 1);
    mbar_init(bar(C::B_DRAIN), 1);
    mbar_init(bar(C::B_DRAIN2), 1);
    // A CTA launched after an earlier one timed out gives up at its first
    // wait that does not complete at once.
    *abort_flag = (*reinterpret_cast<volatile unsigned int*>(p.status) != 0u) ? 1 : 0;
    fence_mbar_init();
  }
  if (warp == C::WARP_MMA) {
    tmem_alloc_pair(smem_u32(tmem_slot), C::TM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  // both CTAs' barriers initialised and TMEM allocated before any cross-CTA use
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == C::WARP_TMA) {
    // ------------------------------------------------------ TMA producer --
    // Both CTAs load their own halves; the bytes complete on the leader's
    // barriers, whose expected counts the leader posts for both CTAs.
    if (lane == 0) {
      prefetch_tmap(&tm_q);
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_v);
      // ends of the query and key rows this launch covers (debug-build bounds)
      const int q_rows_end = (p.Sq + C::ROWS_PER_PAIR - 1) / C::ROWS_PER_PAIR * C::ROWS_PER_PAIR;
      const int kv_rows_end = nkv * C::BN;
      if (leader) mbar_arrive_expect_tx(bar(C::B_Q), 2 * C::Q_BYTES);
      const uint32_t lq = map_to_rank(bar(C::B_Q), 0);
#pragma unroll
      for (int sb = 0; sb < 2; ++sb)
        tma_load_3d_pair_chk(sQ + sb * C::QSUB, C::QSUB, raw_u32, &tm_q, lq, sb * 64, head, q0, D, p.H, q_rows_end);
      int issued = 0;
      bool ok = true;
      for (int j = 0; j < nkv && ok; ++j) {
        const int st = j % C::STAGES;
        if (!mbar_wait(bar(C::B_KVE + st), ((j / C::STAGES) & 1) ^ 1, abort_flag, p.status)) {
          ok = false;
          break;
        }
        if (leader) mbar_arrive_expect_tx(bar(C::B_KVF + st), 2 * C::STAGE_BYTES);
        if (leader) B2A_TR(kTrKLoad, j);
        const uint32_t lf = map_to_rank(bar(C::B_KVF + st), 0);
        const uint32_t dst = sKV + st * C::STAGE_BYTES;
#pragma unroll
        for (int sb = 0; sb < 2; ++sb)
          tma_load_3d_pair_chk(dst + sb * C::KSUB, C::KSUB, raw_u32, &tm_k, lf, sb * 64, head,
                               j * C::BN + static_cast<int>(rank) * 64, D, p.H, kv_rows_end);
        tma_load_3d_pair_chk(dst + C::KH_BYTES, C::VH_BYTES, raw_u32, &tm_v, lf, static_cast<int>(rank) * 64, head,
                             j * C::BN, D, p.H, kv_rows_end);
        ++issued;
      }
      // The leader's barriers count both CTAs' bytes; after a failed wait
      // the leader drains them at the end of the kernel, up to the larger
      // of the two producers' counts.
      st_cluster_u32(map_to_rank(smem_u32(const_cast<uint32_t*>(issued_by + rank)), 0),
                     static_cast<uint32_t>(issued));
    }
    __syncwarp();
  } else if (warp == C::WARP_MMA) {
    // --------------------------------------------------- PV issuer (leader) --
    // The MMAs come from two threads (tcgen05.mma from several threads is
    // unordered between them, ordered within each).  This one issues PV(j)
    // into O; warp WARP_QK issues QK(j+3) into S[j%3] once PV(j) has read
    // P(j) from there (its kv_empty commit).  A synchronising instruction of
    // an issuing thread (a barrier poll, a named barrier) waits behind the
    // MMAs it has queued while the tensor core drains, so with one issuer
    // every poll left a gap; with two, each fills the other's gaps (probe:
    // 1438 -> 1172 cycles per tile with no softmax work).  The helper warp
    // waits for P(j) for this thread, and the two meet at a named barrier
    // per tile (which also carries whether to go on).
    if (leader) {
      constexpr uint32_t idesc_pv = idesc_f16_f32(256, D, false, true);
      const uint64_t dv = sw128_desc(sKV + C::KH_BYTES, C::KSUB, 1024);  // V half, MN-major
      auto issue_pv = [&](int buf, int st, bool acc) {
#pragma unroll
        for (int kk = 0; kk < C::BN / 16; ++kk)
          mma_ts_pair(tmem + C::TM_O, tmem + C::tm_s(buf) + kk * 8,
                      dv + ((st * C::STAGE_BYTES + kk * 2048) >> 4), idesc_pv, (acc || kk > 0) ? 1u : 0u);
      };
      // score buffer and K/V stage of tile j
      int buf = 0, st = 0;
      for (int j = 0; j < nkv; ++j) {
        if (!pair_barrier_and(C::BAR_HANDOFF, true)) break;
        if (lane == 0) {
          tc_fence_after();
          B2A_TR(kTrPv0Issue, j);
          issue_pv(buf, st, j > 0);
          // PV(j) done: K(j)/V(j) consumed, P(j)'s buffer free for QK(j+3),
          // and O holds PV(0..j) for the softmax's rescale
          tc_commit_pair(bar(C::B_KVE + st));
          if (j + 1 == nkv) tc_commit_pair(bar(C::B_OF));
          B2A_TR(kTrPv0Done, j);
        }
        __syncwarp();
        if (++buf == C::NSB) buf = 0;
        if (++st == C::STAGES) st = 0;
      }
      if (lane == 0) {
        // Every MMA this thread issued must finish before TMEM is released.
        tc_commit_pair(bar(C::B_DRAIN));
        mbar_drain(bar(C::B_DRAIN), 0);
      }
    }
    __syncwarp();
  } else if (warp == C::WARP_QK) {
    // --------------------------------------------------- QK issuer (leader) --
    if (leader && lane == 0) {
      constexpr uint32_t idesc_qk = idesc_f16_f32(256, 128, false, false);
      const uint64_t dq = sw128_desc(sQ, 16, 1024);   // Q, K-major
      const uint64_t dk = sw128_desc(sKV, 16, 1024);  // K half, K-major
      auto issue_qk = [&](int buf, int st) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t qoff = (kk >> 2) * C::QSUB + (kk & 3) * 32;
          const uint32_t koff = st * C::STAGE_BYTES + (kk >> 2) * C::KSUB + (kk & 3) * 32;
          mma_ss_pair(tmem + C::tm_s(buf), dq + (qoff >> 4), dk + (koff >> 4), idesc_qk, kk > 0);
        }
      };
      bool ok = mbar_wait(bar(C::B_Q), 0, abort_flag, p.status);
      for (int j = 0; j < C::NSB && j < nkv && ok; ++j) {
        if (!(ok = mbar_wait(bar(C::B_KVF + j % C::STAGES), (j / C::STAGES) & 1, abort_flag, p.status))) break;
        tc_fence_after();
        issue_qk(j, j % C::STAGES);
        tc_commit_pair(bar(C::B_S + j));
      }
      // QK(j+3) into S[j%3] after PV(j) (kv_empty of tile j's stage: it
      // cannot be a phase ahead, PV(j+STAGES) needs QK(j+STAGES) from this
      // thread) and K(j+3)'s arrival
      int buf = 0, st = 0, sph = 0, st3 = C::NSB % C::STAGES, sph3 = (C::NSB / C::STAGES) & 1;
      for (int j = 0; j + C::NSB < nkv && ok; ++j) {
        if (!(ok = mbar_wait(bar(C::B_KVE + st), sph, abort_flag, p.status))) break;
        if (!(ok = mbar_wait(bar(C::B_KVF + st3), sph3, abort_flag, p.status))) break;
        tc_fence_after();
        issue_qk(buf, st3);
        tc_commit_pair(bar(C::B_S + buf));
        B2A_TR(kTrQk0Issue, j);
        if (++buf == C::NSB) buf = 0;
        if (++st == C::STAGES) { st = 0; sph ^= 1; }
        if (++st3 == C::STAGES) { st3 = 0; sph3 ^= 1; }
      }
      // every QK this thread issued must finish before TMEM is released
      tc_commit_pair(bar(C::B_DRAIN2));
      mbar_drain(bar(C::B_DRAIN2), 0);
    }
    __syncwarp();
  } else if (warp == C::WARP_SYNC) {
    // ---------------------------------------------- helper (leader only) --
    if (leader) {
      int bph = 0, buf = 0;
      for (int j = 0; j < nkv; ++j) {
        int ok = 1;
        if (lane == 0) {
          B2A_TR(kTrSlotWait, j);
          // arrivals from the other CTA do not wake a suspended try_wait
          // promptly: poll without suspending
          ok = mbar_spin(bar(C::B_P + buf), bph, abort_flag, p.status);
          B2A_TR(kTrSlotReady, j);
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!pair_barrier_and(C::BAR_HANDOFF, ok != 0)) break;
        if (++buf == C::NSB) { buf = 0; bph ^= 1; }
      }
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------- softmax --
    const int half = warp >> 2;             // which 64 of the 128 score columns
    const int quarter = warp & 3;           // TMEM lane quarter
    const int row_in_tile = quarter * 32 + lane;
    const int pair_id = 1 + quarter;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t tO = tmem + lane_off + C::TM_O + half * C::HALF;
    float* red = reinterpret_cast<float*>(smem + C::OFF_RED);
    float* lsum = reinterpret_cast<float*>(smem + C::OFF_LSUM);
    const uint32_t lp_base = map_to_rank(bar(C::B_P), 0);  // the leader's p_full barriers
    const float sl2 = p.scale_log2;
    float m_used = -INFINITY;  // running max, log2-scaled units (same in both halves)
    float l = 0.f;             // this half's running sum of 2^(t - m_used)
    bool ok = true;
#ifdef B2A_TRACE
    const bool tr_me = (quarter == 0 && half == 0 && lane == 0);
#endif

    // score buffer of tile j and its phase bit; K/V stage of tile j - 1 and
    // the phase bit of its kv_empty barrier
    int buf = 0, bph = 0, pst = C::STAGES - 1, psph = 1;
    for (int j = 0; j < nkv; ++j) {
      const uint32_t tS = tmem + lane_off + C::tm_s(buf);
      // A failed wait still runs the (harmless) TMEM reads below so that the
      // pair reaches its barrier together; the barrier then stops both.
      const bool got = mbar_wait_warp(bar(C::B_S + buf), bph, abort_flag, p.status);
      tc_fence_after();
#ifdef B2A_TRACE
      if (tr_me) B2A_TR(kTrSReady0 + tr_off, j);
#endif
      uint32_t r0[32], r1[32];
      tmem_ld32(tS + half * C::HALF + 0, r0);
      tmem_ld32(tS + half * C::HALF + 32, r1);
      tmem_wait_ld(r0);
      tmem_wait_ld(r1);
#ifdef B2A_TRACE
      if (tr_me) B2A_TR(kTrLdDone0 + tr_off, j);
#endif
      float s[64];
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        s[c] = __uint_as_float(r0[c]);
        s[32 + c] = __uint_as_float(r1[c]);
      }
      const int valid = p.Skv - j * C::BN - half * C::HALF;
      if (valid < C::HALF) {
#pragma unroll
        for (int c = 0; c < 64; ++c)
          if (c >= valid) s[c] = -INFINITY;
      }
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
#ifdef B2A_TRACE
      if (tr_me) B2A_TR(kTrMaxDone0 + tr_off, j);
#endif
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
        uint32_t pk[16];
#pragma unroll
        for (int c = 0; c < 32; c += 2) {
          const float a0 = ex2_approx(fmaf(s[cb + c], sl2, neg_m));
          const float a1 = ex2_approx(fmaf(s[cb + c + 1], sl2, neg_m));
          sum[(c >> 1) & 3] += a0 + a1;
          pk[c >> 1] = pack_half2(a0, a1);
        }
        tmem_st16(tS + ((half * C::HALF + cb) >> 1), pk);
      }
      l += (sum[0] + sum[1]) + (sum[2] + sum[3]);
      if (j > 0 && __any_sync(0xffffffffu, need)) {
        // O holds PV(0..j-1); wait for PV(j-1) to complete (the commit
        // right behind it: kv_empty of tile j-1's stage), then rescale.
        // PV(j) waits for this warp's p_full arrival below.  That barrier
        // cannot be a phase ahead (PV(j-1+STAGES) needs P(j-1+STAGES)) nor two
        // behind (tile j-1 was loaded into the stage only after the producer
        // saw PV(j-1-STAGES) signal it).  A later commit, such as the one
        // after QK(j+2), is not used: on B200 it was seen to complete before
        // PV(j-1)'s accumulator writes had landed.
        if (!mbar_wait_warp(bar(C::B_KVE + pst), psph, abort_flag, p.status)) {
          ok = false;  // the pair stops at the next exchange (or after the loop)
        } else {
          tc_fence_after();
#pragma unroll
          for (int cb = 0; cb < C::HALF; cb += 32) {
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
#ifdef B2A_TRACE
      if (tr_me) B2A_TR(kTrPDone0 + tr_off, j);
#endif
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster_relaxed(lp_base + 8u * static_cast<uint32_t>(buf));
      if (++buf == C::NSB) { buf = 0; bph ^= 1; }
      if (++pst == C::STAGES) { pst = 0; psph ^= 1; }
    }

    const int row = q0 + row_in_tile;
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

    if (ok) ok = mbar_wait_warp(bar(C::B_OF), 0, abort_flag, p.status);
    {
      tc_fence_after();
      // staged over this CTA's K/V ring: o_final follows the pair's last MMA,
      // and every load into this CTA had landed before the MMAs that read it
      static_assert(C::STAGES * C::STAGE_BYTES >= C::BM * D * 4, "an fp32 output tile fits the K/V ring");
      // (the row-max exchange slots hold the rows' o_acc weights: both
      // halves have read them)
      attn_epilogue<D, MODE, C::HALF>(p, q0, row_in_tile, head, half * C::HALF, half == 0, tO, m_used, l,
                                             la, smem + C::OFF_KV, red, C::BAR_EPI, warp, lane, ok);
    }
  }

  tc_fence_before();
  __syncthreads();
  // The drain commit also lands in the peer: wait for it there before the
  // CTA can exit.  (Not earlier: a thread polling a barrier for the whole
  // kernel slows the pair's tensor-core work on that SM.)
  if (!leader && warp == C::WARP_MMA && lane == 0) {
    mbar_drain(bar(C::B_DRAIN), 0);
    mbar_drain(bar(C::B_DRAIN2), 0);
  }
  // neither CTA releases TMEM or exits while the pair's MMAs or loads may
  // still touch its TMEM, shared memory or barriers
  cluster_sync();
  if (leader && warp == C::WARP_TMA && lane == 0 &&
      (*abort_flag || *reinterpret_cast<volatile unsigned int*>(p.status) != 0u)) {
    const int n = static_cast<int>(issued_by[0] > issued_by[1] ? issued_by[0] : issued_by[1]);
    mbar_drain(bar(C::B_Q), 0);
    for (int i = n - C::STAGES; i < n; ++i) {
      if (i < 0) continue;
      mbar_drain(bar(C::B_KVF + i % C::STAGES), (i / C::STAGES) & 1);
    }
  }
  cluster_sync();
  if (warp == C::WARP_MMA) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, C::TM_COLS);
  }
}

}  // namespace b2a
