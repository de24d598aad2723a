// C-ABI implementation of libb200attn.so: argument validation, TMA
// descriptor encoding, kernel launches.  All kernels live in this single
// translation unit so that they can name the device status word directly.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <atomic>
#include <climits>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "b200attn.h"
#include "attn_fwd.cuh"
#include "attn_pair.cuh"
#include "attn_merge.cuh"
#include "gemm.cuh"
#include "ptx.cuh"

namespace {

thread_local int t_last_cuda_error = 0;

int cuda_fail(cudaError_t e) {
  t_last_cuda_error = static_cast<int>(e);
  return B2A_ERR_CUDA;
}

constexpr int kMaxDevices = 64;

struct DeviceInfo {
  bool probed = false;
  bool supported = false;
  int sm_count = 0;
  unsigned int* status = nullptr;
  mutable std::atomic<int> gemm_clusters{0};  // co-resident clusters of gemm_tn_kernel (0: not queried yet)
};

std::mutex g_dev_mu;
DeviceInfo g_dev[kMaxDevices];

// Current device; checks it is an sm_100 part and caches facts about it.
int current_device(const DeviceInfo** info) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e);
  if (dev < 0 || dev >= kMaxDevices) return B2A_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lk(g_dev_mu);
  DeviceInfo& di = g_dev[dev];
  if (!di.probed) {
    int major = 0, minor = 0, sms = 0;
    if ((e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev)) != cudaSuccess)
      return cuda_fail(e);
    if ((e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev)) != cudaSuccess)
      return cuda_fail(e);
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
      return cuda_fail(e);
    di.supported = (major == 10 && minor == 0);
    di.sm_count = sms;
    if (di.supported) {
      void* p = nullptr;
      if ((e = cudaGetSymbolAddress(&p, b2a::g_status_word)) != cudaSuccess) return cuda_fail(e);
      di.status = static_cast<unsigned int*>(p);
    }
    di.probed = true;
  }
  if (!di.supported) return B2A_ERR_UNSUPPORTED;
  *info = &di;
  return B2A_OK;
}

// Failure-path self test: thread 0 waits, through the kernels' own bounded
// wait, on an mbarrier that nothing arrives on; after ``limit_ns`` the wait
// gives up and sets the status word, exactly as a lost arrival would in an
// attention or GEMM kernel.  Thread 1 checks a wait that does complete.
// result[0] = 1 if the first wait reported failure, result[1] = 1 if the
// second reported success.
__global__ void selftest_wait_kernel(unsigned int* status, uint64_t limit_ns, int* result) {
  __shared__ uint64_t bars[2];
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    b2a::mbar_init(b2a::smem_u32(&bars[0]), 1);
    b2a::mbar_init(b2a::smem_u32(&bars[1]), 1);
    abort_flag = 0;
    b2a::fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 1) {
    b2a::mbar_arrive(b2a::smem_u32(&bars[1]));
    result[1] = b2a::mbar_wait(b2a::smem_u32(&bars[1]), 0, &abort_flag, status) ? 1 : 0;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const bool got = b2a::mbar_try_wait(b2a::smem_u32(&bars[0]), 0) ||
                     b2a::mbar_wait_slow(b2a::smem_u32(&bars[0]), 0, &abort_flag, status, limit_ns);
    result[0] = got ? 0 : 1;
  }
}

// ------------------------------------------------------------ TMA maps ----

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

PFN_cuTensorMapEncodeTiled_v12000 encoder() {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  return g_encode;
}

// [rows, H, d] fp16 with row stride ld elements; box = box_rows x 1 head x 64.
int attn_map(CUtensorMap* m, const void* base, int d, int H, int rows, int ld, int box_rows) {
  auto enc = encoder();
  if (!enc) return cuda_fail(cudaErrorNotSupported);
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(H),
                        static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2, static_cast<cuuint64_t>(ld) * 2};
  cuuint32_t box[3] = {64, 1, static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, const_cast<void*>(base), dims, strides, box,
                   estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return cuda_fail(cudaErrorInvalidValue);
  return B2A_OK;
}

// [rows, K] fp16 row-major; box = box_rows x 64.
int gemm_map(CUtensorMap* m, const void* base, int rows, int K, int box_rows) {
  auto enc = encoder();
  if (!enc) return cuda_fail(cudaErrorNotSupported);
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(K) * 2};
  cuuint32_t box[2] = {64, static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(base), dims, strides, box,
                   estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return cuda_fail(cudaErrorInvalidValue);
  return B2A_OK;
}

// ---------------------------------------------------------- validation ----

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline bool good_ld(int ld, int H, int d) {
  return ld > 0 && (ld % 8) == 0 && static_cast<long long>(ld) >= static_cast<long long>(H) * d;
}

inline bool good_scale(float s) { return std::isfinite(s) && s > 0.f; }

int validate_attn(const void* q, const void* k, const void* v, int Sq, int Skv, int H, int d,
                  float scale, int ld_q, int ld_k, int ld_v) {
  if (!q || !k || !v) return B2A_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v)) return B2A_ERR_INVALID_ARG;
  if (Sq < 1 || Skv < 0 || H < 1) return B2A_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return B2A_ERR_INVALID_ARG;
  if (!good_scale(scale)) return B2A_ERR_INVALID_ARG;
  if (!good_ld(ld_q, H, d) || !good_ld(ld_k, H, d) || !good_ld(ld_v, H, d)) return B2A_ERR_INVALID_ARG;
  if (H > 65535) return B2A_ERR_UNSUPPORTED;  // grid.y
  return B2A_OK;
}

constexpr float kLog2e = 1.4426950408889634f;

// Columns (of every 16) whose exponential runs on the FMA pipe.
#ifndef B2A_ATTN_EMU
#define B2A_ATTN_EMU 0
#endif

template <int D, int MODE>
int launch_attn(const void* q, const void* k, const void* v, int Sq, int Skv, int H, int ld_q,
                int ld_k, int ld_v, float scale, b2a::AttnParams prm, cudaStream_t stream) {
  using C = b2a::AttnShape<D>;
  CUtensorMap tq, tk, tv;
  int st;
  if ((st = attn_map(&tq, q, D, H, Sq, ld_q, C::BM)) != B2A_OK) return st;
  if ((st = attn_map(&tk, k, D, H, Skv, ld_k, C::BN)) != B2A_OK) return st;
  if ((st = attn_map(&tv, v, D, H, Skv, ld_v, C::BN)) != B2A_OK) return st;
  prm.Sq = Sq;
  prm.Skv = Skv;
  prm.H = H;
  if (prm.lse_ld == 0) prm.lse_ld = Sq;
  prm.scale_log2 = scale * kLog2e;
  auto kern = b2a::attn_fwd_kernel<D, MODE, B2A_ATTN_EMU>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
  if (e != cudaSuccess) return cuda_fail(e);
  const DeviceInfo* di = nullptr;
  if ((st = current_device(&di)) != B2A_OK) return st;
  prm.wave = di->sm_count;  // shared memory and TMEM allow one CTA per SM
  // one CTA per (row block, key chunk), the chunk varying fastest
  const long long gx = static_cast<long long>((Sq + C::ROWS_PER_CTA - 1) / C::ROWS_PER_CTA) *
                       (prm.nchunks > 1 ? prm.nchunks : 1);
  if (gx > INT_MAX) return B2A_ERR_UNSUPPORTED;
  dim3 grid(static_cast<unsigned>(gx), H);
  kern<<<grid, C::THREADS, C::SMEM_BYTES, stream>>>(tq, tk, tv, prm);
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e);
  return B2A_OK;
}

// Head dim 128 runs on CTA pairs (one M = 256 MMA per pair, each SM loading
// half of every K/V tile) when a launch has at least kPairMinKeyTiles key
// tiles; shorter key ranges and head dim 64 run on single CTAs with two
// query tiles, whose pipeline fills and drains in fewer SM-cycles per row
// (measured on B200 with 32768 query rows: the pair kernel is faster from
// 6144 keys up, by 0.5-1% there and 2-3% at 8192-12288, the single-CTA one by
// 3% at 4096 keys).
constexpr int kPairMinKeyTiles = 48;
std::atomic<int> g_attn_kernel{B2A_ATTN_KERNEL_AUTO};

bool use_pair(int d, int Skv) {
  if (d != 128) return false;
  const int choice = g_attn_kernel.load(std::memory_order_relaxed);
  if (choice == B2A_ATTN_KERNEL_SINGLE) return false;
  if (choice == B2A_ATTN_KERNEL_PAIR) return true;
  return (Skv + 127) / 128 >= kPairMinKeyTiles;
}

template <int MODE>
int launch_attn_pair(const void* q, const void* k, const void* v, int Sq, int Skv, int H, int ld_q,
                     int ld_k, int ld_v, float scale, b2a::AttnParams prm, cudaStream_t stream) {
  using C = b2a::AttnPairShape;
  CUtensorMap tq, tk, tv;
  int st;
  if ((st = attn_map(&tq, q, C::D, H, Sq, ld_q, C::BM)) != B2A_OK) return st;
  if ((st = attn_map(&tk, k, C::D, H, Skv, ld_k, C::BN / 2)) != B2A_OK) return st;
  if ((st = attn_map(&tv, v, C::D, H, Skv, ld_v, C::BN)) != B2A_OK) return st;
  prm.Sq = Sq;
  prm.Skv = Skv;
  prm.H = H;
  if (prm.lse_ld == 0) prm.lse_ld = Sq;
  prm.scale_log2 = scale * kLog2e;
  auto kern = b2a::attn_pair_kernel<MODE>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
  if (e != cudaSuccess) return cuda_fail(e);
  // two CTAs (one cluster) per 256 query rows
  dim3 grid(2 * ((Sq + C::ROWS_PER_PAIR - 1) / C::ROWS_PER_PAIR), H);
  kern<<<grid, C::THREADS, C::SMEM_BYTES, stream>>>(tq, tk, tv, prm);
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e);
  return B2A_OK;
}

template <int MODE>
int launch_any(const void* q, const void* k, const void* v, int Sq, int Skv, int H, int d, int ld_q, int ld_k,
               int ld_v, float scale, b2a::AttnParams prm, cudaStream_t stream) {
  if (use_pair(d, Skv)) return launch_attn_pair<MODE>(q, k, v, Sq, Skv, H, ld_q, ld_k, ld_v, scale, prm, stream);
  if (d == 128) return launch_attn<128, MODE>(q, k, v, Sq, Skv, H, ld_q, ld_k, ld_v, scale, prm, stream);
  return launch_attn<64, MODE>(q, k, v, Sq, Skv, H, ld_q, ld_k, ld_v, scale, prm, stream);
}

int attn_fwd_impl(const uint16_t* q, const uint16_t* k, const uint16_t* v, uint16_t* out, float* lse,
                  int Sq, int Skv, int H, int d, float scale, int ld_q, int ld_k, int ld_v, int ld_o,
                  cudaStream_t stream, int lse_ld = 0) {
  if (Skv < 1) return B2A_ERR_INVALID_ARG;
  int st = validate_attn(q, k, v, Sq, Skv, H, d, scale, ld_q, ld_k, ld_v);
  if (st != B2A_OK) return st;
  if (!out || !aligned16(out) || !good_ld(ld_o, H, d)) return B2A_ERR_INVALID_ARG;
  if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) return B2A_ERR_INVALID_ARG;
  const DeviceInfo* di = nullptr;
  if ((st = current_device(&di)) != B2A_OK) return st;
  b2a::AttnParams prm{};
  prm.out = out;
  prm.ld_o = ld_o;
  prm.lse = lse;
  prm.lse_ld = lse_ld;
  prm.status = di->status;
  return launch_any<b2a::kModeFwd>(q, k, v, Sq, Skv, H, d, ld_q, ld_k, ld_v, scale, prm, stream);
}

int attn_partial_impl(const uint16_t* q, const uint16_t* k, const uint16_t* v, float* o_part,
                      float* lse_part, int Sq, int Skv, int H, int d, float scale, int ld_q, int ld_kv,
                      cudaStream_t stream) {
  int st = validate_attn(q, k, v, Sq, Skv, H, d, scale, ld_q, ld_kv, ld_kv);
  if (st != B2A_OK) return st;
  if (!o_part || !lse_part || !aligned16(o_part) || (reinterpret_cast<uintptr_t>(lse_part) & 3u))
    return B2A_ERR_INVALID_ARG;
  const DeviceInfo* di = nullptr;
  if ((st = current_device(&di)) != B2A_OK) return st;
  if (Skv == 0) {
    const size_t n_o = static_cast<size_t>(Sq) * H * d;
    const size_t n_l = static_cast<size_t>(Sq) * H;
    b2a::attn_empty_partial_kernel<float><<<di->sm_count * 4, 256, 0, stream>>>(o_part, lse_part, n_o, n_l);
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? B2A_OK : cuda_fail(e);
  }
  b2a::AttnParams prm{};
  prm.o_part = o_part;
  prm.lse_part = lse_part;
  prm.status = di->status;
  return launch_any<b2a::kModePartial>(q, k, v, Sq, Skv, H, d, ld_q, ld_kv, ld_kv, scale, prm, stream);
}

// FP16 split-reduction partial: the monolithic epilogue (o / l rounded to
// fp16, lse in fp32) pointed at the chunk's [Sq, H, d] slot and [H, Sq] row.
int attn_partial_f16_impl(const uint16_t* q, const uint16_t* k, const uint16_t* v, uint16_t* o_part,
                          float* lse_part, int Sq, int Skv, int H, int d, float scale, int ld_q, int ld_kv,
                          cudaStream_t stream) {
  int st = validate_attn(q, k, v, Sq, Skv, H, d, scale, ld_q, ld_kv, ld_kv);
  if (st != B2A_OK) return st;
  if (!o_part || !lse_part || !aligned16(o_part) || (reinterpret_cast<uintptr_t>(lse_part) & 3u))
    return B2A_ERR_INVALID_ARG;
  const DeviceInfo* di = nullptr;
  if ((st = current_device(&di)) != B2A_OK) return st;
  if (Skv == 0) {
    const size_t n_o = static_cast<size_t>(Sq) * H * d;
    const size_t n_l = static_cast<size_t>(Sq) * H;
    b2a::attn_empty_partial_kernel<uint16_t><<<di->sm_count * 4, 256, 0, stream>>>(o_part, lse_part, n_o, n_l);
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? B2A_OK : cuda_fail(e);
  }
  b2a::AttnParams prm{};
  prm.out = o_part;
  prm.ld_o = H * d;
  prm.lse = lse_part;
  prm.lse_ld = Sq;
  prm.status = di->status;
  return launch_any<b2a::kModeFwd>(q, k, v, Sq, Skv, H, d, ld_q, ld_kv, ld_kv, scale, prm, stream);
}

// All P key chunks' partials of one call (chunk c = keys [c*Skv/P,
// (c+1)*Skv/P)): one launch of the single-CTA kernel over (row block, chunk,
// head) when the chunks are short enough for it, else one CTA-pair launch
// per chunk.  Per row the arithmetic is that of one attn_fwd_partial call
// per chunk.
int attn_partials_impl(const uint16_t* q, const uint16_t* k, const uint16_t* v, void* o_parts, float* lse_parts,
                       int Sq, int Skv, int P, int H, int d, float scale, int ld_q, int ld_kv, bool f16,
                       cudaStream_t stream) {
  if (P < 1) return B2A_ERR_INVALID_ARG;
  int st = validate_attn(q, k, v, Sq, Skv, H, d, scale, ld_q, ld_kv, ld_kv);
  if (st != B2A_OK) return st;
  if (!o_parts || !lse_parts || !aligned16(o_parts) || (reinterpret_cast<uintptr_t>(lse_parts) & 3u))
    return B2A_ERR_INVALID_ARG;
  const size_t plane = static_cast<size_t>(Sq) * H * d;  // elements of one chunk's o_part
  const size_t lplane = static_cast<size_t>(Sq) * H;
  const int longest = static_cast<int>((static_cast<long long>(Skv) + P - 1) / P);
  // every chunk has keys when Skv >= P (the kernel does not handle empty chunks)
  if (Skv < P || use_pair(d, longest)) {
    for (int c = 0; c < P; ++c) {
      const long long lo = static_cast<long long>(c) * Skv / P;
      const long long hi = static_cast<long long>(c + 1) * Skv / P;
      const size_t off = static_cast<size_t>(lo) * ld_kv;
      const int n = static_cast<int>(hi - lo);
      st = f16 ? attn_partial_f16_impl(q, k + off, v + off, static_cast<uint16_t*>(o_parts) + c * plane,
                                       lse_parts + c * lplane, Sq, n, H, d, scale, ld_q, ld_kv, stream)
               : attn_partial_impl(q, k + off, v + off, static_cast<float*>(o_parts) + c * plane,
                                   lse_parts + c * lplane, Sq, n, H, d, scale, ld_q, ld_kv, stream);
      if (st != B2A_OK) return st;
    }
    return B2A_OK;
  }
  const DeviceInfo* di = nullptr;
  if ((st = current_device(&di)) != B2A_OK) return st;
  b2a::AttnParams prm{};
  prm.status = di->status;
  prm.nchunks = P;
  prm.out_chunk_stride = static_cast<long long>(plane);
  prm.lse_chunk_stride = static_cast<long long>(lplane);
  prm.lse_ld = Sq;
  if (f16) {
    prm.out = static_cast<uint16_t*>(o_parts);
    prm.ld_o = H * d;
    prm.lse = lse_parts;
    return d == 128 ? launch_attn<128, b2a::kModeFwd>(q, k, v, Sq, Skv, H, ld_q, ld_kv, ld_kv, scale, prm, stream)
                    : launch_attn<64, b2a::kModeFwd>(q, k, v, Sq, Skv, H, ld_q, ld_kv, ld_kv, scale, prm, stream);
  }
  prm.o_part = static_cast<float*>(o_parts);
  prm.lse_part = lse_parts;
  return d == 128 ? launch_attn<128, b2a::kModePartial>(q, k, v, Sq, Skv, H, ld_q, ld_kv, ld_kv, scale, prm, stream)
                  : launch_attn<64, b2a::kModePartial>(q, k, v, Sq, Skv, H, ld_q, ld_kv, ld_kv, scale, prm, stream);
}

int attn_accum_impl(const uint16_t* q, const uint16_t* k, const uint16_t* v, float* o_acc, float* lse_acc,
                    uint16_t* out, int Sq, int Skv, int H, int d, float scale, int ld_q, int ld_kv,
                    cudaStream_t stream) {
  int st = validate_attn(q, k, v, Sq, Skv, H, d, scale, ld_q, ld_kv, ld_kv);
  if (st != B2A_OK) return st;
  if (!o_acc || !lse_acc || !aligned16(o_acc) || (reinterpret_cast<uintptr_t>(lse_acc) & 3u))
    return B2A_ERR_INVALID_ARG;
  if (out && !aligned16(out)) return B2A_ERR_INVALID_ARG;
  const DeviceInfo* di = nullptr;
  if ((st = current_device(&di)) != B2A_OK) return st;
  if (Skv == 0) {
    if (!out) return B2A_OK;
    b2a::attn_accum_empty_kernel<<<di->sm_count * 4, 256, 0, stream>>>(o_acc, lse_acc, out, Sq, H, d);
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? B2A_OK : cuda_fail(e);
  }
  b2a::AttnParams prm{};
  prm.o_part = o_acc;
  prm.lse_part = lse_acc;
  prm.out = out;
  prm.ld_o = H * d;
  prm.status = di->status;
  return launch_any<b2a::kModeAccum>(q, k, v, Sq, Skv, H, d, ld_q, ld_kv, ld_kv, scale, prm, stream);
}

template <typename T>
int launch_merge(const T* o_parts, const float* lse_parts, int P, uint16_t* out, float* lse_out, int S, int H,
                 int d, cudaStream_t stream) {
  if (!o_parts || !lse_parts || !out) return B2A_ERR_INVALID_ARG;
  if (!aligned16(o_parts) || !aligned16(out) || (reinterpret_cast<uintptr_t>(lse_parts) & 3u))
    return B2A_ERR_INVALID_ARG;
  if (lse_out && (reinterpret_cast<uintptr_t>(lse_out) & 3u)) return B2A_ERR_INVALID_ARG;
  if (P < 1 || S < 1 || H < 1 || (d != 64 && d != 128)) return B2A_ERR_INVALID_ARG;
  if (P > b2a::kMergeMaxP) return B2A_ERR_UNSUPPORTED;
  const long long npairs = static_cast<long long>(S) * H;
  const long long blocks = (npairs + b2a::kMergePairs - 1) / b2a::kMergePairs;
  if (blocks > INT_MAX) return B2A_ERR_UNSUPPORTED;
  const DeviceInfo* di = nullptr;
  int st = current_device(&di);
  if (st != B2A_OK) return st;
#ifndef B2A_MERGE_PIPE
#define B2A_MERGE_PIPE 1
#endif
  if (B2A_MERGE_PIPE && P <= b2a::kMergePipeMaxP) {
    // persistent, two blocks per SM, weights of the next pair group computed
    // while the current one streams
    auto pk = d == 128 ? b2a::attn_merge_pipe_kernel<128, T> : b2a::attn_merge_pipe_kernel<64, T>;
    const long long grid = blocks < 2LL * di->sm_count ? blocks : 2LL * di->sm_count;
    pk<<<static_cast<unsigned>(grid), b2a::kMergePairs, 0, stream>>>(o_parts, lse_parts, P, S, H, out, lse_out);
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? B2A_OK : cuda_fail(e);
  }
  const int smem = P * b2a::kMergePairs * static_cast<int>(sizeof(float));
  auto kern = d == 128 ? b2a::attn_merge_kernel<128, T> : b2a::attn_merge_kernel<64, T>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return cuda_fail(e);
  kern<<<static_cast<unsigned>(blocks), b2a::kMergePairs, smem, stream>>>(o_parts, lse_parts, P, S, H, out,
                                                                          lse_out);
  e = cudaGetLastError();
  return e == cudaSuccess ? B2A_OK : cuda_fail(e);
}

int attn_merge_impl(const float* o_parts, const float* lse_parts, int P, uint16_t* out, float* lse_out,
                    int S, int H, int d, cudaStream_t stream) {
  return launch_merge<float>(o_parts, lse_parts, P, out, lse_out, S, H, d, stream);
}

// q/k RMSNorm epilogue parameters (null: plain projection).
struct QkNorm {
  const uint16_t* g_q;
  const uint16_t* g_k;
  int H, d;
  float eps;
};

int gemm_impl(const uint16_t* a, const uint16_t* w, const uint16_t* r, uint16_t* c, int M, int N, int K,
              cudaStream_t stream, const QkNorm* norm = nullptr) {
  if (!a || !w || !c) return B2A_ERR_INVALID_ARG;
  if (!aligned16(a) || !aligned16(w) || !aligned16(c) || (r && !aligned16(r))) return B2A_ERR_INVALID_ARG;
  if (M < 1 || N < 1 || K < 1 || (N % 8) != 0 || (K % 8) != 0) return B2A_ERR_INVALID_ARG;
  using G = b2a::GemmShape;
  const long long tiles_m = (M + G::PAIR_M - 1) / G::PAIR_M;  // 256 x 256 tiles, one per CTA pair
  const long long tiles_n = (N + G::BN - 1) / G::BN;
  if (tiles_m * tiles_n > INT_MAX) return B2A_ERR_UNSUPPORTED;
  const DeviceInfo* di = nullptr;
  int st = current_device(&di);
  if (st != B2A_OK) return st;
  CUtensorMap ta, tb;
  if ((st = gemm_map(&ta, a, M, K, G::BM)) != B2A_OK) return st;
  if ((st = gemm_map(&tb, w, N, K, G::BN / 2)) != B2A_OK) return st;
  b2a::GemmParams prm{};
  prm.M = M;
  prm.N = N;
  prm.K = K;
  prm.tiles_m = static_cast<int>(tiles_m);
  prm.tiles_n = static_cast<int>(tiles_n);
  prm.num_tiles = static_cast<int>(tiles_m * tiles_n);
  prm.c = c;
  prm.r = r;
  prm.status = di->status;
  if (norm) {
    prm.g_q = norm->g_q;
    prm.g_k = norm->g_k;
    prm.hsec = norm->H * norm->d;
    prm.dh = norm->d;
    prm.eps = norm->eps;
  }
  auto kern = norm ? b2a::gemm_tn_kernel<true> : b2a::gemm_tn_kernel<false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, G::SMEM_BYTES);
  if (e != cudaSuccess) return cuda_fail(e);
  // persistent: as many clusters of two CTAs as run at once
  int resident = di->gemm_clusters.load(std::memory_order_relaxed);
  if (resident == 0) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(di->sm_count & ~1), 1, 1);
    cfg.blockDim = dim3(G::THREADS, 1, 1);
    cfg.dynamicSmemBytes = G::SMEM_BYTES;
    int n = 0;
    e = cudaOccupancyMaxActiveClusters(&n, kern, &cfg);
    if (e != cudaSuccess || n < 1) {
      (void)cudaGetLastError();
      n = di->sm_count / 2;
    }
    resident = n > 0 ? n : 1;
    di->gemm_clusters.store(resident, std::memory_order_relaxed);
  }
  const int clusters = prm.num_tiles < resident ? prm.num_tiles : resident;
  kern<<<dim3(2 * clusters, 1, 1), G::THREADS, G::SMEM_BYTES, stream>>>(ta, tb, prm);
  e = cudaGetLastError();
  return e == cudaSuccess ? B2A_OK : cuda_fail(e);
}

int qkv_qknorm_impl(const uint16_t* x, const uint16_t* w_qkv, const uint16_t* g_q, const uint16_t* g_k,
                    uint16_t* qkv, int M, int H, int d, int K, float eps, cudaStream_t stream) {
  if (!g_q || !g_k || !aligned16(g_q) || !aligned16(g_k)) return B2A_ERR_INVALID_ARG;
  if (H < 1 || (d != 64 && d != 128) || !std::isfinite(eps) || eps < 0.f) return B2A_ERR_INVALID_ARG;
  const long long n = 3LL * H * d;
  if (n > INT_MAX) return B2A_ERR_UNSUPPORTED;
  const QkNorm norm{g_q, g_k, H, d, eps};
  return gemm_impl(x, w_qkv, nullptr, qkv, M, static_cast<int>(n), K, stream, &norm);
}

// Static scratch of attn_block_fwd_static: qkv [S, 3h] then the attention
// output [S, h], fp16.  A file-scope device array, so no allocator is called;
// host code only ever passes its device address (looked up per device).
constexpr size_t kBlockStaticScratchBytes = size_t(64) << 20;
__device__ __align__(256) uint8_t g_block_static_scratch[kBlockStaticScratchBytes];

uint8_t* g_block_static_ptr[kMaxDevices] = {};

// Address of the static scratch on the current device (set up once per
// device, with that device current).
int block_static_scratch(uint8_t** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e);
  if (dev < 0 || dev >= kMaxDevices) return B2A_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lk(g_dev_mu);
  if (!g_block_static_ptr[dev]) {
    void* ptr = nullptr;
    e = cudaGetSymbolAddress(&ptr, g_block_static_scratch);
    if (e != cudaSuccess) return cuda_fail(e);
    g_block_static_ptr[dev] = static_cast<uint8_t*>(ptr);
  }
  *out = g_block_static_ptr[dev];
  return B2A_OK;
}

// Workspace layout of attn_fwd_host: q | k | v | out | lse [| o_parts | lse_parts],
// each region starting on a 256-byte boundary.
struct HostWs {
  uint64_t q, k, v, out, lse, o_parts, lse_parts, total;
};

inline uint64_t up256(uint64_t x) { return (x + 255u) & ~static_cast<uint64_t>(255u); }

bool host_ws_layout(int S, int H, int d, int P, HostWs* w) {
  if (S < 1 || H < 1 || (d != 64 && d != 128) || P < 1 || P > b2a::kMergeMaxP) return false;
  const uint64_t n = static_cast<uint64_t>(S) * H * d;
  const uint64_t nl = static_cast<uint64_t>(S) * H;
  uint64_t off = 0;
  w->q = off; off = up256(off + n * 2);
  w->k = off; off = up256(off + n * 2);
  w->v = off; off = up256(off + n * 2);
  w->out = off; off = up256(off + n * 2);
  w->lse = off; off = up256(off + nl * 4);
  w->o_parts = off;
  w->lse_parts = off;
  if (P > 1) {
    w->o_parts = off; off = up256(off + static_cast<uint64_t>(P) * n * 4);
    w->lse_parts = off; off = up256(off + static_cast<uint64_t>(P) * nl * 4);
  }
  w->total = off;
  return true;
}

// Copy streams and events of attn_fwd_host, created on first use per device
// (not memory allocations: two streams and a ring of events).
struct HostPipe {
  static constexpr int kEvents = 16;
  std::mutex mu;  // the event ring is shared: one host caller at a time
  cudaStream_t h2d = nullptr, d2h = nullptr;
  cudaEvent_t ev[kEvents] = {};
  bool ready = false;
};
HostPipe g_pipe[kMaxDevices];
std::mutex g_pipe_init_mu;
constexpr int kHostRowBlock = 1024;  // P = 1 splits the query rows in 4 blocks from 4*1024 rows up

int host_pipe(HostPipe** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e);
  if (dev < 0 || dev >= kMaxDevices) return B2A_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lk(g_pipe_init_mu);
  HostPipe& hp = g_pipe[dev];
  if (!hp.ready) {
    if ((e = cudaStreamCreateWithFlags(&hp.h2d, cudaStreamNonBlocking)) != cudaSuccess) return cuda_fail(e);
    if ((e = cudaStreamCreateWithFlags(&hp.d2h, cudaStreamNonBlocking)) != cudaSuccess) return cuda_fail(e);
    for (int i = 0; i < HostPipe::kEvents; ++i)
      if ((e = cudaEventCreateWithFlags(&hp.ev[i], cudaEventDisableTiming)) != cudaSuccess) return cuda_fail(e);
    hp.ready = true;
  }
  *out = &hp;
  return B2A_OK;
}

}  // namespace

extern "C" {

int attn_fwd(const uint16_t* q, const uint16_t* k, const uint16_t* v, uint16_t* out, float* lse, int S,
             int H, int d, float scale, int ld_q, int ld_k, int ld_v, int ld_o, void* stream) {
  return attn_fwd_impl(q, k, v, out, lse, S, S, H, d, scale, ld_q, ld_k, ld_v, ld_o,
                       static_cast<cudaStream_t>(stream));
}

int attn_fwd_batched(const uint16_t* q, const uint16_t* k, const uint16_t* v, uint16_t* out, float* lse, int S,
                     int B, int H, int d, float scale, void* stream) {
  // [S, B, H, d] is [S, B*H, d] with row stride B*H*d: batch b's head h is
  // head b*H + h, and lse [B, H, S] is [B*H, S].  One launch covers every
  // (row block, head, batch).
  if (B < 1 || H < 1 || S < 1) return B2A_ERR_INVALID_ARG;
  const long long bh = static_cast<long long>(B) * H;
  if (bh * d > INT_MAX) return B2A_ERR_UNSUPPORTED;
  const int ld = static_cast<int>(bh * d);
  return attn_fwd_impl(q, k, v, out, lse, S, S, static_cast<int>(bh), d, scale, ld, ld, ld, ld,
                       static_cast<cudaStream_t>(stream));
}

int attn_fwd_gathered_kv(const uint16_t* q, const uint16_t* k, const uint16_t* v, uint16_t* out, float* lse,
                         int Sq, int Skv, int H, int d, float scale, int ld_q, int ld_k, int ld_v, int ld_o,
                         void* stream) {
  return attn_fwd_impl(q, k, v, out, lse, Sq, Skv, H, d, scale, ld_q, ld_k, ld_v, ld_o,
                       static_cast<cudaStream_t>(stream));
}

int attn_fwd_partial(const uint16_t* q, const uint16_t* k_chunk, const uint16_t* v_chunk, float* o_part,
                     float* lse_part, int Sq, int Skv, int H, int d, float scale, int ld_q, int ld_kv,
                     void* stream) {
  return attn_partial_impl(q, k_chunk, v_chunk, o_part, lse_part, Sq, Skv, H, d, scale, ld_q, ld_kv,
                           static_cast<cudaStream_t>(stream));
}

int attn_fwd_partial_f16(const uint16_t* q, const uint16_t* k_chunk, const uint16_t* v_chunk, uint16_t* o_part,
                         float* lse_part, int Sq, int Skv, int H, int d, float scale, int ld_q, int ld_kv,
                         void* stream) {
  return attn_partial_f16_impl(q, k_chunk, v_chunk, o_part, lse_part, Sq, Skv, H, d, scale, ld_q, ld_kv,
                               static_cast<cudaStream_t>(stream));
}

int attn_fwd_partials(const uint16_t* q, const uint16_t* k, const uint16_t* v, float* o_parts, float* lse_parts,
                      int Sq, int Skv, int P, int H, int d, float scale, int ld_q, int ld_kv, void* stream) {
  return attn_partials_impl(q, k, v, o_parts, lse_parts, Sq, Skv, P, H, d, scale, ld_q, ld_kv, false,
                            static_cast<cudaStream_t>(stream));
}

int attn_fwd_partials_f16(const uint16_t* q, const uint16_t* k, const uint16_t* v, uint16_t* o_parts,
                          float* lse_parts, int Sq, int Skv, int P, int H, int d, float scale, int ld_q, int ld_kv,
                          void* stream) {
  return attn_partials_impl(q, k, v, o_parts, lse_parts, Sq, Skv, P, H, d, scale, ld_q, ld_kv, true,
                            static_cast<cudaStream_t>(stream));
}

int attn_fwd_accumulate(const uint16_t* q, const uint16_t* k_chunk, const uint16_t* v_chunk, float* o_acc,
                        float* lse_acc, uint16_t* out, int Sq, int Skv, int H, int d, float scale, int ld_q,
                        int ld_kv, void* stream) {
  return attn_accum_impl(q, k_chunk, v_chunk, o_acc, lse_acc, out, Sq, Skv, H, d, scale, ld_q, ld_kv,
                         static_cast<cudaStream_t>(stream));
}

int b2a_set_attn_kernel(int choice) {
  if (choice != B2A_ATTN_KERNEL_AUTO && choice != B2A_ATTN_KERNEL_SINGLE && choice != B2A_ATTN_KERNEL_PAIR)
    return B2A_ERR_INVALID_ARG;
  g_attn_kernel.store(choice, std::memory_order_relaxed);
  return B2A_OK;
}

int b2a_get_attn_kernel(void) { return g_attn_kernel.load(std::memory_order_relaxed); }

int b2a_attn_kernel_for(int d, int Skv) { return use_pair(d, Skv) ? B2A_ATTN_KERNEL_PAIR : B2A_ATTN_KERNEL_SINGLE; }

int attn_merge(const float* o_parts, const float* lse_parts, int P, uint16_t* out, float* lse_out, int S,
               int H, int d, void* stream) {
  return attn_merge_impl(o_parts, lse_parts, P, out, lse_out, S, H, d, static_cast<cudaStream_t>(stream));
}

int attn_merge_f16(const uint16_t* o_parts, const float* lse_parts, int P, uint16_t* out, float* lse_out, int S,
                   int H, int d, void* stream) {
  return launch_merge<uint16_t>(o_parts, lse_parts, P, out, lse_out, S, H, d, static_cast<cudaStream_t>(stream));
}

int qkv_proj(const uint16_t* x, const uint16_t* w_qkv, uint16_t* qkv, int M, int N, int K, void* stream) {
  return gemm_impl(x, w_qkv, nullptr, qkv, M, N, K, static_cast<cudaStream_t>(stream));
}

int qkv_proj_qknorm(const uint16_t* x, const uint16_t* w_qkv, const uint16_t* g_q, const uint16_t* g_k,
                    uint16_t* qkv, int M, int H, int d, int K, float eps, void* stream) {
  return qkv_qknorm_impl(x, w_qkv, g_q, g_k, qkv, M, H, d, K, eps, static_cast<cudaStream_t>(stream));
}

int out_proj(const uint16_t* a, const uint16_t* w_o, const uint16_t* residual, uint16_t* y, int M, int N,
             int K, void* stream) {
  return gemm_impl(a, w_o, residual, y, M, N, K, static_cast<cudaStream_t>(stream));
}

int attn_block_fwd(const uint16_t* x, const uint16_t* w_qkv, const uint16_t* w_o, uint16_t* y,
                   uint16_t* qkv_ws, uint16_t* attn_ws, int S, int H, int d, float scale, void* stream_) {
  return attn_block_fwd_qknorm(x, w_qkv, nullptr, nullptr, 0.f, w_o, y, qkv_ws, attn_ws, S, H, d, scale, stream_);
}

int attn_block_fwd_qknorm(const uint16_t* x, const uint16_t* w_qkv, const uint16_t* g_q, const uint16_t* g_k,
                          float eps, const uint16_t* w_o, uint16_t* y, uint16_t* qkv_ws, uint16_t* attn_ws, int S,
                          int H, int d, float scale, void* stream_) {
  if (!x || !w_qkv || !w_o || !y || !qkv_ws || !attn_ws) return B2A_ERR_INVALID_ARG;
  if (S < 1 || H < 1 || (d != 64 && d != 128) || !good_scale(scale)) return B2A_ERR_INVALID_ARG;
  if ((g_q == nullptr) != (g_k == nullptr)) return B2A_ERR_INVALID_ARG;
  const long long h = static_cast<long long>(H) * d;
  if (3 * h > INT_MAX) return B2A_ERR_UNSUPPORTED;
  const int hi = static_cast<int>(h);
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  int st = g_q ? qkv_qknorm_impl(x, w_qkv, g_q, g_k, qkv_ws, S, H, d, hi, eps, stream)
               : gemm_impl(x, w_qkv, nullptr, qkv_ws, S, 3 * hi, hi, stream);
  if (st != B2A_OK) return st;
  st = attn_fwd_impl(qkv_ws, qkv_ws + h, qkv_ws + 2 * h, attn_ws, nullptr, S, S, H, d, scale, 3 * hi,
                     3 * hi, 3 * hi, hi, stream);
  if (st != B2A_OK) return st;
  return gemm_impl(attn_ws, w_o, x, y, S, hi, hi, stream);
}

int attn_block_fwd_static(const uint16_t* x, const uint16_t* w_qkv, const uint16_t* w_o, uint16_t* y, int S,
                          int H, int d, float scale, void* stream) {
  if (!x || !w_qkv || !w_o || !y) return B2A_ERR_INVALID_ARG;
  if (S < 1 || H < 1 || (d != 64 && d != 128) || !good_scale(scale)) return B2A_ERR_INVALID_ARG;
  const uint64_t elems = static_cast<uint64_t>(S) * H * d;
  const uint64_t qkv_bytes = (elems * 6 + 255) & ~static_cast<uint64_t>(255);
  if (qkv_bytes + elems * 2 > kBlockStaticScratchBytes) return B2A_ERR_UNSUPPORTED;
  const DeviceInfo* di = nullptr;
  int st = current_device(&di);
  if (st != B2A_OK) return st;
  uint8_t* scratch = nullptr;
  if ((st = block_static_scratch(&scratch)) != B2A_OK) return st;
  return attn_block_fwd(x, w_qkv, w_o, y, reinterpret_cast<uint16_t*>(scratch),
                        reinterpret_cast<uint16_t*>(scratch + qkv_bytes), S, H, d, scale, stream);
}

uint64_t attn_fwd_host_workspace_bytes(int S, int H, int d, int P) {
  HostWs w;
  return host_ws_layout(S, H, d, P, &w) ? w.total : 0;
}

int attn_fwd_host(const uint16_t* q, const uint16_t* k, const uint16_t* v, uint16_t* out, float* lse, int S,
                  int H, int d, float scale, int P, void* workspace, uint64_t workspace_bytes,
                  void* stream_) {
  if (!q || !k || !v || !out || !workspace) return B2A_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return B2A_ERR_INVALID_ARG;
  if (P > b2a::kMergeMaxP) return B2A_ERR_UNSUPPORTED;
  HostWs w;
  if (!host_ws_layout(S, H, d, P, &w)) return B2A_ERR_INVALID_ARG;
  if (!good_scale(scale)) return B2A_ERR_INVALID_ARG;
  if (workspace_bytes < w.total) return B2A_ERR_INVALID_ARG;
  const DeviceInfo* di = nullptr;
  int st = current_device(&di);
  if (st != B2A_OK) return st;
  HostPipe* hp = nullptr;
  if ((st = host_pipe(&hp)) != B2A_OK) return st;
  std::lock_guard<std::mutex> lk(hp->mu);
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  uint16_t* dq = reinterpret_cast<uint16_t*>(ws + w.q);
  uint16_t* dk = reinterpret_cast<uint16_t*>(ws + w.k);
  uint16_t* dv = reinterpret_cast<uint16_t*>(ws + w.v);
  uint16_t* dout = reinterpret_cast<uint16_t*>(ws + w.out);
  float* dlse = reinterpret_cast<float*>(ws + w.lse);
  const int ld = H * d;
  const size_t row16 = static_cast<size_t>(ld) * 2;  // bytes of one fp16 row
  cudaError_t e;
  int ev = 0;
  // signal ``from`` -> ``to`` through the next event of the ring: every wait
  // is enqueued before that event is recorded again, so reuse is safe
  auto handoff = [&](cudaStream_t from, cudaStream_t to) -> cudaError_t {
    cudaEvent_t x = hp->ev[ev++ % HostPipe::kEvents];
    cudaError_t r = cudaEventRecord(x, from);
    return r == cudaSuccess ? cudaStreamWaitEvent(to, x, 0) : r;
  };
  // Copies run on the library's own two copy streams (one per direction) so
  // that they overlap the kernels on ``stream``; events keep every step in
  // order with the caller's earlier and later work on ``stream``.
  if ((e = handoff(stream, hp->h2d)) != cudaSuccess) return cuda_fail(e);
  if ((e = handoff(stream, hp->d2h)) != cudaSuccess) return cuda_fail(e);
  if (P == 1) {
    // K and V first (every query row needs all of them), then query rows in
    // blocks: block b's copy-in, attention and copy-out overlap the others.
    if ((e = cudaMemcpyAsync(dk, k, S * row16, cudaMemcpyHostToDevice, hp->h2d)) != cudaSuccess) return cuda_fail(e);
    if ((e = cudaMemcpyAsync(dv, v, S * row16, cudaMemcpyHostToDevice, hp->h2d)) != cudaSuccess) return cuda_fail(e);
    const int nb = S >= 4 * kHostRowBlock ? 4 : 1;
    for (int b = 0; b < nb; ++b) {
      const int r0 = static_cast<int>(static_cast<long long>(b) * S / nb);
      const int r1 = static_cast<int>(static_cast<long long>(b + 1) * S / nb);
      const size_t off = static_cast<size_t>(r0) * ld;
      if ((e = cudaMemcpyAsync(dq + off, q + off, (r1 - r0) * row16, cudaMemcpyHostToDevice, hp->h2d)) != cudaSuccess)
        return cuda_fail(e);
      if ((e = handoff(hp->h2d, stream)) != cudaSuccess) return cuda_fail(e);
      st = attn_fwd_impl(dq + off, dk, dv, dout + off, dlse + r0, r1 - r0, S, H, d, scale, ld, ld, ld, ld, stream, S);
      if (st != B2A_OK) return st;
      if ((e = handoff(stream, hp->d2h)) != cudaSuccess) return cuda_fail(e);
      if ((e = cudaMemcpyAsync(out + off, dout + off, (r1 - r0) * row16, cudaMemcpyDeviceToHost, hp->d2h)) !=
          cudaSuccess)
        return cuda_fail(e);
      if (lse && (e = cudaMemcpy2DAsync(lse + r0, static_cast<size_t>(S) * 4, dlse + r0, static_cast<size_t>(S) * 4,
                                        static_cast<size_t>(r1 - r0) * 4, H, cudaMemcpyDeviceToHost, hp->d2h)) !=
                     cudaSuccess)
        return cuda_fail(e);
    }
  } else {
    // Ring-attention emulation: Q first, then each key chunk's K/V copy
    // overlaps the previous chunk's partial.
    float* op = reinterpret_cast<float*>(ws + w.o_parts);
    float* lp = reinterpret_cast<float*>(ws + w.lse_parts);
    const size_t n = static_cast<size_t>(S) * H * d;
    const size_t nl = static_cast<size_t>(S) * H;
    if ((e = cudaMemcpyAsync(dq, q, S * row16, cudaMemcpyHostToDevice, hp->h2d)) != cudaSuccess) return cuda_fail(e);
    for (int c = 0; c < P; ++c) {
      const long long lo = static_cast<long long>(c) * S / P;
      const long long hi = static_cast<long long>(c + 1) * S / P;
      const size_t off = static_cast<size_t>(lo) * ld;
      if (hi > lo) {
        if ((e = cudaMemcpyAsync(dk + off, k + off, (hi - lo) * row16, cudaMemcpyHostToDevice, hp->h2d)) != cudaSuccess)
          return cuda_fail(e);
        if ((e = cudaMemcpyAsync(dv + off, v + off, (hi - lo) * row16, cudaMemcpyHostToDevice, hp->h2d)) != cudaSuccess)
          return cuda_fail(e);
      }
      if ((e = handoff(hp->h2d, stream)) != cudaSuccess) return cuda_fail(e);
      st = attn_partial_impl(dq, dk + off, dv + off, op + c * n, lp + c * nl, S, static_cast<int>(hi - lo), H, d,
                             scale, ld, ld, stream);
      if (st != B2A_OK) return st;
    }
    if ((st = attn_merge_impl(op, lp, P, dout, dlse, S, H, d, stream)) != B2A_OK) return st;
    if ((e = handoff(stream, hp->d2h)) != cudaSuccess) return cuda_fail(e);
    if ((e = cudaMemcpyAsync(out, dout, S * row16, cudaMemcpyDeviceToHost, hp->d2h)) != cudaSuccess)
      return cuda_fail(e);
    if (lse && (e = cudaMemcpyAsync(lse, dlse, static_cast<size_t>(S) * H * 4, cudaMemcpyDeviceToHost, hp->d2h)) !=
                   cudaSuccess)
      return cuda_fail(e);
  }
  // the caller's stream resumes after the last copy-out
  if ((e = handoff(hp->d2h, stream)) != cudaSuccess) return cuda_fail(e);
  return B2A_OK;
}

int b2a_selftest_wait_timeout(int limit_ms, int* result, void* stream) {
  if (limit_ms < 1 || limit_ms > 2000 || !result) return B2A_ERR_INVALID_ARG;
  const DeviceInfo* di = nullptr;
  int st = current_device(&di);
  if (st != B2A_OK) return st;
  selftest_wait_kernel<<<1, 64, 0, static_cast<cudaStream_t>(stream)>>>(
      di->status, static_cast<uint64_t>(limit_ms) * 1000000ull, result);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? B2A_OK : cuda_fail(e);
}

int b2a_check_status(void* stream) {
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e);
  const DeviceInfo* di = nullptr;
  int st = current_device(&di);
  if (st != B2A_OK) return st;
  unsigned int v = 0;
  if ((e = cudaMemcpy(&v, di->status, sizeof(v), cudaMemcpyDeviceToHost)) != cudaSuccess) return cuda_fail(e);
  if (v == 0) return B2A_OK;
  const unsigned int zero = 0;
  if ((e = cudaMemcpy(di->status, &zero, sizeof(zero), cudaMemcpyHostToDevice)) != cudaSuccess)
    return cuda_fail(e);
  // a failed bounds check (debug builds) is the cause of any wait that then gave up
  return (v & b2a::kDevErrBounds) ? B2A_ERR_DEVICE_CHECK : B2A_ERR_TIMEOUT;
}

const char* b2a_status_string(int status) {
  switch (status) {
    case B2A_OK: return "ok";
    case B2A_ERR_INVALID_ARG: return "invalid argument";
    case B2A_ERR_UNSUPPORTED: return "unsupported device or size";
    case B2A_ERR_CUDA: return "CUDA runtime error";
    case B2A_ERR_TIMEOUT: return "device-side wait timed out";
    case B2A_ERR_DEVICE_CHECK: return "device-side bounds check failed (debug build)";
    default: return "unknown status";
  }
}

int b2a_last_cuda_error(void) { return t_last_cuda_error; }

int b2a_version(void) { return 104; }

int b2a_debug_build(void) { return b2a::kDebugBuild ? 1 : 0; }

#ifdef B2A_TRACE
// Trace builds only: choose the traced CTA, then read the event table
// ([event][tile] SM clock stamps, b2a::kTrEvents x b2a::kTraceTiles).
__attribute__((visibility("default"))) int b2a_trace_select(int bx, int by) {
  const int v[2] = {bx, by};
  cudaError_t e = cudaMemcpyToSymbol(b2a::g_attn_trace_cta, v, sizeof(v));
  return e == cudaSuccess ? B2A_OK : cuda_fail(e);
}
__attribute__((visibility("default"))) int b2a_trace_read(unsigned long long* host) {
  cudaError_t e = cudaMemcpyFromSymbol(host, b2a::g_attn_trace, sizeof(b2a::g_attn_trace));
  return e == cudaSuccess ? B2A_OK : cuda_fail(e);
}
__attribute__((visibility("default"))) int b2a_trace_read_ns(unsigned long long* host) {
  cudaError_t e = cudaMemcpyFromSymbol(host, b2a::g_attn_trace_ns, sizeof(b2a::g_attn_trace_ns));
  return e == cudaSuccess ? B2A_OK : cuda_fail(e);
}
#endif

}  // extern "C"
