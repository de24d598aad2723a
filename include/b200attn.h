/*
 * b200attn -- non-causal long-sequence self-attention for NVIDIA B200 (sm_100a).
 *
 * C ABI of libb200attn.so.  Plain pointers and sizes only.
 *
 * Conventions for every entry point
 * ---------------------------------
 * - fp16 tensors are passed as uint16_t* holding IEEE binary16 bit patterns.
 * - "device" pointers must be CUDA device memory of the current device;
 *   "host" pointers are ordinary (preferably page-locked) host memory.
 * - Ownership: the caller owns every buffer.  The library allocates no
 *   device memory on any call path and keeps no pointer after a call returns
 *   (TMA descriptors are built per call).
 * - Asynchrony: work is enqueued on `stream` (a cudaStream_t passed as
 *   void*, NULL = the legacy default stream) and the call returns without
 *   waiting, except where stated.  Buffers must stay valid until the stream
 *   reaches the work.
 * - Errors: every entry point returns a b2a_status.  Arguments are checked
 *   before anything is enqueued; on B2A_ERR_INVALID_ARG or
 *   B2A_ERR_UNSUPPORTED nothing was enqueued and no output was touched.
 *   B2A_ERR_CUDA means a CUDA runtime call failed; b2a_last_cuda_error()
 *   returns its cudaError_t.  Kernels never trap: a device-side wait that
 *   runs out (a lost arrival) sets a device status word and the kernel
 *   returns; b2a_check_status() reports it as B2A_ERR_TIMEOUT.
 * - Batch is 1.  Token-major layouts follow the pages' (S, B, hidden)
 *   activations with B = 1 ("Multi-Device Attention Inference with
 *   TensorRT", Generating the ONNX Models).
 */
#ifndef B200ATTN_H
#define B200ATTN_H

#include <stdint.h>

#if defined(__GNUC__)
#define B2A_API __attribute__((visibility("default")))
#else
#define B2A_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  B2A_OK = 0,
  B2A_ERR_INVALID_ARG = 1, /* null/misaligned pointer, bad size, stride or scale */
  B2A_ERR_UNSUPPORTED = 2, /* not an sm_100 device, or a size beyond an implementation limit */
  B2A_ERR_CUDA = 3,        /* a CUDA runtime call failed; see b2a_last_cuda_error() */
  B2A_ERR_TIMEOUT = 4,     /* a kernel's bounded wait ran out (reported by b2a_check_status) */
  B2A_ERR_DEVICE_CHECK = 5 /* debug build: a device-side bounds check failed (reported by b2a_check_status) */
} b2a_status;

/*
 * attn_fwd -- monolithic non-causal scaled-dot-product attention.
 *
 * Per head h and query row i (every token attends to every token:
 * "Multi-Device Attention Inference with TensorRT", Introduction; per-head
 * attention: "Tensor Parallelism: Sharding Weights for Parallel Layer
 * Execution", section 3, step 3):
 *   out[i, h, :] = sum_j softmax_j(scale * q[i,h,:] . k[j,h,:]) * v[j, h, :]
 *   lse[h, i]    = ln sum_j exp(scale * q[i,h,:] . k[j,h,:])
 *
 * q, k, v   device fp16, row-major [S, H, d] with row strides ld_q, ld_k,
 *           ld_v elements (head h at columns h*d .. h*d+d-1 of a row); for
 *           views into a fused QKV buffer [S, 3*H*d] pass ld = 3*H*d.
 * out       device fp16 [S, H, d] with row stride ld_o.
 * lse       device fp32 [H, S] (natural log, scale included); may be NULL.
 * S >= 1, H >= 1, d in {64, 128}, scale > 0 and finite.
 * Every ld >= H*d and a multiple of 8; every pointer 16-byte aligned.
 * Arithmetic: fp16 products, fp32 accumulation and softmax, P rounded to
 * fp16 for the P.V product, output rounded once to fp16.
 */
B2A_API int attn_fwd(const uint16_t* q, const uint16_t* k, const uint16_t* v, uint16_t* out, float* lse,
             int S, int H, int d, float scale, int ld_q, int ld_k, int ld_v, int ld_o, void* stream);

/*
 * attn_fwd_batched -- attn_fwd over a batch in the pages' (S, B, hidden)
 * activation layout ("Multi-Device Attention Inference with TensorRT",
 * Generating the ONNX Models: input/output (sequence_length, batch_size,
 * 4096)).  Batch b is the strided view that starts at column b*H*d with row
 * stride B*H*d.  Heads of different batches are independent, so [S, B, H, d]
 * is taken as [S, B*H, d] (batch b's head h = head b*H + h, lse [B*H, S]) and
 * one launch covers every (row block, head, batch).  Results equal attn_fwd
 * on each batch's view, bit for bit.
 *
 * q, k, v, out  device fp16 [S, B, H, d] contiguous.
 * lse           device fp32 [B, H, S], or NULL.
 * B >= 1, B*H <= 65535 and B*H*d <= 2^31 - 1; other requirements as attn_fwd.
 */
B2A_API int attn_fwd_batched(const uint16_t* q, const uint16_t* k, const uint16_t* v, uint16_t* out,
                             float* lse, int S, int B, int H, int d, float scale, void* stream);

/*
 * attn_fwd_gathered_kv -- attn_fwd for Sq query rows against Skv keys: the
 * attention one rank computes in the AllGather-KV form of context
 * parallelism, where each rank keeps its own chunk of query rows and
 * gathers K and V from all ranks before attention (TensorRT 11.0
 * multi-device article, the three context-parallel implementations,
 * AllGather-KV; the sample's sharding hint gathers K/V and keeps Q local:
 * "Multi-Device Attention Inference with TensorRT", What is hint.json?).
 *   out[i, h, :] = sum_j softmax_j(scale * q[i,h,:] . k[j,h,:]) * v[j, h, :]
 *   lse[h, i]    = ln sum_j exp(scale * q[i,h,:] . k[j,h,:])
 *
 * q    device fp16 [Sq, H, d], row stride ld_q.
 * k, v device fp16 [Skv, H, d], row strides ld_k, ld_v.
 * out  device fp16 [Sq, H, d], row stride ld_o;  lse fp32 [H, Sq] or NULL.
 * Sq >= 1, Skv >= 1; other requirements as attn_fwd (attn_fwd is the case
 * Sq = Skv = S).
 */
B2A_API int attn_fwd_gathered_kv(const uint16_t* q, const uint16_t* k, const uint16_t* v, uint16_t* out,
                                 float* lse, int Sq, int Skv, int H, int d, float scale, int ld_q, int ld_k,
                                 int ld_v, int ld_o, void* stream);

/*
 * attn_fwd_partial -- attention of all queries against one contiguous chunk
 * of keys, the per-step work of ring attention (TensorRT 11.0 multi-device
 * article, the three context-parallel implementations, Ring Attention).
 *
 *   o_part[i, h, :] = softmax over the chunk's keys only, times their values
 *   lse_part[h, i]  = ln sum_{j in chunk} exp(scale * q_i . k_j)
 *
 * q         device fp16 [Sq, H, d], row stride ld_q.
 * k_chunk,
 * v_chunk   device fp16 [Skv, H, d], row stride ld_kv (pointer offsets into
 *           the full K/V give the chunk; chunk p of P is conventionally keys
 *           [floor(p*S/P), floor((p+1)*S/P))).
 * o_part    device fp32 [Sq, H, d], contiguous (normalised by the chunk's
 *           own sum).
 * lse_part  device fp32 [H, Sq].
 * Sq >= 1, Skv >= 0: an empty chunk writes o_part = 0 and lse_part = -inf.
 * Other requirements as attn_fwd.
 */
B2A_API int attn_fwd_partial(const uint16_t* q, const uint16_t* k_chunk, const uint16_t* v_chunk,
                     float* o_part, float* lse_part, int Sq, int Skv, int H, int d, float scale,
                     int ld_q, int ld_kv, void* stream);

/*
 * attn_fwd_partial_f16 -- attn_fwd_partial with the partial output stored in
 * fp16: the "FP16 split-reduction" that the accuracy table of "TensorRT
 * Multi-Device (multi-GPU) support" (Validation) names as the source of its
 * multi-device error.  o_part = round_fp16(o_c) where o_c is the chunk's
 * normalised output computed in fp32; lse_part stays fp32.  Half the bytes
 * of attn_fwd_partial's o_part, which attn_merge_f16 reads back.
 *
 * o_part    device fp16 [Sq, H, d], contiguous, 16-byte aligned.
 * Every other argument, the empty chunk (o_part = 0, lse_part = -inf) and
 * the error behaviour as attn_fwd_partial.
 */
B2A_API int attn_fwd_partial_f16(const uint16_t* q, const uint16_t* k_chunk, const uint16_t* v_chunk,
                                 uint16_t* o_part, float* lse_part, int Sq, int Skv, int H, int d, float scale,
                                 int ld_q, int ld_kv, void* stream);

/*
 * attn_fwd_partials -- every key chunk's partial in one call: for c < P,
 * chunk c = keys [floor(c*Skv/P), floor((c+1)*Skv/P)) of k, v, and
 * (o_parts[c], lse_parts[c]) is what attn_fwd_partial returns for that
 * chunk (the one-device form of ring attention's per-chunk partials, TensorRT
 * 11.0 multi-device article, Ring Attention), bit for bit.  Chunks short
 * enough for the single-CTA kernel (see b2a_set_attn_kernel) run as one
 * launch over (row block, chunk, head), the chunk varying fastest so that
 * the CTAs running at once share their Q tiles and K/V in L2; longer chunks
 * run one CTA-pair launch each.
 *
 * q          device fp16 [Sq, H, d], row stride ld_q.
 * k, v       device fp16 [Skv, H, d], row stride ld_kv (all keys).
 * o_parts    device fp32 [P, Sq, H, d] contiguous, 16-byte aligned.
 * lse_parts  device fp32 [P, H, Sq] contiguous.
 * P >= 1; Skv >= 0 (empty chunks give o = 0, lse = -inf); other
 * requirements and errors as attn_fwd_partial.
 */
B2A_API int attn_fwd_partials(const uint16_t* q, const uint16_t* k, const uint16_t* v, float* o_parts,
                              float* lse_parts, int Sq, int Skv, int P, int H, int d, float scale, int ld_q,
                              int ld_kv, void* stream);

/* attn_fwd_partials with fp16 o_parts ([P, Sq, H, d]; attn_fwd_partial_f16 per chunk). */
B2A_API int attn_fwd_partials_f16(const uint16_t* q, const uint16_t* k, const uint16_t* v, uint16_t* o_parts,
                                  float* lse_parts, int Sq, int Skv, int P, int H, int d, float scale, int ld_q,
                                  int ld_kv, void* stream);

/*
 * attn_fwd_accumulate -- one ring-attention step in place: fold the keys of
 * one chunk into a running result, the way each rank of ring attention
 * updates its output as K/V blocks arrive (TensorRT 11.0 multi-device
 * article, the three context-parallel implementations, Ring Attention: an
 * online softmax over the streamed K/V blocks).  With (o_c, lse_c) the
 * chunk's attn_fwd_partial result:
 *   lse_new = ln(exp(lse_acc) + exp(lse_c))
 *   o_new   = exp(lse_acc - lse_new) * o_acc + exp(lse_c - lse_new) * o_c
 * computed in the kernel's epilogue without writing o_c anywhere.
 *
 * q, k_chunk, v_chunk, Sq, Skv, H, d, scale, ld_q, ld_kv: as attn_fwd_partial.
 * o_acc    device fp32 [Sq, H, d] contiguous, read and written in place.
 * lse_acc  device fp32 [H, Sq], read and written in place (natural log).
 *          -inf marks a row that has seen no key yet: its o_acc is then
 *          ignored (it may hold anything) and replaced by o_c.  Start a ring
 *          pass with lse_acc = -inf; o_acc needs no initialisation.
 * out      device fp16 [Sq, H, d] contiguous, or NULL.  When given it also
 *          receives the fp16 rounding of o_new (pass it on the last step).
 *          Rows that have seen no key get 0.
 * Skv == 0 leaves o_acc and lse_acc unchanged (and still writes out).
 * After the last of P steps over the chunks of attn_fwd_partial, o_acc and
 * lse_acc equal attn_merge's result before its fp16 rounding.
 */
B2A_API int attn_fwd_accumulate(const uint16_t* q, const uint16_t* k_chunk, const uint16_t* v_chunk,
                                float* o_acc, float* lse_acc, uint16_t* out, int Sq, int Skv, int H, int d,
                                float scale, int ld_q, int ld_kv, void* stream);

/*
 * attn_merge -- exact merge of P chunk partials (ring attention's
 * online-softmax combine; the "split-reduction" of the accuracy table in
 * "TensorRT Multi-Device (multi-GPU) support", Validation):
 *   L = max_p lse_p;  lse = L + ln sum_p exp(lse_p - L)
 *   out = sum_p exp(lse_p - lse) * o_p        (chunks with lse_p = -inf add 0)
 *
 * o_parts    device fp32 [P, S, H, d] contiguous (chunk p's o_part at
 *            offset p*S*H*d).
 * lse_parts  device fp32 [P, H, S] contiguous.
 * out        device fp16 [S, H, d] contiguous.
 * lse_out    device fp32 [H, S]; may be NULL.
 * 1 <= P <= 64 (B2A_ERR_UNSUPPORTED above), S >= 1, H >= 1, d in {64, 128}.
 */
B2A_API int attn_merge(const float* o_parts, const float* lse_parts, int P, uint16_t* out, float* lse_out,
               int S, int H, int d, void* stream);

/*
 * attn_merge_f16 -- attn_merge over fp16 partials (attn_fwd_partial_f16's
 * o_part): the same weights and lse in fp32, the partial values widened to
 * fp32 before the weighted sum, one rounding of the result to fp16.
 *
 * o_parts    device fp16 [P, S, H, d] contiguous, 16-byte aligned.
 * Every other argument and the error behaviour as attn_merge.
 */
B2A_API int attn_merge_f16(const uint16_t* o_parts, const float* lse_parts, int P, uint16_t* out,
                           float* lse_out, int S, int H, int d, void* stream);

/*
 * qkv_proj -- fused Q/K/V projection qkv = x * w_qkv^T ("Tensor Parallelism:
 * Sharding Weights for Parallel Layer Execution", section 3, step 1:
 * Q = X W_Q, K = X W_K, V = X W_V, here as one weight).
 *
 * x      device fp16 [M, K] row-major.
 * w_qkv  device fp16 [N, K] row-major ([out, in]); N = 3*H*d with rows
 *        [W_Q; W_K; W_V], each head-major.
 * qkv    device fp16 [M, N] row-major.
 * M, N, K >= 1; N and K multiples of 8; pointers 16-byte aligned.
 * fp32 accumulation, one rounding to fp16.
 */
B2A_API int qkv_proj(const uint16_t* x, const uint16_t* w_qkv, uint16_t* qkv, int M, int N, int K,
             void* stream);

/*
 * qkv_proj_qknorm -- qkv_proj with the block's RMSNorm applied to q and k.
 *
 * The sample's block names an RMSNorm among its layers, after the Q/K/V
 * projections and before the attention ("Multi-Device Attention Inference
 * with TensorRT", Generating the ONNX Models), without placement or epsilon;
 * the reading taken here normalises every head of q and of k after the
 * projection, in the GEMM's epilogue from the fp32 accumulator:
 *   q[i, h, :] <- q[i, h, :] / sqrt(mean_e q[i, h, e]^2 + eps) * g_q
 *   k[i, h, :] <- k[i, h, :] / sqrt(mean_e k[i, h, e]^2 + eps) * g_k
 * v is stored as projected; each value is rounded once to fp16.
 *
 * x      device fp16 [M, K];  w_qkv device fp16 [3*H*d, K] ([out, in]).
 * g_q,
 * g_k    device fp16 [d] per-feature weights (shared by the heads), 16-byte
 *        aligned.
 * qkv    device fp16 [M, 3*H*d] (columns [q | k | v], head-major).
 * d in {64, 128}, H >= 1, eps >= 0 and finite (1e-6 is the usual choice);
 * other requirements as qkv_proj.
 */
B2A_API int qkv_proj_qknorm(const uint16_t* x, const uint16_t* w_qkv, const uint16_t* g_q,
                            const uint16_t* g_k, uint16_t* qkv, int M, int H, int d, int K, float eps,
                            void* stream);

/*
 * out_proj -- output projection with residual, y = residual + a * w_o^T
 * (section 3, step 4 of the same lesson: Z = Concat(heads) W_O; the block
 * adds its input back).  The residual is added to the fp32 accumulator and
 * the sum is rounded once to fp16.
 *
 * a         device fp16 [M, K] (the concatenated head outputs).
 * w_o       device fp16 [N, K] ([out, in]).
 * residual  device fp16 [M, N] or NULL (then y = a * w_o^T); may equal y.
 * y         device fp16 [M, N].
 * Requirements as qkv_proj.
 */
B2A_API int out_proj(const uint16_t* a, const uint16_t* w_o, const uint16_t* residual, uint16_t* y, int M,
             int N, int K, void* stream);

/*
 * attn_block_fwd -- one self-attention block of the stacked model:
 *   qkv = x * w_qkv^T;  a = attention(q, k, v) per head;  y = x + a * w_o^T
 * (the sample's block of Q/K/V projections, scaled dot-product attention and
 * output projection: "Multi-Device Attention Inference with TensorRT",
 * Generating the ONNX Models; six of them stacked: "TensorRT Multi-Device
 * (multi-GPU) support", Validation, multi-layer model).  Runs qkv_proj,
 * attn_fwd on strided views of qkv (ld = 3*H*d) and out_proj with the
 * residual, in that order on `stream`.
 *
 * x        device fp16 [S, H*d] (block input; also the residual).
 * w_qkv    device fp16 [3*H*d, H*d] ([out, in]; rows [W_Q; W_K; W_V]).
 * w_o      device fp16 [H*d, H*d] ([out, in]).
 * y        device fp16 [S, H*d]; may equal x (in-place block).
 * qkv_ws   device fp16 [S, 3*H*d] workspace (holds q|k|v after the call).
 * attn_ws  device fp16 [S, H*d] workspace (holds the attention output).
 * Requirements as attn_fwd and qkv_proj; workspaces must not overlap x, y
 * or each other.
 */
B2A_API int attn_block_fwd(const uint16_t* x, const uint16_t* w_qkv, const uint16_t* w_o, uint16_t* y,
                           uint16_t* qkv_ws, uint16_t* attn_ws, int S, int H, int d, float scale,
                           void* stream);

/*
 * attn_block_fwd_qknorm -- attn_block_fwd with qkv_proj_qknorm as its first
 * step (g_q, g_k, eps as there; both NULL: exactly attn_block_fwd).
 */
B2A_API int attn_block_fwd_qknorm(const uint16_t* x, const uint16_t* w_qkv, const uint16_t* g_q,
                                  const uint16_t* g_k, float eps, const uint16_t* w_o, uint16_t* y,
                                  uint16_t* qkv_ws, uint16_t* attn_ws, int S, int H, int d, float scale,
                                  void* stream);

/*
 * attn_block_fwd_static -- attn_block_fwd for callers that cannot allocate.
 *
 * The pages have no counterpart to this entry point; it exists for users of
 * the library.  Some callers cannot call cudaMalloc (or any allocator) on
 * their inference path: a host application or plugin framework that reserved
 * the GPU's memory up front and forbids further device allocations, code
 * that must not block or fail on an allocation in a latency-critical loop,
 * or a caller in another runtime that can hand over only its own input and
 * output buffers.  This variant computes exactly what attn_block_fwd does,
 * but keeps its two intermediates -- qkv [S, 3*H*d] and the attention output
 * [S, H*d], fp16, 8*S*H*d bytes together -- in one static device array of
 * 64 MiB inside the library instead of caller workspaces.  It calls no
 * allocator.
 *
 * x, w_qkv, w_o, y, S, H, d, scale, stream: as attn_block_fwd (y may equal x).
 * Limit: S*H*d <= 8388608 (e.g. S = 2048 at hidden 4096); larger sizes
 * return B2A_ERR_UNSUPPORTED before anything is enqueued.
 * Memory: every GPU that loads the library holds the 64 MiB array until the
 * process exits.
 * First call: the first call on a device looks up the array's address on
 * that device (cudaGetSymbolAddress), so make it before any stream capture.
 * Sharing: every call uses the same array, and it keeps the last call's
 * contents.  Calls that can overlap on the GPU (other streams, other host
 * threads) race on it; the caller must order them.  Nothing in the array
 * needs to start at zero: each call writes both intermediates in full
 * before reading them.
 */
B2A_API int attn_block_fwd_static(const uint16_t* x, const uint16_t* w_qkv, const uint16_t* w_o,
                                  uint16_t* y, int S, int H, int d, float scale, void* stream);

/*
 * attn_fwd_host -- attention end to end from host memory.
 *
 * Copies q, k, v (host fp16 [S, H, d] contiguous) into the caller's device
 * workspace, runs attn_fwd (P == 1) or P attn_fwd_partial calls plus
 * attn_merge (P > 1, the one-device emulation of ring attention), and copies
 * out (host fp16 [S, H, d]) and lse (host fp32 [H, S], may be NULL) back.
 * The copies run on two copy streams the library creates on first use per
 * device (one per direction) so that they overlap the kernels: with P = 1
 * and S >= 4096 the query rows go in 4 blocks (block b's copy-in, attention
 * and copy-out overlap the others; K and V are copied first), with P > 1
 * each key chunk's copy overlaps the previous chunk's partial.  Events order
 * every step after the work already on `stream` and make `stream` wait for
 * the last copy-out, so to the caller the call behaves as if enqueued on
 * `stream`.  The call returns after enqueueing: host buffers must stay valid
 * until the stream is synchronised.  Page-locked host buffers are needed for
 * the copies to be asynchronous.  Calls from several host threads on one
 * device are serialised while they enqueue.
 *
 * workspace        device memory of at least attn_fwd_host_workspace_bytes(S,H,d,P)
 *                  bytes, 256-byte aligned.
 * workspace_bytes  its size (checked).
 * 1 <= P <= 64; other requirements as attn_fwd.
 */
B2A_API int attn_fwd_host(const uint16_t* q, const uint16_t* k, const uint16_t* v, uint16_t* out,
                  float* lse, int S, int H, int d, float scale, int P, void* workspace,
                  uint64_t workspace_bytes, void* stream);

/* Device workspace attn_fwd_host needs; 0 for invalid sizes. */
B2A_API uint64_t attn_fwd_host_workspace_bytes(int S, int H, int d, int P);

/*
 * b2a_check_status -- synchronise `stream`, then read and clear the device
 * status word that kernels set when a bounded wait runs out or, in the
 * debug build, when a bounds check fails.  Returns B2A_OK,
 * B2A_ERR_DEVICE_CHECK (a bounds check failed; waits that then gave up are
 * its consequence), B2A_ERR_TIMEOUT, or B2A_ERR_CUDA if the synchronisation
 * failed.  Blocks the calling host thread.
 */
B2A_API int b2a_check_status(void* stream);

/*
 * b2a_selftest_wait_timeout -- exercise the failure path without a fault.
 *
 * Launches one small kernel on `stream` whose bounded wait (the same code
 * every kernel here uses for its mbarrier waits) waits on a barrier that
 * nothing arrives on.  After limit_ms (1..2000) the wait gives up and sets
 * the device status word, as a lost arrival would; the next
 * b2a_check_status() returns B2A_ERR_TIMEOUT and clears it.  Until then,
 * kernels launched afterwards give up at their first wait that does not
 * complete at once.  result: device int[2], set to {1, 1} when the expired
 * wait reported failure and a completed wait (checked alongside) reported
 * success.  The pages have no counterpart; this is for testing callers'
 * error handling.
 */
B2A_API int b2a_selftest_wait_timeout(int limit_ms, int* result, void* stream);

/* Static text for a b2a_status value. */
B2A_API const char* b2a_status_string(int status);

/* cudaError_t of the most recent failed CUDA call in this thread (0 if none). */
B2A_API int b2a_last_cuda_error(void);

/*
 * b2a_set_attn_kernel / b2a_get_attn_kernel -- which attention kernel the
 * attention entry points (attn_fwd, attn_fwd_partial, attn_fwd_accumulate,
 * and those built on them) use for head dim 128.  The pages have no
 * counterpart; this is a tuning and testing control.
 *   B2A_ATTN_KERNEL_AUTO    (default) CTA pairs when the call has at least
 *                           48 key tiles of 128 (Skv > 6016), else single CTAs
 *   B2A_ATTN_KERNEL_SINGLE  single CTAs, two 128-row query tiles each
 *   B2A_ATTN_KERNEL_PAIR    two-SM CTA pairs issuing M = 256 MMAs
 * Both compute the same result (the same arithmetic in the same order per
 * row).  Head dim 64 always uses single CTAs.  Process-wide; takes effect
 * for calls made after it returns.  Returns B2A_ERR_INVALID_ARG for any
 * other value.
 */
enum { B2A_ATTN_KERNEL_AUTO = 0, B2A_ATTN_KERNEL_SINGLE = 1, B2A_ATTN_KERNEL_PAIR = 2 };
B2A_API int b2a_set_attn_kernel(int choice);
B2A_API int b2a_get_attn_kernel(void);
/* The kernel a call with head dim d and Skv keys would use now:
   B2A_ATTN_KERNEL_SINGLE or B2A_ATTN_KERNEL_PAIR. */
B2A_API int b2a_attn_kernel_for(int d, int Skv);

/* Library ABI version (major*100 + minor). */
/*
 * b2a_debug_build -- 1 if this library is the debug build
 * (libb200attn_debug.so, compiled with -DB2A_DEBUG), else 0.  The pages have
 * no counterpart: the debug build is this library's stand-in for a memory
 * checker.  Before every tiled TMA copy it checks the box's start against
 * the tensor map's extents (the innermost coordinate also for 16-byte
 * alignment) and the destination against the CTA's shared memory; before
 * every tcgen05.ld / tcgen05.st / tcgen05.mma it checks the TMEM lane field
 * and columns against the 512-column allocation.  A failed check skips the
 * access, ORs a bit into the device status word (the kernel's waits then give
 * up at once and it returns) and b2a_check_status() returns
 * B2A_ERR_DEVICE_CHECK.  Same entry points and results as the release build,
 * slower.
 */
B2A_API int b2a_debug_build(void);

B2A_API int b2a_version(void);

#ifdef __cplusplus
}
#endif

#endif /* B200ATTN_H */
