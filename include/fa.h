/*
 * fa.h - C ABI of libfa.so: exact fused attention (FlashAttention forward and backward)
 * for NVIDIA B200 (sm_100a).
 *
 * What is computed.  For every (batch b, head h) pair, with Q, K, V the N x d matrices of
 * that head:
 *     S = scale * Q K^T                 (scaled scores; "xinc.fun archive 235", section 6
 *                                        标准注意力为什么慢)
 *     P = softmax(S) row-wise,  O = P V (exact attention; same section, and "Flash
 *                                        Attention" on special-jiahao.github.io, section
 *                                        Standard Attention)
 * computed tile by tile with a running row max, denominator and unnormalised accumulator
 * (the online softmax of "xinc.fun archive 235", section 7, a whole key block per step), so
 * that S and P never reach device memory.  The forward also saves, per query row, the
 * natural-log log-sum-exp of the scaled scores, LSE_i = ln sum_j exp(S_ij).  The backward
 * recomputes S and P tile by tile from Q, K and LSE (same section: "recompute local scores
 * from the saved inputs and a few statistics") and returns
 *     dV = P^T dO,  dP = dO V^T,  D_i = rowsum(dO o O) = rowsum(P o dP),
 *     dS = P o (dP - D_i),  dQ = scale * dS K,  dK = scale * dS^T Q.
 * With causal != 0, key j is visible to query i only when j <= i (square self-attention).
 *
 * Layout.  Q, K, V, O, dO, dQ, dK, dV are bf16 tensors [B, H, N, d], contiguous
 * (row-major: d fastest, then N, then H, then B).  LSE is fp32 [B, H, N], contiguous.
 * Supported: d in {64, 128} for the forward and the backward; N >= 0;
 * B * H * N * d < 2^62.  B, H or N equal to 0 is an empty problem: the call returns FA_OK
 * without launching anything.
 *
 * Ownership and memory.  Every pointer is a device pointer owned by the caller; the
 * library allocates no device memory per call.  Tensors handed to a TMA unit must start on
 * a 16-byte boundary (q, k, v, o, dO, dq, dk, dv); lse, dQ-workspace need 4-byte alignment.
 * Outputs are fully overwritten (the backward's dq, dk, dv are not accumulated into).
 * The only state kept by the library: per-device kernel attributes, set on first use, and
 * one device status word (see fa_get_device_status).
 *
 * Streams and errors.  stream is a cudaStream_t passed as void* (NULL = legacy default
 * stream).  Calls are asynchronous on that stream.  Argument errors are detected on the
 * host before any launch and returned synchronously: FA_ERR_INVALID_ARG (null pointer,
 * negative size, misalignment, non-finite or non-positive scale, causal not 0/1, workspace
 * too small, size overflow) or FA_ERR_UNSUPPORTED (head dimension, or a device that is not
 * sm_100).  A failed launch returns FA_ERR_CUDA.  Every wait inside a kernel is bounded;
 * a wait that runs out sets a bit in the device status word and the kernel exits early
 * (its outputs are then undefined); fa_get_device_status reports that as FA_ERR_TIMEOUT.
 * No C++ exception crosses this interface.
 */
#ifndef FA_H_
#define FA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  FA_OK = 0,
  FA_ERR_INVALID_ARG = 1,
  FA_ERR_UNSUPPORTED = 2,
  FA_ERR_CUDA = 3,
  FA_ERR_TIMEOUT = 4,
  FA_ERR_DEVICE_CHECK = 5
} fa_status_t;

/*
 * Forward pass ("xinc.fun archive 235", sections 6-7).
 *   q, k, v : in,  bf16 [B,H,N,d]
 *   o       : out, bf16 [B,H,N,d]   O = softmax(scale * Q K^T [masked]) V, rounded to bf16
 *   lse     : out, fp32 [B,H,N]     natural-log log-sum-exp of each row of the scaled,
 *                                   masked scores (-inf for a row with no visible key)
 *   scale   : finite, > 0 (1/sqrt(d) for standard attention)
 *   causal  : 0 or 1
 */
fa_status_t fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
                   int B, int H, int N, int d, float scale, int causal, void* stream);

/*
 * Forward pass split over the key range (split-KV), for problems too small to fill the GPU
 * (few heads or few query rows against many keys).  Each (head, 256 query rows) work item is
 * divided into num_splits contiguous ranges of 128-key blocks; every range yields the
 * normalised partial output O_s (fp32) and its LSE_s, and a second kernel combines them with
 * the two-block softmax merge of "Flash Attention" (special-jiahao.github.io, section 增量求解
 * softmax) extended to num_splits blocks:
 *     M = max_s LSE_s,  w_s = exp(LSE_s - M),  O = sum_s w_s O_s / sum_s w_s,
 *     LSE = M + ln sum_s w_s.
 * The result equals fa_fwd's up to rounding.  Arguments as in fa_fwd, plus:
 *   num_splits      : >= 1, or <= 0 for fa_fwd_splitkv_default_splits(...); values above the
 *                     number of 128-key blocks are clamped to it.  1 runs fa_fwd itself.
 *   workspace       : device scratch, 256-byte aligned, at least
 *                     fa_fwd_splitkv_workspace_bytes(B,H,N,d,splits) bytes for the number of
 *                     splits used (not needed, may be NULL, when that number is 1).
 *
 * fa_fwd_splitkv_default_splits returns the split count (1-4) that the library would choose:
 * it simulates the grid's makespan on the current device's SMs (CTAs in launch order to the
 * first free SM) for 1-4 splits and splits only when that predicts a gain of at least 1.25
 * (the partial outputs and the merge cost the rest), which in practice means causal, long
 * sequences over few heads.  Host-only; without a CUDA device it assumes 148 SMs.
 */
int fa_fwd_splitkv_default_splits(int B, int H, int N, int d, int causal);
size_t fa_fwd_splitkv_workspace_bytes(int B, int H, int N, int d, int num_splits);
fa_status_t fa_fwd_splitkv(const void* q, const void* k, const void* v, void* o, float* lse,
                           int B, int H, int N, int d, float scale, int causal, int num_splits,
                           void* workspace, size_t workspace_bytes, void* stream);

/*
 * Forward pass with FP8 operands for both tile GEMMs ("xinc.fun archive 235", section 4: matmuls
 * in a low-precision format, accumulation and softmax kept at higher precision).
 *   q, k, v   : in,  E4M3 (1 byte per element) [B,H,N,d]; the values are x * descale
 *   descale_q, descale_k, descale_v
 *             : in,  fp32 [B*H] per-(b,h) dequantisation factors (index b*H + h), or NULL
 *               for 1.0 each
 *   o, lse, scale, causal : as for fa_fwd; O = softmax(scale * Q K^T [masked]) V of the
 *               dequantised values
 * S = Q K^T and O += P V run as E4M3 x E4M3 -> fp32 MMAs; P (scaled by 2^8, so that it spans
 * E4M3's range) is rounded to E4M3 for the PV product, while the row sums and the normaliser
 * use the unrounded fp32 P.  Each element of O is then within 2^-4 * max|v| (P's rounding)
 * plus bf16 output rounding of the exact attention of the dequantised inputs.
 * Supported: d == 128.  Same layout, alignment (16 bytes for q, k, v, o; 4 for lse and the
 * descale arrays), error and empty-problem rules as fa_fwd.
 */
fa_status_t fa_fwd_fp8(const void* q, const void* k, const void* v, const float* descale_q,
                       const float* descale_k, const float* descale_v, void* o, float* lse,
                       int B, int H, int N, int d, float scale, int causal, void* stream);

/*
 * The two halves of the split-KV forward, for callers that hold the keys in pieces (for
 * instance one piece per GPU of a sequence sharded across GPUs).
 *
 * fa_fwd_partial: attention of q over one set of keys k, v (all [B,H,N,d] bf16, the same N),
 * returned as that key set's normalised partial result:
 *   o_part   : out, fp32 [B,H,N,d]  O_s = softmax over these keys of scale * Q K^T, times V
 *   lse_part : out, fp32 [B,H,N]    LSE_s, natural log (-inf for a row with no visible key)
 * causal != 0 masks key j for query i when j > i within this key set (the diagonal piece);
 * causal == 0 sees every key (a piece that lies entirely before the queries).  Alignment as
 * fa_fwd, o_part 16 bytes.
 *
 * fa_merge_partials: combines nparts such results of the same queries with the two-block
 * softmax merge of "Flash Attention" (special-jiahao.github.io, section 增量求解 softmax)
 * extended to nparts blocks (M = max_s LSE_s, w_s = exp(LSE_s - M), O = sum_s w_s O_s / sum_s
 * w_s, LSE = M + ln sum_s w_s; parts with LSE_s = -inf contribute nothing):
 *   o_parts   : in, fp32 [nparts,B,H,N,d] contiguous (16-byte aligned)
 *   lse_parts : in, fp32 [nparts,B,H,N]
 *   o, lse    : out, bf16 [B,H,N,d] (16-byte aligned) and fp32 [B,H,N]
 *   nparts    : 1 .. 1024.  d in {64, 128}.
 */
fa_status_t fa_fwd_partial(const void* q, const void* k, const void* v, float* o_part,
                           float* lse_part, int B, int H, int N, int d, float scale, int causal,
                           void* stream);
fa_status_t fa_merge_partials(const float* o_parts, const float* lse_parts, int nparts, void* o,
                              float* lse, int B, int H, int N, int d, void* stream);

/*
 * The same pieces combined as they come, without one partial result per piece: attention of q
 * over one more set of keys k, v (all [B,H,N,d] bf16, the same N; causal as fa_fwd_partial),
 * folded into a running partial result of these queries over the key sets seen before.  The
 * running result (o_part fp32 [B,H,N,d], lse_part fp32 [B,H,N], fa_fwd_partial's format) is
 * the state the kernel starts from: each row's LSE is its softmax reference, its sum relative to
 * that reference is 1 and its output starts as o_part's row, and the key blocks of this set then
 * update them exactly as blocks of one longer key range would ("Flash Attention",
 * special-jiahao.github.io, section 增量求解 softmax: block results rescaled to a common
 * reference and added).
 *   flags & FA_CARRY_IN    : (o_part, lse_part) hold the running result, read first (rows with
 *                            LSE = -inf have seen no key); without it the running result is
 *                            empty and their contents do not matter
 *   flags & FA_CARRY_FINAL : the result goes to o (bf16 [B,H,N,d], 16-byte aligned) and lse
 *                            (fp32 [B,H,N], natural log), as fa_fwd writes them; without it it
 *                            is written back into (o_part, lse_part), in place
 * Calls for one set of queries run in order on one stream.  fa_fwd_carry over key sets 1..P,
 * the first without FA_CARRY_IN and the last with FA_CARRY_FINAL, gives what fa_fwd over the
 * concatenated keys gives (up to rounding order); memory is one running result whatever P is.
 * d in {64, 128}; alignment as fa_fwd_partial; other flag bits return FA_ERR_INVALID_ARG.
 */
#define FA_CARRY_IN 1
#define FA_CARRY_FINAL 2
fa_status_t fa_fwd_carry(const void* q, const void* k, const void* v, float* o_part, float* lse_part,
                         void* o, float* lse, int B, int H, int N, int d, float scale, int causal,
                         int flags, void* stream);

/*
 * Bytes of device workspace that fa_bwd needs: per 64-row query tile, the fp32 base-2 LSE and
 * row term D_i of its 64 rows (B*H*ceil(N/64)*128 floats, rounded up to 256 bytes), followed
 * by the fp32 dQ accumulator [B*H*N*d] and a 256-byte block holding the work counter of the
 * persistent key-tile kernel.  Returns 0 for an empty or invalid shape.
 */
size_t fa_bwd_workspace_bytes(int B, int H, int N, int d);

/*
 * Backward pass (recomputation, "xinc.fun archive 235", section 7; formulas above).
 *   q, k, v, o, dO : in,  bf16 [B,H,N,d]  (o is the forward's output)
 *   lse            : in,  fp32 [B,H,N]    (the forward's lse)
 *   dq, dk, dv     : out, bf16 [B,H,N,d]
 *   workspace      : device scratch of at least fa_bwd_workspace_bytes(B,H,N,d) bytes,
 *                    256-byte aligned; its contents on entry do not matter and on exit
 *                    are unspecified.  Concurrent calls need distinct workspaces.
 * dQ is summed over key tiles with fp32 reductions (dK, dV in a fixed order), at both head
 * dimensions; fa_bwd_deterministic gives a dQ summed in a fixed order instead.
 */
fa_status_t fa_bwd(const void* q, const void* k, const void* v, const void* o,
                   const void* dO, const float* lse, void* dq, void* dk, void* dv,
                   void* workspace, size_t workspace_bytes,
                   int B, int H, int N, int d, float scale, int causal, void* stream);

/*
 * Size of the scratch array that fa_bwd_noalloc uses in place of a workspace: 64 MiB, held in
 * device memory on every GPU that has loaded the library, for as long as it stays loaded.
 */
#define FA_BWD_NOALLOC_MAX_SCRATCH_BYTES ((size_t)64 << 20)

/*
 * fa_bwd for callers that cannot allocate device memory.  (The pages have no counterpart: this
 * is an interface convenience, not part of the method.)
 *
 * Who needs it: code that runs inside a host framework owning all device memory and offering
 * its extensions no allocator, and hot paths whose rules forbid cudaMalloc (which can
 * synchronise the device).  Arguments and results are those of fa_bwd minus the workspace;
 * inputs and outputs are still the caller's buffers.  No memory is allocated by this call.
 *
 * Scratch: a fixed FA_BWD_NOALLOC_MAX_SCRATCH_BYTES array inside the library replaces the
 * workspace.  Problems whose fa_bwd_workspace_bytes(B,H,N,d) exceeds that size are refused with
 * FA_ERR_INVALID_ARG before any GPU work (at d = 128 this allows B*H*N up to about 129,000
 * query rows).  The first call on each device looks up the array's device address (a CUDA
 * runtime query) and caches it; make that first call before any stream capture on that device.
 * Every call shares the one array: calls that overlap on the GPU (other streams, other host
 * threads) race on it and must be serialised by the caller.  Each call rewrites the scratch it
 * reads, so leftovers from an earlier call do not affect results.
 */
fa_status_t fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* o,
                           const void* dO, const float* lse, void* dq, void* dk, void* dv,
                           int B, int H, int N, int d, float scale, int causal, void* stream);

/*
 * fa_bwd with a deterministic dQ: same arguments, workspace and results (within rounding), but
 * dQ is accumulated per 128-row query tile in a fixed order (a query-tile-outer pass that
 * recomputes S and dP and keeps dQ on chip until it is written once) instead of with
 * floating-point atomics, so repeated calls on the same inputs give bitwise-identical dQ, dK
 * and dV.  Supported: d in {64, 128}.
 */
fa_status_t fa_bwd_deterministic(const void* q, const void* k, const void* v, const void* o,
                                 const void* dO, const float* lse, void* dq, void* dk, void* dv,
                                 void* workspace, size_t workspace_bytes,
                                 int B, int H, int N, int d, float scale, int causal, void* stream);

/*
 * The backward in three steps, for callers that hold the keys in pieces (the sequence-sharded
 * backward: every key set's contribution is added in turn).  d in {64, 128}.  The workspace has
 * fa_bwd's layout and size; dk_acc, dv_acc are caller-owned fp32 [B,H,N,d] accumulators
 * (16-byte aligned) for the keys of one piece, zeroed by the caller before the first addition.
 *   fa_bwd_prepare    : from this rank's o, dO (bf16) and lse (fp32), the per-row statistics
 *                       (LSE * log2 e, D_i = rowsum(dO o O)) into the workspace, and its fp32
 *                       dQ accumulator zeroed.
 *   fa_bwd_accumulate : the contribution of one key set k, v (same N) to the gradients of these
 *                       queries: dQ added into the workspace's accumulator (fp32 reductions),
 *                       scale * dK and dV added into dk_acc and dv_acc.  causal != 0 applies the
 *                       mask within the key set (the diagonal piece); 0 sees every key.
 *   fa_bwd_finish     : dq = scale * accumulator, dk = dk_acc, dv = dv_acc, rounded to bf16.
 * Summed over all key sets, the results are fa_bwd's (up to summation order).
 */
fa_status_t fa_bwd_prepare(const void* o, const void* dO, const float* lse, void* workspace,
                           size_t workspace_bytes, int B, int H, int N, int d, void* stream);
fa_status_t fa_bwd_accumulate(const void* q, const void* k, const void* v, const void* dO,
                              void* workspace, size_t workspace_bytes, float* dk_acc,
                              float* dv_acc, int B, int H, int N, int d, float scale, int causal,
                              void* stream);
fa_status_t fa_bwd_finish(const void* workspace, size_t workspace_bytes, const float* dk_acc,
                          const float* dv_acc, void* dq, void* dk, void* dv,
                          int B, int H, int N, int d, float scale, void* stream);
/*
 * fa_bwd_accumulate with the key set's contribution stored instead of added: dk_out = scale *
 * dK and dv_out = dV of this key set alone (fp32 [B,H,N,d], 16-byte aligned, every row
 * written), dQ still added into the workspace's accumulator.  The sequence-sharded backward
 * computes a passing key set's contribution this way while that key set's accumulators are
 * on their way, then adds it in with fa_bwd_acc_add.  Same arguments and error rules as
 * fa_bwd_accumulate.
 */
fa_status_t fa_bwd_contribute(const void* q, const void* k, const void* v, const void* dO,
                              void* workspace, size_t workspace_bytes, float* dk_out,
                              float* dv_out, int B, int H, int N, int d, float scale, int causal,
                              void* stream);

/*
 * acc += x, element by element, for two fp32 [B,H,N,d] accumulators (16-byte aligned, d in
 * {64, 128}): the sequence-sharded backward computes a key set's contribution into a zeroed
 * local pair while that key set's dK/dV accumulators are still arriving from the previous
 * rank, then adds it in with this call.  Same error rules as fa_bwd_finish.
 */
fa_status_t fa_bwd_acc_add(float* acc, const float* x, int B, int H, int N, int d, void* stream);

/*
 * fa_bwd taken apart into its three kernels, so that each can be launched, and
 * timed, on its own.  fa_bwd_prepare (above), then fa_bwd_main, then fa_bwd_dq_post, on one
 * stream and one workspace, give exactly what fa_bwd gives.
 *   fa_bwd_main    : the key-tile pass on prepared statistics: recomputes S and P tile by tile,
 *                    stores dk = scale * dS^T Q and dv = P^T dO (bf16 [B,H,N,d], 16-byte
 *                    aligned) and adds dS K into the workspace's fp32 dQ accumulator.
 *                    q, k, v, dO as for fa_bwd.
 *   fa_bwd_dq_post : dq = scale * accumulator, rounded to bf16 ([B,H,N,d], 16-byte aligned).
 * Same error rules as fa_bwd (d in {64, 128}).
 */
fa_status_t fa_bwd_main(const void* q, const void* k, const void* v, const void* dO,
                        void* workspace, size_t workspace_bytes, void* dk, void* dv,
                        int B, int H, int N, int d, float scale, int causal, void* stream);
fa_status_t fa_bwd_dq_post(const void* workspace, size_t workspace_bytes, void* dq,
                           int B, int H, int N, int d, float scale, void* stream);

/*
 * Synchronises `stream`, reads and clears the device status word of the current device.
 * Returns FA_ERR_TIMEOUT if a kernel's bounded wait ran out since the last call,
 * FA_ERR_DEVICE_CHECK if a device-side check failed (a full-TMEM allocation that did not start
 * at column 0, or, in the debug build, an index outside its range), FA_ERR_CUDA if the
 * synchronisation itself failed, FA_OK otherwise.
 */
fa_status_t fa_get_device_status(void* stream);

/*
 * Self-test of the bounded waits (failure detection; no counterpart on the pages).
 * Launches one CTA whose single thread waits on an mbarrier phase that nothing completes,
 * for at most limit_ms milliseconds (1..1000) of %globaltimer; the wait then runs out, the
 * kernel records the timeout in the device status word and exits normally (no trap, no
 * fault: the context stays usable).  A following fa_get_device_status(stream) returns
 * FA_ERR_TIMEOUT and clears the word.  Returns FA_ERR_INVALID_ARG for a limit out of range,
 * FA_ERR_CUDA if the launch fails.  Kernels launched while the timeout bit is set exit early,
 * so read the status before launching anything else.
 */
fa_status_t fa_selftest_wait_timeout(int limit_ms, void* stream);

/*
 * Debug build (libfa_debug.so: the same sources compiled with FA_DEBUG; no counterpart on the
 * pages, it stands in for a memory checker).  Its kernels check their tile indices and global
 * offsets on the device (a failed check skips the access and sets a status bit that
 * fa_get_device_status reports as FA_ERR_DEVICE_CHECK; nothing traps) and count the tile pairs
 * they visit, per kernel kind, in three blocks of 2^20 int counters kept by the library:
 *   block 0, forward kernel:           [B*H][ceil(N/128) query tiles][ceil(N/128) key blocks]
 *   block 1, backward key-tile kernel: [B*H][ceil(N/64) query tiles][ceil(N/128) key tiles]
 *   block 2, deterministic dQ kernel:  [B*H][ceil(N/128) query tiles][ceil(N/64) key blocks]
 * (row-major, one count per visit of the pair).
 * fa_debug_build      : 1 in the debug build, 0 in the release build.
 * fa_debug_visits     : synchronises `stream`, copies the first n counters (n <= 3 * 2^20,
 *                       block b starting at b * 2^20) to the host array `counts`, then zeroes
 *                       all of them when clear != 0.  FA_ERR_UNSUPPORTED in the release build.
 */
int fa_debug_build(void);
fa_status_t fa_debug_visits(int* counts, size_t n, int clear, void* stream);

/* Static, human-readable name of a status code. */
const char* fa_status_string(fa_status_t s);

/* Library version, major*10000 + minor*100 + patch. */
int fa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FA_H_ */
