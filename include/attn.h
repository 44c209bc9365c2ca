/*
 * attn.h — C ABI of the exact softmax attention library (libattn.so), sm_100a.
 *
 * Operation (all entry points):  O = softmax(scale * Q Kᵀ + mask) V, computed
 * tile by tile with an online softmax so the score matrix never reaches device
 * memory, plus the per-row natural log-sum-exp of the scaled, masked scores.
 *   - Plain definition: "Attention Is O(n²): FlashAttention vs Linear
 *     Attention", section "Why Attention Is O(n²)".
 *   - Tiled loop with running max / running sum / rescaled accumulator: same
 *     page, section "FlashAttention — Same FLOPs, Linear Memory"; the online
 *     softmax of "Modern Attention: MQA, GQA, FlashAttention, Sliding Window
 *     and RoPE", section 3.
 *   - Grouped-query heads: query head h reads K/V head h / (Hq / Hkv)
 *     ("Chapter 3: MHA Limitations, MQA, GQA, and FlashAttention", section 3.3).
 *   - Sliding window: "Modern Attention ...", section 4.
 *   - Decode over a KV cache, combined from key-split partial states by the
 *     merge rule of "Chapter 3 ...", section 3.5.
 *
 * Mask convention. Query row i sits at key position qpos(i) = i + Nk - Nq
 * (bottom-right alignment). Key j is allowed iff 0 <= j < Nk and
 *   j <= qpos(i)                  when causal != 0, and
 *   j >= qpos(i) - window_left    when window_left >= 0.
 * window_left counts keys strictly before the query's own position, so a
 * window of the "last W tokens" is window_left = W - 1. A negative
 * window_left means no window; a window without causal limits the left side
 * only. A row with no allowed key gets O = 0 and LSE = -inf.
 *
 * Layouts (row-major, contiguous, element strides implied by the shapes):
 *   Q, O : [B, Nq, Hq, d]      K, V : [B, Nk, Hkv, d]      LSE : [B, Hq, Nq]
 * Q/K/V are bfloat16; O is bfloat16 (attn_fwd) or float32 (attn_fwd_f32o);
 * LSE is float32 in natural-log units of the scaled scores.
 *
 * Ownership. The caller allocates and owns every buffer (device memory),
 * including the decode workspace; the library never allocates or frees device
 * memory (the one exception is the fixed scratch array of
 * attn_decode_noalloc, described there). All calls are asynchronous on `stream` (may be NULL = legacy default
 * stream) and never synchronise, except attn_device_status.
 *
 * Errors. Every entry point validates its arguments on the host first; on any
 * error it returns a non-zero attn_status, launches nothing, and records a
 * message readable with attn_last_error() (thread-local).
 *
 * Size limits (ATTN_ERR_INVALID_ARG beyond them): the kernels index rows and
 * positions in 32 bits, so B * Nq, B * Nk, B * Hq (and B * Lmax for decode)
 * stay below 2^31; a decode cache holds at most 2^31 - 128 keys; the backward
 * pass needs B * Nq * Hq * d <= 8 * (2^31 - 1); a decode workspace may not
 * exceed 2^62 bytes.
 */
#ifndef ATTN_H_
#define ATTN_H_

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  ATTN_OK = 0,
  ATTN_ERR_INVALID_ARG = 1,   /* null pointer, bad size, misalignment, Hq % Hkv != 0, ...;
                                 also from attn_device_status after a device-side input check */
  ATTN_ERR_UNSUPPORTED = 2,   /* device is not sm_100, or head dim not in {64, 128} */
  ATTN_ERR_CUDA = 3,          /* a CUDA runtime/driver call failed (message has the code) */
  ATTN_ERR_TIMEOUT = 4,       /* a bounded device-side wait gave up (see attn_device_status) */
  ATTN_ERR_WORKSPACE = 5,     /* decode or backward workspace missing or smaller than required */
  ATTN_ERR_INTERNAL = 6       /* bounds-checking debug build only: a kernel's index left its
                                 buffer or two of its roles disagreed on a protocol count; the
                                 access was skipped (see attn_debug_checks) */
} attn_status;

/*
 * Prefill / full forward pass, bf16 output.
 *   q   : device, bf16 [B, Nq, Hq, d], 16-byte aligned
 *   k,v : device, bf16 [B, Nk, Hkv, d], 16-byte aligned
 *   o   : device, bf16 [B, Nq, Hq, d], 16-byte aligned (written)
 *   lse : device, f32 [B, Hq, Nq], 4-byte aligned, or NULL (not written)
 *   B, Hq, Hkv, Nq, Nk >= 1; Hq % Hkv == 0; d in {64, 128}
 *   scale : finite, > 0 (usually 1/sqrt(d))
 *   causal : 0 or 1;  window_left : < 0 for none, else keys before the query
 * Returns ATTN_OK or an attn_status; nothing is launched on error.
 */
int attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
             int B, int Hq, int Hkv, int Nq, int Nk, int d, float scale,
             int causal, int window_left, cudaStream_t stream);

/* Same as attn_fwd, but o is float32 [B, Nq, Hq, d]. */
int attn_fwd_f32o(const void* q, const void* k, const void* v, float* o, float* lse,
                  int B, int Hq, int Hkv, int Nq, int Nk, int d, float scale,
                  int causal, int window_left, cudaStream_t stream);

/*
 * Forward pass over packed variable-length sequences (no padding): sequence b
 * owns query rows [cu_seqlens_q[b], cu_seqlens_q[b+1]) of Q/O and keys
 * [cu_seqlens_k[b], cu_seqlens_k[b+1]) of K/V, and attends only to its own
 * keys with the mask convention above applied per sequence (qpos(i) =
 * i + Nk_b - Nq_b). Packing sequences removes the work spent on padding, and
 * packed sequence boundaries need variable-length kernels ("How to Reduce
 * Attention Computation Cost in LLM Training": its FlashAttention section, its
 * comparison table, and "How much does sequence packing actually help?").
 * Each sequence's result is that of attn_fwd on it alone, bit for bit.
 *   q   : device, bf16 [total_q, Hq, d];  k, v : device, bf16 [total_k, Hkv, d]
 *   o   : device, bf16 [total_q, Hq, d] (rows of sequences are written; rows
 *         outside every [cu_q[b], cu_q[b+1]) are left untouched)
 *   lse : device, f32 [Hq, total_q], or NULL
 *   cu_seqlens_q, cu_seqlens_k : device, int32 [B + 1], non-decreasing,
 *         cu[0] >= 0, cu[B] <= total; 4-byte aligned
 *   max_seqlen_q / max_seqlen_k : >= every sequence's length (host values;
 *         they size the work list) and <= total_q / total_k
 *   other arguments : as attn_fwd (B = number of sequences)
 * The offsets are device data and are checked on the device: a sequence whose
 * offsets fall outside the packed tensors or exceed the max lengths is
 * skipped (nothing of it is written) and attn_device_status then returns
 * ATTN_ERR_INVALID_ARG.
 */
int attn_fwd_varlen(const void* q, const void* k, const void* v, void* o, float* lse,
                    const int* cu_seqlens_q, const int* cu_seqlens_k, int B, int Hq, int Hkv,
                    int total_q, int total_k, int max_seqlen_q, int max_seqlen_k, int d,
                    float scale, int causal, int window_left, cudaStream_t stream);

/*
 * Backward pass: gradients dQ, dK, dV of the attn_fwd operation for an
 * upstream gradient dO, with P recomputed from the forward's LSE ("Chapter 3:
 * MHA Limitations, MQA, GQA, and FlashAttention", section 3.5: the saved
 * log-sum-exp serves the backward pass). dV = Pᵀ dO; dS = P * (dP - rowsum(dO
 * * O)) with dP = dO Vᵀ; dQ = scale dS K; dK = scale dSᵀ Q; a K/V head's
 * gradients sum over its group's query heads.
 *   q, k, v, o, dout : device bf16, layouts of attn_fwd (o = its output)
 *   lse  : device f32 [B, Hq, Nq], the LSE attn_fwd wrote for this o
 *   dq   : device bf16 [B, Nq, Hq, d];  dk, dv : device bf16 [B, Nk, Hkv, d]
 *   workspace : device, >= attn_bwd_workspace_bytes(B, Hq, Nq, d) bytes,
 *          256-byte aligned (fp32 dQ accumulator and per-row dO.O sums)
 *   other arguments : as attn_fwd (the same causal / window_left / scale)
 * Returns ATTN_OK or an attn_status; nothing is launched on error.
 * attn_bwd_workspace_bytes returns 0 for invalid sizes or sizes past the
 * limits above.
 */
size_t attn_bwd_workspace_bytes(int B, int Hq, int Nq, int d);
int attn_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout,
             const float* lse, void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int Nq,
             int Nk, int d, float scale, int causal, int window_left, void* workspace,
             size_t workspace_bytes, cudaStream_t stream);

/*
 * Merge attention results computed over disjoint key sets (for example the
 * key shards of sequence-sharded attention): per query row, each part r has a
 * normalised output O_r and its log-sum-exp LSE_r; the merged result rescales
 * the parts to the common maximum before adding ("Chapter 3: MHA Limitations,
 * MQA, GQA, and FlashAttention", section 3.5): M = max LSE_r,
 * w_r = exp(LSE_r - M), O = sum w_r O_r / sum w_r, LSE = M + ln sum w_r.
 * A row no part saw a key for (every LSE_r = -inf) gets O = 0, LSE = -inf.
 *   o_parts   : device f32 [R, B, Nq, Hq, d], 16-byte aligned
 *   lse_parts : device f32 [R, B, Hq, Nq]
 *   o         : device bf16 [B, Nq, Hq, d], 8-byte aligned (written)
 *   lse       : device f32 [B, Hq, Nq] or NULL
 *   1 <= R <= 64; B, Nq, Hq >= 1; d in {64, 128}
 * Returns ATTN_OK or an attn_status; nothing is launched on error.
 */
int attn_merge(const float* o_parts, const float* lse_parts, int R, void* o, float* lse, int B,
               int Nq, int Hq, int d, cudaStream_t stream);

/*
 * Bytes of device workspace attn_decode needs for these sizes.
 * num_splits = 0 picks the split count attn_decode would pick automatically.
 * Returns 0 for invalid sizes, including sizes past the limits above.
 */
size_t attn_decode_workspace_bytes(int B, int Hq, int d, int num_splits, int Lmax);

/*
 * Single-query decode over a contiguous KV cache (split-KV + combine).
 *   q        : device, bf16 [B, Hq, d]
 *   k_cache  : device, bf16 [B, Lmax, Hkv, d]; v_cache likewise
 *   o        : device, bf16 [B, Hq, d] (written)
 *   lse      : device, f32 [B, Hq] or NULL
 *   seqlens  : device, int32 [B] with 0 <= seqlens[b] <= Lmax, or NULL (= Lmax
 *              for all). The query of sequence b sits at position
 *              seqlens[b] - 1: its own K/V are already in the cache. A
 *              sequence with seqlens[b] == 0 gets O = 0, LSE = -inf. Values
 *              outside [0, Lmax] are clamped into that range on the device.
 *   window_left : < 0 for none, else keys before the query's own position
 *   num_splits  : key splits per (sequence, kv head); 0 = automatic
 *   workspace   : device, >= attn_decode_workspace_bytes(...) bytes,
 *                 256-byte aligned; contents on entry are ignored
 * Returns ATTN_OK or an attn_status (ATTN_ERR_WORKSPACE if too small).
 */
int attn_decode(const void* q, const void* k_cache, const void* v_cache, void* o,
                float* lse, const int* seqlens, int B, int Hq, int Hkv, int Lmax,
                int d, float scale, int window_left, int num_splits,
                void* workspace, size_t workspace_bytes, cudaStream_t stream);

/*
 * Single-query decode over a paged KV cache: the cache is split into
 * fixed-size pages reached through a lookup table, so a sequence's keys need
 * not be contiguous ("Inference Engineering", section 2.5 "Optimizing
 * Attention", the PagedAttention paragraph). Logical key t of sequence b is
 * row (t % page_size) of page block_table[b * pages_per_seq + t / page_size].
 * Apart from where keys live, the operation, masks, splits and results are
 * those of attn_decode with Lmax = pages_per_seq * page_size; for the same
 * logical cache both return the same bits.
 *   k_pages  : device, bf16 [num_pages, page_size, Hkv, d], 16-byte aligned;
 *              v_pages likewise
 *   block_table : device, int32 [B, pages_per_seq], 4-byte aligned; only the
 *              entries covering keys [0, seqlens[b]) are read. An entry
 *              outside [0, num_pages) reads zeros, never other memory.
 *   page_size : 16, 32, 64, or a multiple of 128
 *   num_pages, pages_per_seq >= 1
 *   workspace : >= attn_decode_workspace_bytes(B, Hq, d, num_splits,
 *              pages_per_seq * page_size) bytes, 256-byte aligned
 *   q, o, lse, seqlens, window_left, num_splits : as attn_decode
 * Returns ATTN_OK or an attn_status; nothing is launched on error.
 */
int attn_decode_paged(const void* q, const void* k_pages, const void* v_pages, void* o,
                      float* lse, const int* block_table, const int* seqlens, int B, int Hq,
                      int Hkv, int num_pages, int page_size, int pages_per_seq, int d,
                      float scale, int window_left, int num_splits, void* workspace,
                      size_t workspace_bytes, cudaStream_t stream);

/*
 * Decode without a workspace argument, for callers that cannot allocate
 * device memory. The pages have no counterpart to this; it exists for library
 * users only. Typical callers: a host program that owns every byte of device
 * memory through its own pool and forbids outside allocations, or a code path
 * with a hard latency bound, where cudaMalloc (which may synchronise the
 * device or fail under memory pressure) is not acceptable.
 *
 * Arguments, layouts and results are those of attn_decode, minus workspace
 * and workspace_bytes. The partial results live instead in one fixed scratch
 * array inside the library: ATTN_DECODE_NOALLOC_SCRATCH_BYTES bytes of device
 * memory that every GPU which loads the library holds until the process exits.
 * A call whose split count needs more scratch than that (see
 * attn_decode_workspace_bytes) returns ATTN_ERR_WORKSPACE and launches
 * nothing; use attn_decode with a caller buffer, or fewer splits, instead.
 *
 * The first call on each device (with that device current) looks up the
 * scratch array's device address once; make that first call before any stream
 * capture. The scratch array is shared by every call on a device and keeps
 * the last call's contents; nothing in it needs to start at zero, because
 * each call writes every word it later reads. Calls that may overlap on the
 * GPU (for example on two streams without ordering) race on the scratch and
 * must not be issued that way. This entry point calls no cudaMalloc, cudaFree
 * or other allocating routine.
 */
#define ATTN_DECODE_NOALLOC_SCRATCH_BYTES ((size_t)8 << 20)
int attn_decode_noalloc(const void* q, const void* k_cache, const void* v_cache, void* o,
                        float* lse, const int* seqlens, int B, int Hq, int Hkv, int Lmax,
                        int d, float scale, int window_left, int num_splits,
                        cudaStream_t stream);

/* Message for the last non-OK status returned on this host thread ("" if none). */
const char* attn_last_error(void);

/*
 * Synchronises `stream`, then reads and clears the device status word that
 * kernels set on a device-side failure. Returns ATTN_OK, ATTN_ERR_TIMEOUT (a
 * bounded wait gave up), ATTN_ERR_INVALID_ARG (a device-side input check
 * failed: inconsistent packed-sequence offsets, whose sequences were skipped),
 * ATTN_ERR_INTERNAL (bounds-checking debug build only) or ATTN_ERR_CUDA (a
 * CUDA error surfaced by the synchronisation).
 */
int attn_device_status(cudaStream_t stream);

/*
 * 1 if this library is the bounds-checking debug build, else 0. That build
 * (libattn_debug.so, compiled with ATTN_DEBUG_BOUNDS; never the default)
 * checks, in every kernel, each computed global-memory index against the
 * extent of the buffer it addresses and, at the end of each CTA, that the
 * producer, tensor-core issuer and consumer roles counted the same number of
 * pipeline stages. A failed check skips the access, records a code that
 * attn_device_status() returns as ATTN_ERR_INTERNAL, and never traps. It is
 * the stand-in for a memory checker on machines where none can run.
 */
int attn_debug_checks(void);

/*
 * Diagnostic for the failure-detection path. Launches one small kernel whose
 * thread waits on a shared-memory barrier that nothing ever completes. The
 * wait is bounded like every wait in this library's kernels: after about one
 * second it gives up, sets the device status word and the kernel returns, so
 * the context stays usable. A following attn_device_status(stream) then
 * returns ATTN_ERR_TIMEOUT (and clears the word). Returns ATTN_OK when the
 * launch was issued.
 */
int attn_selftest_wait_timeout(cudaStream_t stream);

/* Number of kernel launches this library has issued in this process. */
unsigned long long attn_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* ATTN_H_ */
