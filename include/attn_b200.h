/*
 * attn_b200.h: C ABI of the B200 (sm_100a) fused exact-attention library.
 *
 * Operations computing  O = softmax(scale * Q K^T + mask) V  and the per-row
 * log-sum-exp, exactly (up to floating-point rounding), without ever writing
 * the score matrix to device memory, and the gradients of the forward:
 *
 *   attn_fwd               prefill / training forward over dense Q, K, V
 *   attn_fwd_fp8           the same on E4M3 inputs with per-tensor descales
 *   attn_bwd               dQ, dK, dV of attn_fwd, recomputing S and P
 *   attn_decode_paged      one-token MLA ("MQA-absorb") decode over a paged cache
 *   attn_decode_paged_mtp  the same with s_q query tokens per sequence
 *   attn_decode_paged_gqa  one-token decode over paged, grouped K and V caches
 *
 * Sources for what is computed (web pages, cited by title and section):
 *   - "FlashAttention (KO)", section on the problems of standard attention:
 *     Attention(Q,K,V) = softmax(Q K^T / sqrt(d_k)) V; the N x N matrix S is
 *     what the IO-aware method never stores.
 *   - same page, sections on tiling, online softmax (running max and running
 *     exp-sum reach the exact result) and fusion of QK^T, masking, softmax
 *     and the product with V into one kernel.
 *   - "FlashMLA" page, technical basis: BF16, variable-length sequences, a KV
 *     cache paged in 64-token pages.
 *   - "GQLA: Group-Query Latent Attention ...", sections 1-3: MLA compresses K
 *     and V into one low-rank latent; in the MQA-absorb decode path every
 *     query head attends to that one shared latent.
 *
 * Conventions shared by every entry point
 *   - All tensors are device pointers, contiguous, row-major, bf16 unless
 *     stated; the caller owns every buffer (allocates and frees it).  The
 *     library allocates no device memory except one status word per device,
 *     created on first use.
 *   - Calls only enqueue work on `stream` (a cudaStream_t passed as void*,
 *     NULL = legacy default stream) and return; they never synchronise.
 *   - Argument errors are detected on the host before anything is enqueued
 *     and leave every output untouched.
 *   - Nothing is thrown across the ABI; every call returns an attn_status.
 *   - A kernel that finds a barrier phase stuck for more than 2 s aborts,
 *     frees its tensor memory, and records ATTN_ERR_TIMEOUT in the device
 *     status word (read it with attn_read_device_status after synchronising).
 */
#ifndef ATTN_B200_H_
#define ATTN_B200_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  ATTN_OK = 0,
  ATTN_ERR_INVALID_ARG = 1, /* null/misaligned pointer, bad size or scale    */
  ATTN_ERR_UNSUPPORTED = 2, /* valid request outside what is implemented     */
  ATTN_ERR_CUDA = 3,        /* a CUDA runtime/driver call or launch failed   */
  ATTN_ERR_TIMEOUT = 4,     /* device-side bounded wait expired (status word)*/
  ATTN_ERR_WORKSPACE = 5    /* workspace missing or smaller than required    */
} attn_status;

/* Version of this ABI; bumped on any incompatible change. */
int attn_abi_version(void);

/* Human-readable name of a status code (static string, never NULL). */
const char* attn_status_string(int status);

/*
 * attn_fwd: fused exact attention forward.
 *
 *   q   [B, Nq, Hq,  D ] bf16      k [B, Nk, Hkv, D] bf16
 *   v   [B, Nk, Hkv, Dv] bf16      o [B, Nq, Hq, Dv] bf16 (written)
 *   lse [B, Hq, Nq]      fp32 (written): natural log of sum_j exp(scale*q_i.k_j)
 *       over the visible keys j.
 *
 * Query head h reads KV head h / (Hq / Hkv) (grouped-query attention; Hkv = 1
 * is multi-query attention, Hkv = Hq multi-head).
 * causal != 0 masks key j for query i when j > i + (Nk - Nq) (mask aligned to
 * the bottom-right corner; the usual lower triangle when Nq == Nk).  A query
 * row with no visible key gets O = 0 and LSE = -inf.
 *
 * Supported: D == Dv in {64, 128, 256}; Hq % Hkv == 0; scale finite and > 0;
 * q, k, v, o 16-byte aligned; lse 4-byte aligned; Nq, Nk >= 0, B, Hq, Hkv >= 1,
 * B and Hq at most 65535.  Accumulation is fp32; probabilities are rounded to
 * bf16 before the product with V; O is rounded to bf16 once at the end.
 * Results are deterministic run to run.
 */
int attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv, int Nq,
             int Nk, int D, int Dv, int causal, float scale, void* stream);

/*
 * attn_fwd_fp8: attn_fwd with e4m3 inputs ("FlashAttention (KO)", section
 * "FlashAttention-3 (2024)": FP8 support on Hopper).
 *
 *   q [B, Nq, Hq, D], k [B, Nk, Hkv, D], v [B, Nk, Hkv, D]: OCP FP8 E4M3 bytes
 *   q_descale, k_descale, v_descale: per-tensor factors; the represented
 *       values are q_descale * e4m3(q) and likewise for k and v
 *   o [B, Nq, Hq, D] bf16 (written), lse [B, Hq, Nq] fp32 (written)
 *
 * Computes O = softmax(scale * Q K^T + causal mask) V and the LSE of the
 * represented values, exactly as attn_fwd defines them.  Q K^T is taken on
 * the e4m3 tensor cores with fp32 accumulation; each probability is rounded
 * to e4m3 before the product with V (relative error up to 2^-4), the row sums
 * and the LSE use the unrounded probabilities.  Supported: D == 128; descales
 * finite and > 0; the other rules as attn_fwd.
 */
int attn_fwd_fp8(const void* q, const void* k, const void* v, float q_descale, float k_descale, float v_descale,
                 void* o, float* lse, int B, int Hq, int Hkv, int Nq, int Nk, int D, int causal, float scale,
                 void* stream);

/*
 * attn_bwd_workspace_size: bytes of device workspace that attn_bwd needs for
 * B x Nq query rows of Hq heads of width D (an fp32 dQ accumulator plus one
 * fp32 value per query row).  0 for an unsupported D.  The caller allocates
 * it, 256-byte aligned.
 */
size_t attn_bwd_workspace_size(int B, int Hq, int Nq, int D);

/*
 * attn_bwd: gradients of attn_fwd with respect to q, k and v, with S and P
 * recomputed block by block from q, k and the forward's LSE ("Flash
 * Attention" wiki page, section "구조화된 지식 (Synthesized Content)", item
 * "Recomputation (재계산)": the backward pass recomputes what it needs
 * instead of storing N x N matrices).  For an upstream gradient dout = dL/dO:
 *
 *   P = exp(scale * q k^T - lse) (0 where masked), dv = P^T dout,
 *   dP = dout v^T, dS = P * (dP - rowsum(dout * o)),
 *   dq = scale * dS k, dk = scale * dS^T q
 *
 * with dk and dv summed over the query heads that share a KV head.
 *
 *   q, o, dout  [B, Nq, Hq, D] bf16     k, v [B, Nk, Hkv, D] bf16
 *   lse         [B, Hq, Nq] fp32, as written by attn_fwd for the same inputs
 *   dq          [B, Nq, Hq, D] bf16 (written)
 *   dk, dv      [B, Nk, Hkv, D] bf16 (written)
 *   workspace   at least attn_bwd_workspace_size(B, Hq, Nq, D) bytes; content
 *               on entry irrelevant, undefined on return
 *
 * causal, scale, the head grouping and the mask alignment are those of
 * attn_fwd.  Supported: D == Dv in {64, 128}; Hq % Hkv == 0; scale finite and
 * > 0; tensors 16-byte aligned, lse 4-byte aligned.  Accumulation is fp32; P
 * and dS are rounded to bf16 before their products; outputs are rounded to
 * bf16 once.  dk and dv are deterministic run to run; dq is summed over key
 * blocks in an fp32 accumulator (each key block's contribution is added at L2
 * by a TMA reduce-add of a shared-memory tile, in whatever order the CTAs
 * reach it), so its last bits may vary from run to run.  Returns
 * ATTN_ERR_WORKSPACE if the workspace is missing, too small or misaligned.
 */
int attn_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout, const float* lse,
             void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int Nq, int Nk, int D, int Dv, int causal,
             float scale, void* workspace, size_t workspace_bytes, void* stream);

/*
 * attn_bwd_head_group: the unit order attn_bwd takes for this shape on a
 * device with sm_count SMs.  Host-only: it launches nothing and needs no GPU.
 * attn_bwd runs one CTA per (key block of 128 keys, KV head, batch) and hands
 * the CTAs out g (batch, KV head) pairs at a time, key block slowest inside
 * a group, so the causal blocks that see the most queries start first.
 * Returns g: B * Hkv is key block slowest over every pair.  A smaller g,
 * ceil(sm_count / key blocks), keeps fewer heads' Q, dO and dQ rows live in
 * L2 at once.  It is taken only when a model of the block scheduler gives it
 * at most 1 % more makespan.  In that model each unit goes, in order, to the
 * SM that frees first and costs its query steps plus 4.  Returns 0 for
 * arguments that attn_bwd would reject, and for Nk == 0 (no units).
 */
int attn_bwd_head_group(int B, int Hq, int Hkv, int Nq, int Nk, int D, int causal, int sm_count);

/*
 * attn_decode_paged_workspace_size: bytes of device workspace that
 * attn_decode_paged needs for a batch of B sequences with Hq heads of width
 * Dv when it runs on CUDA device `device` (the split-KV plan depends on the
 * device's SM count).  Returns 0 for an unsupported shape, or when `device`
 * is not a valid CUDA device index.  The caller allocates it, 256-byte
 * aligned, on that device.
 */
size_t attn_decode_paged_workspace_size(int B, int Hq, int Dv, int device);

/*
 * attn_decode_paged: one new query token per sequence attending to a paged
 * latent KV cache, MLA absorbed ("MQA-absorb") form.
 *
 *   q             [B, 1, Hq, Dk] bf16   absorbed queries
 *   kv_pages      [num_pages, page_size, 1, Dk] bf16 latent rows; K = all Dk
 *                 entries of a row, V = its first Dv entries
 *   block_table   [B, max_pages_per_seq] int32: token t of sequence b lives in
 *                 page block_table[b][t / page_size], row t % page_size
 *   cache_seqlens [B] int32: number of cached tokens of each sequence
 *   o             [B, 1, Hq, Dv] bf16 (written)
 *   lse           [B, Hq] fp32 (written), natural-log LSE of the scaled scores
 *   workspace     device scratch of at least attn_decode_paged_workspace_size
 *                 bytes (split-KV partial results); its content on entry is
 *                 irrelevant and undefined on return.
 *
 * The new token sees every cached token of its sequence (no mask inside the
 * length).  A sequence of length 0 gets O = 0 and LSE = -inf.  Rows of a page
 * past the sequence length and pages past its last page are never used in
 * the result, but must hold finite values (they may be read).
 *
 * Supported: Dk = 576, Dv = 512, page_size = 64, Hq = 128; block-table
 * entries in [0, num_pages) for every page a sequence uses; lengths in
 * [0, max_pages_per_seq * page_size]; pointers 16-byte aligned.
 * Lengths and block-table entries are read on the device (no host sync); out
 * of range entries make the kernel skip that sequence and record
 * ATTN_ERR_INVALID_ARG in the device status word.
 */
int attn_decode_paged(const void* q, const void* kv_pages, const int32_t* block_table,
                      const int32_t* cache_seqlens, void* o, float* lse, int B, int Hq, int Dk, int Dv,
                      int page_size, int num_pages, int max_pages_per_seq, float scale, void* workspace,
                      size_t workspace_bytes, void* stream);

/*
 * attn_decode_paged_mtp_workspace_size: workspace bytes of attn_decode_paged_mtp
 * for B sequences with s_q query tokens each on CUDA device `device` (0 for an
 * unsupported shape or an invalid device index).
 */
size_t attn_decode_paged_mtp_workspace_size(int B, int s_q, int Hq, int Dv, int device);

/*
 * attn_decode_paged_mtp: attn_decode_paged with s_q >= 1 new query tokens per
 * sequence (multi-token prediction / speculative decoding; "GQLA ..." page,
 * MTP with the MQA-absorb path).  The s_q query tokens are the last s_q cached
 * tokens of their sequence (their latent rows are already in the cache), so
 * query token i sees cached positions 0 .. L_b - s_q + i: the causal mask of
 * attn_fwd, aligned to the bottom-right corner.  A token with no visible
 * position gets O = 0 and LSE = -inf.
 *
 *   q    [B, s_q, Hq, Dk] bf16      o   [B, s_q, Hq, Dv] bf16 (written)
 *   lse  [B, s_q, Hq] fp32 (written)
 *
 * Every other argument, layout and error is that of attn_decode_paged, whose
 * call equals this one with s_q = 1.  Supported: B * s_q <= 2048.  Each query
 * token is scheduled as its own unit over the sequence's block-table row (the
 * fp32 accumulator of 128 heads x 512 already fills an SM's tensor memory, so
 * query tokens are not stacked into one MMA tile).
 */
int attn_decode_paged_mtp(const void* q, const void* kv_pages, const int32_t* block_table,
                          const int32_t* cache_seqlens, void* o, float* lse, int B, int s_q, int Hq, int Dk, int Dv,
                          int page_size, int num_pages, int max_pages_per_seq, float scale, void* workspace,
                          size_t workspace_bytes, void* stream);

/*
 * attn_decode_paged_noalloc: attn_decode_paged without a caller workspace.
 * The source pages describe no counterpart of this entry point; it exists for
 * callers that cannot allocate device memory at decode time (a serving engine
 * that gives all of HBM to its own KV-cache pool has no room for a per-call
 * workspace, and latency-critical decode loops may not call the allocator).
 *
 * Arguments, layouts, results and errors are those of attn_decode_paged.  The
 * split-KV scratch is a fixed array inside this library of
 * attn_decode_paged_noalloc_max_bytes() bytes (40 MiB), held on every GPU
 * that loads the library until the process exits; a batch whose workspace
 * (attn_decode_paged_workspace_size) exceeds it is rejected with
 * ATTN_ERR_UNSUPPORTED before anything is enqueued.  The workspace grows with
 * the device's SM count; on a 148-SM B200 every batch up to the decode's
 * limit of 2048 sequences fits, so there only that limit applies.  The call
 * allocates no device memory.  The first call on each device looks up the array's device
 * address (with that device current), so make it before any stream capture.
 * All calls share the array and it keeps the last call's contents: calls whose
 * kernels overlap on the GPU (several streams or threads) race on it and must
 * be serialised by the caller.
 */
int attn_decode_paged_noalloc(const void* q, const void* kv_pages, const int32_t* block_table,
                              const int32_t* cache_seqlens, void* o, float* lse, int B, int Hq, int Dk, int Dv,
                              int page_size, int num_pages, int max_pages_per_seq, float scale, void* stream);

/* Size in bytes of the fixed scratch array used by attn_decode_paged_noalloc. */
size_t attn_decode_paged_noalloc_max_bytes(void);

/*
 * attn_decode_paged_gqa_workspace_size: bytes of device workspace that
 * attn_decode_paged_gqa needs for B sequences, Hq query heads in groups of
 * Hq / Hkv, head dim D, on CUDA device `device` (0 for an unsupported shape or
 * an invalid device index).
 */
size_t attn_decode_paged_gqa_workspace_size(int B, int Hq, int Hkv, int D, int device);

/*
 * attn_decode_paged_gqa: one new query token per sequence attending to a
 * paged cache of separate K and V rows per (token, KV head): the GQA decoding
 * path ("GQLA: Group-Query Latent Attention ...", key terms: each group of
 * query heads reads its own group-expanded cache; "FlashMLA" page: 64-token
 * pages reached through a block table).
 *
 *   q             [B, 1, Hq, D] bf16
 *   k_pages       [num_pages, page_size, Hkv, D] bf16
 *   v_pages       [num_pages, page_size, Hkv, D] bf16
 *   block_table   [B, max_pages_per_seq] int32 (token t of sequence b lives in
 *                 page block_table[b][t / page_size], row t % page_size)
 *   cache_seqlens [B] int32
 *   o             [B, 1, Hq, D] bf16 (written)
 *   lse           [B, Hq] fp32 (written), natural-log LSE of the scaled scores
 *   workspace     device scratch of at least
 *                 attn_decode_paged_gqa_workspace_size(B, Hq, Hkv, D) bytes,
 *                 256-byte aligned; contents irrelevant on entry.
 *
 * Query head h reads KV head h / (Hq / Hkv) and sees every cached token of its
 * sequence.  A sequence of length 0 gets O = 0 and LSE = -inf.  Rows past the
 * sequence length must hold finite values (they may be read).
 *
 * Supported: D in {64, 128}; Hq / Hkv in {1, 2, 4, 8}; page_size = 64;
 * B <= 2048; pointers 16-byte aligned.  Block-table entries out of
 * [0, num_pages) make the kernel read page 0 instead for that page and record
 * ATTN_ERR_INVALID_ARG in the device status word.  Accumulation is fp32; O is
 * rounded to bf16 once.  Deterministic run to run.
 */
int attn_decode_paged_gqa(const void* q, const void* k_pages, const void* v_pages, const int32_t* block_table,
                          const int32_t* cache_seqlens, void* o, float* lse, int B, int Hq, int Hkv, int D,
                          int page_size, int num_pages, int max_pages_per_seq, float scale, void* workspace,
                          size_t workspace_bytes, void* stream);

/*
 * attn_selftest_wait_timeout: exercise the bounded-wait failure path.  The
 * source pages describe no counterpart; this checks this library's own
 * failure detection.  One CTA waits on a barrier that nothing ever releases,
 * with the same bounded wait the attention kernels use but a limit of
 * `limit_us` microseconds (1 .. 10,000,000).  When the limit passes, the kernel
 * records ATTN_ERR_TIMEOUT in the device status word and returns normally:
 * nothing faults or hangs and the context stays usable.  Enqueues on
 * `stream`; read the outcome with attn_read_device_status.
 */
int attn_selftest_wait_timeout(unsigned int limit_us, void* stream);

/*
 * attn_read_device_status: status recorded by kernels on `device` since the
 * last call (ATTN_OK if none), then reset to ATTN_OK.  Synchronises with the
 * device first.  Returns ATTN_ERR_CUDA if the device cannot be queried.
 */
int attn_read_device_status(int device);

#ifdef __cplusplus
}
#endif

#endif /* ATTN_B200_H_ */
