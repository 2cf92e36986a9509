/*
 * attn.h — C ABI of the B200 (sm_100a) fused exact attention: forward (bf16,
 * 8-bit, packed sequences, key-range partials and their merge) and backward.
 *
 * Operation (the definition on "FlashAttention (TR)", systems-analysis.info,
 * section "Standart Attention Mekanizmasının Sorunları"):
 *     O = softmax(scale * Q K^T [+ causal mask]) V,
 *     LSE_i = ln sum_j exp(scale * (Q K^T)_ij)   over the keys row i sees,
 * computed the fused way the same page describes in "Tiling ve Blok Tabanlı
 * İşleme", "Çevrimiçi Softmax Hesaplama" and "İşlemlerin Tek Bir CUDA
 * Çekirdeğinde Birleştirilmesi": K/V tiles streamed through on-chip memory,
 * a running row maximum and exponential sum, one kernel, only O and LSE
 * written to HBM (no N x N matrix is ever stored).
 *
 * Conventions shared by every entry point
 *   - Layout: Q and O are contiguous bf16 [B, Hq, Nq, d]; K and V contiguous
 *     bf16 [B, Hkv, Nkv, d]; LSE contiguous fp32 [B, Hq, Nq] (natural log,
 *     scale included).
 *   - GQA: query head h reads kv head h / (Hq / Hkv) (contiguous groups; the
 *     pages name MQA only, "FlashAttention-2 (2023)" section). Hq % Hkv == 0.
 *   - Causal: key j is visible to query i iff j <= i + (Nkv - Nq), i.e. the
 *     mask is aligned to the bottom right (for Nq == Nkv: j <= i; for Nq < Nkv
 *     a prefill whose first Nkv - Nq keys are a cache). A row that sees no
 *     key (only possible when Nq > Nkv) gets O = 0 and LSE = -inf.
 *   - Head dim d is 64, 96 or 128; attn_fwd and attn_fwd_host also take 256
 *     (the "FlashAttention-2 (2023)" section's largest head dimension; its own
 *     kernel: one query tile per CTA, Q held in tensor memory); the 8-bit
 *     entry points take 64 or 128; the backward, attn_fwd_partial and
 *     attn_fwd_splitkv 64, 96 or 128; attn_merge_partials 64, 96, 128, 256.
 *   - Ownership: the caller owns every buffer; device pointers must stay valid
 *     until the work queued on `stream` has finished. The library allocates no
 *     device memory. `stream` is a cudaStream_t (0 = legacy default stream).
 *   - Asynchrony: work is queued on `stream`; nothing synchronises except
 *     where an entry point says so.
 *   - Errors: the return value is the only channel (nothing is printed, no
 *     exception crosses the ABI). Arguments are validated before anything is
 *     queued; a rejected call leaves every buffer untouched. Device-side
 *     failures (a pipeline wait that exceeded its time budget) are recorded in
 *     a device status word that attn_get_status() reads.
 *   - Alignment: every device pointer must be 16-byte aligned (tensor-memory
 *     accelerator descriptors require it); else ATTN_ERR_ALIGNMENT.
 */
#ifndef EXACT_ATTENTION_134_B200_ATTN_H
#define EXACT_ATTENTION_134_B200_ATTN_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define ATTN_API __attribute__((visibility("default")))
#else
#define ATTN_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  ATTN_OK = 0,
  ATTN_ERR_INVALID_ARG = 1,  /* NULL pointer, a size <= 0, Hq % Hkv != 0, scale not finite or <= 0 */
  ATTN_ERR_UNSUPPORTED = 2,  /* d not supported by the entry point (see "Head dim"); B, Hq or sequence count > 65535; a head beyond 2^40 bytes */
  ATTN_ERR_ALIGNMENT = 3,    /* a device pointer is not 16-byte aligned */
  ATTN_ERR_CUDA = 4,         /* a CUDA runtime/driver call failed (no device, launch failure, ...) */
  ATTN_ERR_TIMEOUT = 5,      /* a kernel pipeline wait exceeded its budget (reported by attn_get_status) */
  ATTN_ERR_WORKSPACE = 6     /* workspace pointer NULL/misaligned or smaller than the required size */
} attn_status_t;

/*
 * attn_fwd — bf16 fused exact attention forward.
 *   q      device, bf16 [B, Hq, Nq, d]          (read)
 *   k, v   device, bf16 [B, Hkv, Nkv, d]        (read)
 *   o      device, bf16 [B, Hq, Nq, d]          (written; RNE from fp32)
 *   lse    device, fp32 [B, Hq, Nq]             (written)
 *   scale  softmax scale applied to Q K^T (typically 1/sqrt(d)); finite, > 0
 *   causal 0 = full attention, 1 = causal mask aligned to the bottom right
 * Allocates nothing; one kernel launch on `stream`. A CTA computes two 128-row
 * query tiles sharing each K/V tile: 256 rows of one query head, or, when
 * Nq <= 128 and Hq / Hkv is even, the rows of two query heads of one kv head.
 */
ATTN_API attn_status_t attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
                       int B, int Hq, int Hkv, int Nq, int Nkv, int d,
                       int causal, float scale, void* stream);

/*
 * attn_fwd_varlen — the same operation on packed variable-length sequences
 * (a batch of prompts of different lengths without padding). Sequence s owns
 * query rows cu_seqlens_q[s] .. cu_seqlens_q[s+1]-1 and key/value rows
 * cu_seqlens_k[s] .. cu_seqlens_k[s+1]-1 and attends only within itself; the
 * causal mask is per sequence, aligned to the bottom right.
 *   q, o           device, bf16 [total_q, Hq, d]        (o written)
 *   k, v           device, bf16 [total_k, Hkv, d]
 *   lse            device, fp32 [Hq, total_q]           (written)
 *   cu_seqlens_q/k device, int32 [num_seqs + 1], non-decreasing, starting at 0
 *                  and ending at total_q / total_k (caller's responsibility;
 *                  offsets outside [0, total] are clamped, never followed)
 *   max_seqlen_q   > 0, kept for interface compatibility: the grid holds one
 *                  CTA per 256-row unit (128 at d = 256) of every sequence,
 *                  sized from total_q and num_seqs, so every row is computed
 *   d              64, 96, 128 or 256 (the head dimension up to 256 of the same
 *                  page's section "FlashAttention-2 (2023)")
 * Allocates nothing; one kernel launch on `stream`.
 */
ATTN_API attn_status_t attn_fwd_varlen(const void* q, const void* k, const void* v, void* o,
                                       float* lse, const int* cu_seqlens_q, const int* cu_seqlens_k,
                                       int num_seqs, int max_seqlen_q, int total_q, int total_k,
                                       int Hq, int Hkv, int d, int causal, float scale,
                                       void* stream);

/*
 * Key-range partial results and their merge ("FlashAttention (TR)", section
 * "Çevrimiçi Softmax Hesaplama": the running maximum / running sum update,
 * applied to whole key ranges). For disjoint key ranges s with normalised
 * partial outputs O_s and LSE_s = ln sum_{j in s} exp(scale q.k_j):
 *     LSE = ln sum_s exp(LSE_s),   O = sum_s exp(LSE_s - LSE) O_s,
 * which is exactly attn_fwd over the union of the ranges.
 *
 * attn_fwd_partial — attn_fwd of all Nq query rows over the Nkv keys of k, v
 * when those keys are one range [lo, lo + Nkv) of a longer sequence that has
 * kv_tail >= 0 more keys after them (a key-sharded multi-GPU forward: each
 * rank holds one range). The causal mask is the full sequence's, aligned to
 * its bottom right: key lo + j is visible to query i iff
 * lo + j <= i + (lo + Nkv + kv_tail - Nq), i.e. j <= i + Nkv + kv_tail - Nq
 * (kv_tail = 0: exactly attn_fwd's mask).
 *   q, k, v   as attn_fwd (d = 64, 96 or 128)
 *   o_part    device, fp32 [B, Hq, Nq, d]   (written; normalised over the range)
 *   lse_part  device, fp32 [B, Hq, Nq]      (written; -inf, with O = 0, for a
 *                                            row that sees no key of the range)
 * Allocates nothing; one kernel launch on `stream`.
 */
ATTN_API attn_status_t attn_fwd_partial(const void* q, const void* k, const void* v,
                                        float* o_part, float* lse_part, int B, int Hq, int Hkv,
                                        int Nq, int Nkv, int d, int causal, float scale,
                                        int kv_tail, void* stream);

/*
 * attn_merge_partials — the merge above over num_parts results stacked along
 * a leading axis (e.g. an all-gather of the ranks' attn_fwd_partial outputs,
 * in any order).
 *   o_parts    device, fp32 [num_parts, B, Hq, Nq, d]
 *   lse_parts  device, fp32 [num_parts, B, Hq, Nq]
 *   o          device, bf16 [B, Hq, Nq, d]   (written; RNE from fp32)
 *   lse        device, fp32 [B, Hq, Nq]      (written)
 * d = 64, 96, 128 or 256. One kernel launch; allocates nothing.
 */
ATTN_API attn_status_t attn_merge_partials(const float* o_parts, const float* lse_parts,
                                           int num_parts, int B, int Hq, int Nq, int d, void* o,
                                           float* lse, void* stream);

/*
 * attn_merge_partials_packed — the same merge over parts laid out one after
 * another in one buffer, each part = its fp32 O [B, Hq, Nq, d] followed by its
 * fp32 LSE [B, Hq, Nq], padded to attn_partial_packed_floats() floats (a
 * multiple of 4, so every part starts 16-byte aligned): the layout one
 * all-gather of every rank's partial produces, so O and LSE cross the
 * interconnect in a single collective.
 *   parts  device, fp32 [num_parts][attn_partial_packed_floats(B, Hq, Nq, d)]
 *   o, lse as attn_merge_partials
 * d = 64, 96, 128 or 256. One kernel launch; allocates nothing.
 */
ATTN_API long long attn_partial_packed_floats(int B, int Hq, int Nq, int d);
ATTN_API attn_status_t attn_merge_partials_packed(const float* parts, int num_parts, int B, int Hq,
                                                  int Nq, int d, void* o, float* lse, void* stream);

/*
 * attn_fwd_splitkv — attn_fwd with the keys split into ranges that run as
 * separate CTAs of one launch, then merged: for shapes with few query rows
 * per head and many keys (prefill against a long cache), where attn_fwd's
 * B * Hq * ceil(Nq / 256) CTAs would leave SMs idle. Same arguments and
 * results as attn_fwd (d = 64, 96 or 128), plus
 *   num_splits  key ranges per (b, h); <= 0 picks floor(SMs / CTAs of
 *               attn_fwd) ranges, one full wave (ranges of whole 128-key
 *               tiles, at least two tiles each, at most 64 ranges);
 *               attn_fwd_splitkv_num_splits() returns
 *               the count used (1 = plain attn_fwd, no workspace needed)
 *   workspace   device scratch of attn_fwd_splitkv_workspace_size() bytes,
 *               16-byte aligned, owned by the caller: the fp32 partials
 * Two launches (partials, merge). ATTN_ERR_UNSUPPORTED if B * ranges > 65535.
 */
ATTN_API int attn_fwd_splitkv_num_splits(int B, int Hq, int Hkv, int Nq, int Nkv, int d,
                                         int num_splits);
ATTN_API size_t attn_fwd_splitkv_workspace_size(int B, int Hq, int Hkv, int Nq, int Nkv, int d,
                                                int num_splits);
ATTN_API attn_status_t attn_fwd_splitkv(const void* q, const void* k, const void* v, void* o,
                                        float* lse, int B, int Hq, int Hkv, int Nq, int Nkv,
                                        int d, int causal, float scale, int num_splits,
                                        void* workspace, size_t workspace_bytes, void* stream);

/*
 * attn_fwd_partial_splitkv — attn_fwd_partial (same arguments, mask and
 * results) with the range's keys split into sub-ranges run as separate CTAs
 * and merged on the device into the fp32 partial result of the whole range
 * (the merge above, with fp32 O): for a rank of a key-sharded forward whose
 * B * Hq * ceil(Nq / 256) CTAs would leave SMs idle. num_splits, workspace and
 * the failure codes as attn_fwd_splitkv (the same attn_fwd_splitkv_num_splits
 * and attn_fwd_splitkv_workspace_size apply). One range: one launch, no
 * workspace; otherwise two launches (partials, merge).
 */
ATTN_API attn_status_t attn_fwd_partial_splitkv(const void* q, const void* k, const void* v,
                                                float* o_part, float* lse_part, int B, int Hq,
                                                int Hkv, int Nq, int Nkv, int d, int causal,
                                                float scale, int kv_tail, int num_splits,
                                                void* workspace, size_t workspace_bytes,
                                                void* stream);

/*
 * attn_fwd_host — the same operation on HOST buffers, for callers whose data
 * lives in host memory. Copies q, k, v into `dev_buf` (a device buffer of at
 * least attn_fwd_host_buffer_size() bytes, 16-byte aligned, owned by the
 * caller), runs attn_fwd, copies o and lse back and synchronises `stream`
 * before returning. The work is pipelined over up to 8 chunks of whole
 * kv-head groups: chunk c's inputs are copied in while chunk c-1 is computed
 * on `stream` and chunk c-2's outputs are copied out, on two copy streams the
 * library creates once per device (with events that order them after the work
 * already queued on `stream`). Host buffers should be page-locked for the
 * copies to overlap and run at full speed (pageable memory works, slower).
 * ATTN_ERR_UNSUPPORTED if a chunk would hold more than 65535 query heads.
 */
ATTN_API size_t attn_fwd_host_buffer_size(int B, int Hq, int Hkv, int Nq, int Nkv, int d);
ATTN_API attn_status_t attn_fwd_host(const void* q_host, const void* k_host, const void* v_host,
                            void* o_host, float* lse_host,
                            int B, int Hq, int Hkv, int Nq, int Nkv, int d,
                            int causal, float scale,
                            void* dev_buf, size_t dev_buf_bytes, void* stream);

/*
 * attn_fwd_q8 — the same operation through the 8-bit mainloop of
 * "Makale Bülteni — SageAttention" (section "İddia ve Gerçeklik:
 * SageAttention"): K is mean-centred per (batch, kv head, channel) over all
 * Nkv tokens (lossless by the shift invariance of softmax; LSE is corrected
 * back), Q and the smoothed K are quantised to INT8 with one fp32 scale per
 * 128-token block, V to FP8 e4m3 with one fp32 scale per channel; S = Q8 K8^T
 * runs on INT8 tensor cores (s32 accumulation), P is encoded as
 * e4m3(2^(t - m_ref) * 448 / 16) against a reference maximum m_ref that lags
 * the row maximum by at most 2^4 (so O is rescaled only when it is overtaken
 * by more), and P8 V8 runs on FP8 tensor cores (fp32 accumulation).
 *   inputs/outputs  as attn_fwd (bf16 q, k, v; bf16 o; fp32 lse)
 *   workspace       device, caller-owned, 16-byte aligned, at least
 *                   attn_fwd_q8_workspace_size() bytes; holds the quantised
 *                   tensors and scales (its contents after the call are the
 *                   prepass results, see attn_q8_workspace_offsets)
 * Four launches on `stream` (three prepass kernels, one main kernel); the
 * last three are dependent launches that may start while their predecessor
 * finishes and wait on the device for its results, the first waits for all
 * earlier work on `stream`.
 * Errors: as attn_fwd, plus ATTN_ERR_WORKSPACE for a NULL, misaligned or too
 * small workspace.
 */
ATTN_API size_t attn_fwd_q8_workspace_size(int B, int Hq, int Hkv, int Nq, int Nkv, int d);
ATTN_API attn_status_t attn_fwd_q8(const void* q, const void* k, const void* v, void* o, float* lse,
                                   int B, int Hq, int Hkv, int Nq, int Nkv, int d,
                                   int causal, float scale,
                                   void* workspace, size_t workspace_bytes, void* stream);

/*
 * attn_fwd_fp8 — the 8-bit forward with FP8 e4m3 Q and K instead of INT8 and
 * no K smoothing, in the manner "Makale Bülteni — FlashAttention-3" ("İddia
 * ve Gerçeklik") describes for its FP8 mode: block-wise dynamic scaling, one
 * fp32 scale = amax / 448 per 128-token block of Q and of K; S = Q8 K8^T on
 * FP8 tensor cores with fp32 accumulation; P and V exactly as in attn_fwd_q8.
 * It is the comparison point for INT8 with K smoothing on channels with
 * outliers. Same arguments, workspace and errors as attn_fwd_q8 (the workspace
 * regions hold e4m3 codes for Q and K, kbar and q.kbar are zero; its
 * statistics kernel reads V only).
 * attn_fp8_prepass runs only its three prepass launches.
 */
ATTN_API attn_status_t attn_fwd_fp8(const void* q, const void* k, const void* v, void* o, float* lse,
                                    int B, int Hq, int Hkv, int Nq, int Nkv, int d,
                                    int causal, float scale,
                                    void* workspace, size_t workspace_bytes, void* stream);
ATTN_API attn_status_t attn_fp8_prepass(const void* q, const void* k, const void* v,
                                        int B, int Hq, int Hkv, int Nq, int Nkv, int d,
                                        void* workspace, size_t workspace_bytes, void* stream);

/*
 * attn_fwd_q8_noalloc — attn_fwd_q8 for callers that cannot allocate device
 * memory, e.g. a plugin inside another framework's inference engine that is
 * handed only its input and output buffers, or a program that must not call
 * cudaMalloc while serving (it can synchronise the device, and fails when
 * another allocator has reserved the GPU's memory). The pages have no
 * counterpart: this is an interface convenience, not part of the method.
 *   arguments      as attn_fwd (bf16 q, k, v; bf16 o; fp32 lse); no workspace
 *   scratch        a static device array of attn_fwd_q8_static_scratch_bytes()
 *                  bytes (32 MiB) inside the library, held on every GPU that
 *                  loads the library until the process exits
 *   size limit     problems whose attn_fwd_q8_workspace_size() exceeds the
 *                  array are rejected with ATTN_ERR_WORKSPACE before anything
 *                  is queued
 *   allocation     none: no cudaMalloc / cudaFree or allocating library call
 *   first call     on each device, looks up the array's device address
 *                  (cudaGetSymbolAddress) with that device current; with
 *                  CUDA's default lazy module loading this is also when the
 *                  32 MiB are reserved on that device, so make the first call
 *                  at start-up, before other allocators take the GPU's memory
 *                  and before any stream capture; a failure of the look-up
 *                  returns ATTN_ERR_CUDA (attn_last_cuda_error has the cause)
 *   concurrency    every call shares the one array: calls whose work overlaps
 *                  on the GPU (different streams, no ordering between them)
 *                  race on it and must be serialised by the caller. The array
 *                  keeps the last call's contents; nothing in it needs to
 *                  start at zero.
 */
ATTN_API size_t attn_fwd_q8_static_scratch_bytes(void);
ATTN_API attn_status_t attn_fwd_q8_noalloc(const void* q, const void* k, const void* v, void* o,
                                           float* lse, int B, int Hq, int Hkv, int Nq, int Nkv,
                                           int d, int causal, float scale, void* stream);

/*
 * attn_q8_prepass — only the three prepass launches of attn_fwd_q8 (K mean,
 * V channel scales, quantisation of Q, K, V), writing the workspace; used to
 * time the prepass on its own and to inspect its results.
 */
ATTN_API attn_status_t attn_q8_prepass(const void* q, const void* k, const void* v,
                                       int B, int Hq, int Hkv, int Nq, int Nkv, int d,
                                       void* workspace, size_t workspace_bytes, void* stream);

/*
 * attn_q8_workspace_offsets — byte offsets of the workspace regions, in
 * order: q8 int8 [B,Hq,Nq,d], k8 int8 [B,Hkv,Nkv,d] (smoothed), v8 e4m3
 * [B,Hkv,Nkv,d], sq fp32 [B,Hq,ceil(Nq/128)], sk fp32 [B,Hkv,ceil(Nkv/128)],
 * sv fp32 [B,Hkv,d], kbar fp32 [B,Hkv,d], qk fp32 [B,Hq,Nq] (q_i . kbar),
 * K partial sums fp64 [B,Hkv,ceil(Nkv/128),d], V partial maxima fp32
 * [B,Hkv,ceil(Nkv/128),d]; offsets[10] = total size. `offsets` holds 11
 * entries.
 */
ATTN_API attn_status_t attn_q8_workspace_offsets(int B, int Hq, int Hkv, int Nq, int Nkv, int d,
                                                 size_t* offsets);

/*
 * attn_bwd — gradients of attn_fwd: given dO = dLoss/dO, writes
 *     dQ = scale * dS K,   dK = scale * dS^T Q,   dV = P^T dO,
 *     dS = P * (dO V^T - D),   D_i = sum_c dO_ic O_ic,
 * with P = exp(scale * Q K^T - LSE) recomputed block by block from the LSE the
 * forward wrote (the glossary page "FlashAttention", aisaas-seo: the backward
 * recomputes a few cheap quantities instead of storing them); no N x N matrix
 * is stored. The formulas are the derivative of the definition on
 * "FlashAttention (TR)" ("Standart Attention Mekanizmasının Sorunları").
 *   q, k, v        bf16 inputs of the forward, layouts as attn_fwd
 *   o, lse         the forward's outputs (bf16 [B,Hq,Nq,d], fp32 [B,Hq,Nq])
 *   dout           bf16 [B, Hq, Nq, d]
 *   dq             bf16 [B, Hq, Nq, d]   (written)
 *   dk, dv         bf16 [B, Hkv, Nkv, d] (written; with GQA the sum over the
 *                  query heads of each group)
 *   causal, scale  as passed to the forward (bottom-right causal alignment)
 *   workspace      device scratch of attn_bwd_workspace_size() bytes, 16-byte
 *                  aligned, owned by the caller; holds the fp32 dQ
 *                  accumulator, D and LSE * log2(e); needs no initial value
 * d must be 64, 96 or 128 (256: ATTN_ERR_UNSUPPORTED). The dQ accumulation
 * adds fp32 partial sums with bulk reductions in L2 whose order is not fixed,
 * so dQ may differ in the last bits between runs; dK and dV are deterministic. Errors as attn_fwd, plus
 * ATTN_ERR_WORKSPACE for a missing, misaligned or short workspace.
 */
ATTN_API size_t attn_bwd_workspace_size(int B, int Hq, int Hkv, int Nq, int Nkv, int d);
ATTN_API attn_status_t attn_bwd(const void* q, const void* k, const void* v, const void* o,
                                const float* lse, const void* dout, void* dq, void* dk, void* dv,
                                int B, int Hq, int Hkv, int Nq, int Nkv, int d, int causal,
                                float scale, void* workspace, size_t workspace_bytes,
                                void* stream);

/*
 * attn_bwd_varlen — attn_bwd for packed variable-length sequences, the
 * gradients of attn_fwd_varlen: q, o, dout, dq [total_q, Hq, d]; k, v, dk, dv
 * [total_k, Hkv, d]; lse fp32 [Hq, total_q] as attn_fwd_varlen writes it;
 * cu_seqlens_q / cu_seqlens_k int32 device arrays [num_seqs + 1] (sequence s
 * owns rows cu[s] .. cu[s+1]); max_seqlen_q must bound every sequence's query
 * rows (it sizes the workspace; query rows beyond it are not computed, and
 * nothing outside the buffers is touched); max_seqlen_k > 0 is kept for
 * interface compatibility (the grid holds one CTA per 128-key unit of every
 * sequence, sized from total_k and num_seqs). Causal masks are
 * aligned to the bottom right of each sequence. Rows of dk / dv that no
 * query sees are written as 0. Workspace: attn_bwd_varlen_workspace_size()
 * bytes (fp32 dQ accumulator with every sequence padded to max_seqlen_q
 * rows, then LSE * log2(e) and D). Errors as attn_bwd and attn_fwd_varlen.
 */
ATTN_API size_t attn_bwd_varlen_workspace_size(int num_seqs, int Hq, int max_seqlen_q, int d);
ATTN_API attn_status_t attn_bwd_varlen(const void* q, const void* k, const void* v, const void* o,
                                       const float* lse, const void* dout, void* dq, void* dk,
                                       void* dv, const int* cu_seqlens_q,
                                       const int* cu_seqlens_k, int num_seqs, int max_seqlen_q,
                                       int max_seqlen_k, int total_q, int total_k, int Hq,
                                       int Hkv, int d, int causal, float scale, void* workspace,
                                       size_t workspace_bytes, void* stream);

/*
 * attn_get_status — synchronises `stream`, returns and clears the device
 * status word (ATTN_OK, or ATTN_ERR_TIMEOUT if a kernel gave up on a pipeline
 * wait since the last call). Returns ATTN_ERR_CUDA if synchronisation fails.
 */
ATTN_API attn_status_t attn_get_status(void* stream);

/* attn_get_status_ex — as attn_get_status; also stores in *where (if not
 * NULL) a diagnostic code naming the kernel role and tile that gave up
 * (0 when nothing failed). */
ATTN_API attn_status_t attn_get_status_ex(void* stream, int* where);

/*
 * attn_selftest_wait_timeout — exercises the failure-detection path without a
 * fault: one GPU thread waits, with the same bounded wait the kernels use, on
 * a barrier that nothing completes; after `budget_us` microseconds (1 ..
 * 10^7) it gives up and records ATTN_ERR_TIMEOUT in the device status word
 * (where = 0xF00), and the kernel returns normally. Read the result with
 * attn_get_status_ex(). Queued on `stream`; ATTN_ERR_INVALID_ARG for a budget
 * outside the range. Not part of the method: a test hook for the timeout
 * machinery every attention kernel relies on.
 */
ATTN_API attn_status_t attn_selftest_wait_timeout(int budget_us, void* stream);

/* attn_set_timeout_ms — budget of every in-kernel pipeline wait (default 1000
 * ms; values < 1 are rejected with ATTN_ERR_INVALID_ARG). Process-wide. */
ATTN_API attn_status_t attn_set_timeout_ms(int ms);

/* Human-readable name of a status code (static storage). */
ATTN_API const char* attn_status_string(attn_status_t status);

/* attn_last_cuda_error — the CUDA runtime error code behind the most recent
 * ATTN_ERR_CUDA returned on this host thread by a launch (0 if none), and
 * its message in *message (static storage) when message is not NULL. */
ATTN_API int attn_last_cuda_error(const char** message);

/* Library version, major * 10000 + minor * 100 + patch. */
ATTN_API int attn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* EXACT_ATTENTION_134_B200_ATTN_H */
