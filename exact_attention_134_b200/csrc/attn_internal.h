// attn_internal.h — declarations shared between the C-ABI layer and the
// kernel translation units (not part of the public ABI).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

#include "../../include/attn.h"

namespace attn_sm100 {

// Raises Kernel's dynamic shared-memory limit to `bytes` once per device: the
// first launch on a device (with that device current) sets the attribute,
// later launches skip the runtime call. Devices beyond 64 set it every time.
template <auto Kernel>
cudaError_t max_dynamic_smem_once(int bytes) {
  static std::atomic<unsigned long long> done{0};  // bit d: set on device d
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const unsigned long long bit = (dev >= 0 && dev < 64) ? 1ull << dev : 0ull;
  if (bit && (done.load(std::memory_order_acquire) & bit)) return cudaSuccess;
  e = cudaFuncSetAttribute(Kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess && bit) done.fetch_or(bit, std::memory_order_release);
  return e;
}

#ifdef __CUDACC__
// Packed sequences: maps work item i of a grid row to a sequence and a unit
// (a block of U rows) of it, with no row per sequence of the longest one.
// Sequence s's ceil(L_s / U) units occupy items [v(s), v(s) + ceil(L_s / U)),
// v(s) = floor(off[s] / U) + s (off = its row offsets, clamped to [0, total]);
// these ranges are disjoint and increase with s, and items
// 0 .. floor(total / U) + num_seqs - 1 cover them all, so a grid row of that
// many items has at most one item per sequence without a unit. Returns s (the
// largest with v(s) <= i, by binary search) and sets `rank` = i - v(s), the
// unit index within the sequence (>= its unit count for an item without one).
__host__ __device__ __forceinline__ int packed_unit(const int* off, int num_seqs, int total, int U,
                                                    int i, int& rank) {
  auto v = [&](int s) { return min(max(off[s], 0), total) / U + s; };
  int lo = 0, hi = num_seqs - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (v(mid) <= i) lo = mid;
    else hi = mid - 1;
  }
  rank = i - v(lo);
  return lo;
}
#endif

// Kernel parameters of the bf16 forward (tensor maps are passed separately).
struct FwdParams {
  void* o;                        // bf16 [B, Hq, Nq, d]
  float* lse;                     // fp32 [B, Hq, Nq]
  int* status;                    // device status word: [0] code, [1] where
  const int* cu_q;                // packed sequences: query row offsets [B + 1] (else null)
  const int* cu_k;                //                   key row offsets [B + 1]
  int B, Nq, Nkv, Hq, Hkv;        // packed: B = sequences, Nq / Nkv = total rows
  int causal;
  int num_row_blocks;             // ceil(Nq / rows per work unit); packed: floor(total_q / rows) + sequences
  float scale_log2;               // scale * log2(e)
  unsigned long long timeout_ns;  // budget of every pipeline wait
  // Partial results over key ranges (dense tensors only; see attn_fwd_partial):
  float* o_part = nullptr;        // fp32 O rows [num_splits, B, Hq, Nq, d] instead of bf16 o;
                                  // lse is then [num_splits, B, Hq, Nq]
  int num_splits = 1;             // key ranges per (b, h): grid z = B * num_splits
  int kv_chunk = 0;               // keys per range (a multiple of 128) when num_splits > 1
  int kv_tail = 0;                // keys after this K/V tensor in the full sequence (causal)
  // Dense, Nq <= 128, Hq / Hkv even: a CTA's two query tiles are two query
  // heads of one kv head (grid y = Hq / 2); num_row_blocks is then ceil(Nq / 128).
  int pair_heads = 0;
  // Dense causal, one head per CTA: dispatch order groups (0 = the grid's own
  // order, each head's row blocks heaviest first). See attn_fwd_bf16_kernel.
  int lpt_group = 0;
};

// Kernel parameters of the 8-bit main kernel.
struct Q8Params {
  float* lse;                     // fp32 [B, Hq, Nq]
  int* status;                    // device status word
  const float* sq;                // [B, Hq, nqb]   Q block scales
  const float* sk;                // [B, Hkv, nkb]  smoothed-K block scales
  const float* sv;                // [B, Hkv, d]    V channel scales
  const float* qk;                // [B, Hq, Nq]    q_i . kbar
  int Nq, Nkv, Hq, Hkv;
  int causal;
  int num_row_blocks;
  int nqb, nkb;                   // 128-token blocks of Q and K/V
  int lpt_group;                  // causal dispatch order groups (0 = grid order)
  float scale_log2;               // scale * log2(e)
  float scale;
  unsigned long long timeout_ns;
};

// Everything one 8-bit forward needs (prepass + main kernel).
struct Q8Launch {
  CUtensorMap tq, tk, tv, to;     // over q8, k8, v8 (uint8) and o (bf16)
  Q8Params p;
  const void* q;                  // bf16 inputs
  const void* k;
  const void* v;
  int8_t* q8;
  int8_t* k8;
  uint8_t* v8;
  float* kbar;
  double* ksum_part;
  float* vmax_part;
  int B, Hkv;
  bool prepass_only;
  bool fp8_qk;                    // e4m3 Q and K with block scales, no smoothing
};

cudaError_t launch_q8(const Q8Launch& L, int d, cudaStream_t stream);

// Backward main kernel parameters (tensor maps of Q, K, V, dO passed separately).
struct BwdParams {
  void* dk;                       // bf16 [B, Hkv, Nkv, d]
  void* dv;                       // bf16 [B, Hkv, Nkv, d]
  float* dq_acc;                  // fp32 [B*Hq][nq_pad/128][d/4][128][4] (packed: B = sequences)
  const float* lse2;              // fp32 [B*Hq][nq_pad]  LSE * log2(e), +inf where P must be 0
  const float* dvec;              // fp32 [B*Hq][nq_pad]  D_i = sum_c dO_ic O_ic
  int* status;
  const int* cu_q;                // packed sequences: row offsets [B + 1] (else null)
  const int* cu_k;
  int Nq, Nkv, Hq, Hkv;           // packed: Nq / Nkv = total rows, B = sequences
  int causal;
  int nq_pad;                     // Nq rounded up to 128
  float scale;
  float scale_log2;
  unsigned long long timeout_ns;
  // Dense causal: dispatch order groups of (batch, kv head) pairs, key blocks
  // heaviest first across a group (0 = the grid's own order).
  int lpt_group;
  int num_seqs;                   // packed sequences: their count (else unused)
};

struct BwdPreParams {
  const void* o;                  // bf16 [B, Hq, Nq, d]
  const void* dout;               // bf16 [B, Hq, Nq, d]
  const float* lse;               // fp32 [B, Hq, Nq]
  float* dvec;
  float* lse2;
  float* dq_acc;
  const int* cu_q;                // packed sequences (else null)
  int Nq, Hq, nq_pad;
};

struct BwdPostParams {
  const float* dq_acc;
  void* dq;                       // bf16 [B, Hq, Nq, d] (packed: [total_q, Hq, d])
  const int* cu_q;
  int Nq, Hq, nq_pad;
  float scale;
};

struct BwdLaunch {
  CUtensorMap tq, tk, tv, tdo;
  BwdParams main;
  BwdPreParams pre;
  BwdPostParams post;
  int B;                          // batch entries, or sequences
  int max_kv;                     // Nkv, or the longest sequence's keys
};

cudaError_t launch_bwd(const BwdLaunch& L, int d, cudaStream_t stream);

// ATTN_OK for cudaSuccess; otherwise remembers `e` for attn_last_cuda_error()
// (per calling thread) and returns ATTN_ERR_CUDA.
attn_status_t cuda_error_status(cudaError_t e);

attn_status_t validate_fwd_args(const void* q, const void* k, const void* v, const void* o,
                                const void* lse, int B, int Hq, int Hkv, int Nq, int Nkv, int d,
                                int causal, float scale);

attn_status_t q8_forward_with_workspace(const void* q, const void* k, const void* v, void* o,
                                        float* lse, int B, int Hq, int Hkv, int Nq, int Nkv, int d,
                                        int causal, float scale, void* workspace,
                                        size_t workspace_bytes, cudaStream_t stream);

cudaError_t launch_fwd_bf16(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                            const CUtensorMap& to, const FwdParams& p, int d, cudaStream_t stream);
int fwd_rows_per_cta();
int fwd_rows_per_cta_paired();

// O = sum_s exp(LSE_s - LSE) O_s, LSE = ln sum_s exp(LSE_s) over num_parts
// partial results: part s's fp32 O rows [rows, d] at o_parts + s * o_stride and
// its fp32 LSE [rows] at lse_parts + s * lse_stride (strides in floats; <= 0:
// stacked, rows * d and rows); writes O [rows, d] (bf16, or fp32 with o_fp32)
// and fp32 LSE [rows].
cudaError_t launch_merge(const float* o_parts, const float* lse_parts, int num_parts,
                         long long rows, int d, void* o, float* lse, cudaStream_t stream,
                         bool o_fp32 = false, long long o_stride = 0, long long lse_stride = 0);

// Head dim 256, dense tensors or (p.cu_q set) packed sequences: K/V tensor maps
// with 64-row boxes; Q is read directly from global memory.
cudaError_t launch_fwd_d256(const CUtensorMap& tk, const CUtensorMap& tv, const void* q,
                            const FwdParams& p, cudaStream_t stream);
int fwd_rows_per_cta_d256();

}  // namespace attn_sm100
