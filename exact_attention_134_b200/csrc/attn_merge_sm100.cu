// attn_merge_sm100.cu — merge of partial attention results over disjoint key
// ranges (the split-key forward and the key-sharded multi-GPU forward).
//
// "FlashAttention (TR)" (systems-analysis.info), section "Çevrimiçi Softmax
// Hesaplama": the softmax is built piece by piece from a running maximum and a
// running sum of exponentials. For whole key ranges s with normalised O_s and
// LSE_s = ln sum_{j in s} exp(S_ij) that update reads
//     LSE = ln sum_s exp(LSE_s),   O = sum_s exp(LSE_s - LSE) O_s,
// exact in real arithmetic. A part with LSE_s = -inf (no visible key) has
// weight 0; a row with no visible key in any part gets O = 0, LSE = -inf.
//
// HBM-bound: reads num_parts * (4 d + 4) bytes per row, writes 2 d + 4 (bf16 O)
// or 4 d + 4 (fp32 O: the merged result is itself a partial over the union of
// the ranges, for a later merge). d / 4 threads per row (one float4 of every
// part each), 8 rows per CTA.
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "attn_internal.h"

namespace attn_sm100 {
namespace {

constexpr int kRowsPerCta = 8;

__device__ __forceinline__ uint32_t pack_bf16x2_rn(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

template <int D, bool F32>
__global__ void __launch_bounds__(D / 4 * kRowsPerCta)
    attn_merge_kernel(const float* __restrict__ o_parts, const float* __restrict__ lse_parts,
                      int num_parts, long long rows, long long o_stride, long long lse_stride,
                      void* __restrict__ o, float* __restrict__ lse) {
  constexpr int kT = D / 4;  // threads per row
  const int c4 = threadIdx.x % kT;
  const long long r = (long long)blockIdx.x * kRowsPerCta + threadIdx.x / kT;
  if (r >= rows) return;
  float m = -INFINITY;
  // part s: O rows at o_parts + s * o_stride, LSE at lse_parts + s * lse_stride (floats)
  for (int s = 0; s < num_parts; ++s) m = fmaxf(m, lse_parts[(size_t)s * lse_stride + r]);
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  float total = 0.0f;
  if (m != -INFINITY) {
    for (int s = 0; s < num_parts; ++s) {
      const float w = expf(lse_parts[(size_t)s * lse_stride + r] - m);  // 0 for a -inf part
      const float4 x = reinterpret_cast<const float4*>(o_parts + (size_t)s * o_stride + (size_t)r * D)[c4];
      acc.x = fmaf(w, x.x, acc.x);
      acc.y = fmaf(w, x.y, acc.y);
      acc.z = fmaf(w, x.z, acc.z);
      acc.w = fmaf(w, x.w, acc.w);
      total += w;
    }
  }
  const float inv = total > 0.0f ? 1.0f / total : 0.0f;
  if (F32) {
    reinterpret_cast<float4*>(static_cast<float*>(o) + r * D)[c4] =
        make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
  } else {
    uint2 out;
    out.x = pack_bf16x2_rn(acc.x * inv, acc.y * inv);
    out.y = pack_bf16x2_rn(acc.z * inv, acc.w * inv);
    reinterpret_cast<uint2*>(static_cast<uint16_t*>(o) + r * D)[c4] = out;
  }
  if (c4 == 0) lse[r] = (m == -INFINITY) ? -INFINITY : m + logf(total);
}

template <int D>
cudaError_t launch_merge_d(const float* o_parts, const float* lse_parts, int num_parts,
                           long long rows, long long o_stride, long long lse_stride, void* o,
                           float* lse, bool o_fp32, cudaStream_t stream) {
  const long long blocks = (rows + kRowsPerCta - 1) / kRowsPerCta;
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  if (o_fp32)
    attn_merge_kernel<D, true><<<(unsigned)blocks, D / 4 * kRowsPerCta, 0, stream>>>(
        o_parts, lse_parts, num_parts, rows, o_stride, lse_stride, o, lse);
  else
    attn_merge_kernel<D, false><<<(unsigned)blocks, D / 4 * kRowsPerCta, 0, stream>>>(
        o_parts, lse_parts, num_parts, rows, o_stride, lse_stride, o, lse);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_merge(const float* o_parts, const float* lse_parts, int num_parts,
                         long long rows, int d, void* o, float* lse, cudaStream_t stream,
                         bool o_fp32, long long o_stride, long long lse_stride) {
  if (o_stride <= 0) o_stride = rows * d;  // parts stacked: [num_parts, rows, d]
  if (lse_stride <= 0) lse_stride = rows;  //                [num_parts, rows]
  switch (d) {
    case 64: return launch_merge_d<64>(o_parts, lse_parts, num_parts, rows, o_stride, lse_stride, o, lse, o_fp32, stream);
    case 96: return launch_merge_d<96>(o_parts, lse_parts, num_parts, rows, o_stride, lse_stride, o, lse, o_fp32, stream);
    case 128: return launch_merge_d<128>(o_parts, lse_parts, num_parts, rows, o_stride, lse_stride, o, lse, o_fp32, stream);
    case 256: return launch_merge_d<256>(o_parts, lse_parts, num_parts, rows, o_stride, lse_stride, o, lse, o_fp32, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace attn_sm100
