// attn_q8_sm100.cu — 8-bit attention forward in the manner of the page
// "Makale Bülteni — SageAttention" (section "İddia ve Gerçeklik:
// SageAttention"): the first GEMM (Q K^T) runs on INT8 tensor cores after K is
// mean-centred ("smoothing" — lossless, softmax is shift invariant), the
// second (P V) on FP8 because P already lies in [0, 1]; accumulation stays in
// fp32.
//
// Steps (one stream, four launches):
//   1. kv_stats   per 128-token chunk: fp64 partial sums of K (per channel),
//                 partial max |V| (per channel); the FP8 Q K^T variant (no
//                 smoothing) reads V only
//   2. kv_final   K channel mean kbar (fp64 sum / Nkv, rounded once to fp32),
//                 V channel scale sv = max|V| / 448
//   3. quantize   Q -> INT8, one fp32 scale per 128-token block, plus
//                 qk_i = q_i . kbar (to undo the smoothing shift in LSE);
//                 K - kbar -> INT8 per 128-token block; V / sv -> e4m3
//   4. main       the fused forward: S = Q8 K8^T (kind::i8, s32 in TMEM),
//                 online softmax on s * sq * sk * scale with a reference
//                 maximum that may lag the row maximum by up to 2^4 (so O
//                 is rescaled only rarely), P -> e4m3(p * 448 / 16) (p <= 16)
//                 written back to TMEM, O += P8 V8 (kind::f8f6f4, fp32 in
//                 TMEM), O = O * sv / (28 l), LSE += scale * qk.
// Every quantisation decision (scale, code) is taken in fp32 with correctly
// rounded division and round-half-even, so the codes are reproducible.
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include <utility>

#include "attn_internal.h"
#include "sm100_ptx.cuh"

namespace attn_sm100 {

namespace {

constexpr int kQ8Threads = 320;
// Exponentials of the softmax: of every 8 groups of 4, the first kPolyOf8 are
// evaluated by exp2_poly2 on the FMA pipe, the rest by ex2.approx. The 8-bit
// softmax's e4m3 packing competes with ex2 for issue, so moving some of the
// exponentials off it pays. Measured on the B200 (8k causal outlier workload,
// main kernel): FP8 Q K^T 0.806 / 0.797 / 0.824 / 0.859 / 0.945 ms for 1 / 2 /
// 3 / 4 / 5 of 8; INT8 0.904 ms for 2 of 8, 0.910 for 3. (The same fraction in
// runs of 16 groups, e.g. the first 4 of 16, is slower than 2 of every 8.)
constexpr int kPolyOf8 = 2;
constexpr int kTok = 128;         // tokens per quantisation block == MMA tile rows
constexpr int kPrepThreads = 256;

// Programmatic dependent launch: the four launches of a call form a chain in
// which each may be scheduled while its predecessor's last CTAs still run.
// A kernel lets its dependent launch once all its CTAs have started, and
// waits for its predecessor's completion (and memory) before it reads
// anything the predecessor wrote; both are no-ops without the launch attribute.
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ void unpack8(const uint4& u, float (&f)[8]) {
  f[0] = bf16_lo(u.x); f[1] = bf16_hi(u.x);
  f[2] = bf16_lo(u.y); f[3] = bf16_hi(u.y);
  f[4] = bf16_lo(u.z); f[5] = bf16_hi(u.z);
  f[6] = bf16_lo(u.w); f[7] = bf16_hi(u.w);
}

// x / s rounded to nearest, without a division per element: with r = RN(1/s)
// (computed once per scale), q0 = RN(x * r) is within an ulp of x / s, the
// residual x - q0 * s is exact in one FMA, and RN(q0 + residual * r) is the
// correctly rounded quotient for normal operands (Markstein's FMA correction,
// P. Markstein, IBM J. Res. Dev. 34(1), 1990). The prepass tests compare the
// resulting codes bit for bit with division on the host.
__device__ __forceinline__ float div_rn(float x, float s, float r) {
  const float q0 = x * r;
  const float e = fmaf(-q0, s, x);
  return fmaf(e, r, q0);
}

// Low bytes of four words, packed: result byte i = byte 0 of word i.
__device__ __forceinline__ uint32_t low_bytes4(uint32_t w0, uint32_t w1, uint32_t w2, uint32_t w3) {
  uint32_t a, b, r;
  asm("prmt.b32 %0, %1, %2, 0x0040;" : "=r"(a) : "r"(w0), "r"(w1));
  asm("prmt.b32 %0, %1, %2, 0x0040;" : "=r"(b) : "r"(w2), "r"(w3));
  asm("prmt.b32 %0, %1, %2, 0x5410;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

// INT8 code of x / s as the low byte of a float: for |y| < 2^22, y + 1.5 * 2^23
// is rounded to an integer, half to even (the float's unit in the last place is
// 1 there), and its bits are 0x4B400000 + round(y), whose low byte is the
// two's-complement code. With s = RN(amax / 127) and |x| <= amax, |x / s| <=
// 127 (1 + 2^-23) rounds to at most 127 in magnitude, so the clamp to +-127 of
// the method never changes a code.
__device__ __forceinline__ uint32_t i8_code_word(float x, float s, float r) {
  return __float_as_uint(div_rn(x, s, r) + 12582912.0f);
}

// Block-wide max of non-negative floats (256 threads).
__device__ __forceinline__ float block_max256(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  const int w = threadIdx.x >> 5;
  __syncthreads();
  if ((threadIdx.x & 31) == 0) red[w] = v;
  __syncthreads();
  float m = red[0];
#pragma unroll
  for (int i = 1; i < kPrepThreads / 32; ++i) m = fmaxf(m, red[i]);
  return m;
}

// ----------------------------------------------------------------- prepass 1
// F8 = true (no smoothing): K is not read; only the V maxima are formed.
template <int D, bool F8>
__global__ void __launch_bounds__(kPrepThreads)
    q8_kv_stats_kernel(const uint16_t* __restrict__ k, const uint16_t* __restrict__ v, int Nkv,
                       int nkb, double* __restrict__ ksum_part, float* __restrict__ vmax_part) {
  constexpr int VPR = D / 8;              // 16-byte vectors per row
  constexpr int RPP = kPrepThreads / VPR;  // rows per pass
  __shared__ double ssum[RPP][D];
  __shared__ float smax[RPP][D];
  const int tid = threadIdx.x, vc = tid % VPR, rs = tid / VPR;
  const size_t bh = (size_t)blockIdx.z * gridDim.y + blockIdx.y;
  const int t0 = blockIdx.x * kTok;
  pdl_launch_dependents();
  double s[8];
  float mx[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) { s[i] = 0.0; mx[i] = 0.0f; }
  constexpr int NP = kTok / RPP;
  uint4 kv[NP], vv[NP];
#pragma unroll
  for (int pp = 0; pp < NP; ++pp) {  // issue every load of the chunk before using any
    const int t = t0 + rs + pp * RPP;
    const size_t off = (bh * Nkv + (t < Nkv ? t : 0)) * D + vc * 8;
    kv[pp] = (!F8 && t < Nkv) ? *reinterpret_cast<const uint4*>(k + off) : make_uint4(0, 0, 0, 0);
    vv[pp] = t < Nkv ? *reinterpret_cast<const uint4*>(v + off) : make_uint4(0, 0, 0, 0);
  }
#pragma unroll
  for (int pp = 0; pp < NP; ++pp) {
    float kf[8], vf[8];
    unpack8(kv[pp], kf);
    unpack8(vv[pp], vf);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if (!F8) s[i] += static_cast<double>(kf[i]);
      mx[i] = fmaxf(mx[i], fabsf(vf[i]));
    }
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    if (!F8) ssum[rs][vc * 8 + i] = s[i];
    smax[rs][vc * 8 + i] = mx[i];
  }
  __syncthreads();
  if (tid < D) {
    double acc = 0.0;
    float m = 0.0f;
    for (int r = 0; r < RPP; ++r) {
      if (!F8) acc += ssum[r][tid];
      m = fmaxf(m, smax[r][tid]);
    }
    if (!F8) ksum_part[(bh * nkb + blockIdx.x) * D + tid] = acc;
    vmax_part[(bh * nkb + blockIdx.x) * D + tid] = m;
  }
}

// ----------------------------------------------------------------- prepass 2
// Grid (B * Hkv, D / 32), 256 threads: 32 channels x 8 slices; slice u sums the
// chunk partials u, u + 8, ... of its channel, the 8 slice sums are added in
// slice order. F8 = true (FP8 Q K^T with block scales, no smoothing): kbar is zero.
constexpr int kFinalSlices = 8;
template <int D, bool F8>
__global__ void __launch_bounds__(32 * kFinalSlices)
    q8_kv_final_kernel(const double* __restrict__ ksum_part, const float* __restrict__ vmax_part, int Nkv,
                       int nkb, float* __restrict__ kbar, float* __restrict__ sv) {
  __shared__ double ss[kFinalSlices][32];
  __shared__ float sm[kFinalSlices][32];
  const size_t bh = blockIdx.x;
  const int c = blockIdx.y * 32 + (threadIdx.x & 31);
  const int u = threadIdx.x >> 5;
  pdl_launch_dependents();
  pdl_wait();  // the statistics' partials
  double acc = 0.0;
  float m = 0.0f;
  for (int i = u; i < nkb; i += kFinalSlices) {
    if (!F8) acc += ksum_part[(bh * nkb + i) * D + c];  // (F8: not written by the statistics)
    m = fmaxf(m, vmax_part[(bh * nkb + i) * D + c]);
  }
  ss[u][threadIdx.x & 31] = acc;
  sm[u][threadIdx.x & 31] = m;
  __syncthreads();
  if (u == 0) {
    acc = 0.0;
    m = 0.0f;
#pragma unroll
    for (int w = 0; w < kFinalSlices; ++w) {
      acc += ss[w][threadIdx.x];
      m = fmaxf(m, sm[w][threadIdx.x]);
    }
    kbar[bh * D + c] = F8 ? 0.0f : static_cast<float>(acc / static_cast<double>(Nkv));
    sv[bh * D + c] = m > 0.0f ? __fdiv_rn(m, 448.0f) : 1.0f;
  }
}

// ----------------------------------------------------------------- prepass 3
// Packs 8 codes of x / s (quotients rounded to nearest): INT8 (round half to
// even, clamped to +-127) or, with F8, e4m3 (round to nearest even, saturating).
template <bool F8>
__device__ __forceinline__ uint2 codes8(const float (&x)[8], float s, float r) {
  if (F8) {
    float y[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) y[i] = div_rn(x[i], s, r);
    return make_uint2(pack_e4m3x2(y[0], y[1]) | (pack_e4m3x2(y[2], y[3]) << 16),
                      pack_e4m3x2(y[4], y[5]) | (pack_e4m3x2(y[6], y[7]) << 16));
  }
  return make_uint2(low_bytes4(i8_code_word(x[0], s, r), i8_code_word(x[1], s, r), i8_code_word(x[2], s, r),
                               i8_code_word(x[3], s, r)),
                    low_bytes4(i8_code_word(x[4], s, r), i8_code_word(x[5], s, r), i8_code_word(x[6], s, r),
                               i8_code_word(x[7], s, r)));
}

// One CTA per 128-token block: Q blocks (B * Hq * nqb), then K blocks and V
// blocks (B * Hkv * nkb each). A thread keeps its rows' raw bf16 vectors in
// registers (all its loads in flight before the first use) and unpacks them
// where they are used.
template <int D, bool F8>
__global__ void __launch_bounds__(kPrepThreads, 4)  // 4 CTAs per SM hide the loads' latency
    q8_quantize_kernel(const uint16_t* __restrict__ q, const uint16_t* __restrict__ k,
                       const uint16_t* __restrict__ v, int B, int Hq, int Hkv, int Nq, int Nkv,
                       int nqb, int nkb, const float* __restrict__ kbar,
                       const float* __restrict__ sv, int8_t* __restrict__ q8,
                       int8_t* __restrict__ k8, uint8_t* __restrict__ v8, float* __restrict__ sq,
                       float* __restrict__ sk, float* __restrict__ qk) {
  constexpr int VPR = D / 8;
  constexpr int RPP = kPrepThreads / VPR;
  constexpr int NP = kTok / RPP;  // passes
  __shared__ float red[kPrepThreads / 32];
  const int tid = threadIdx.x, vc = tid % VPR, rs = tid / VPR;
  const long long n_q_tiles = (long long)B * Hq * nqb;
  const long long n_k_tiles = (long long)B * Hkv * nkb;
  long long tile = blockIdx.x;
  uint4 raw[NP];
  pdl_launch_dependents();
  if (tile < n_q_tiles) {
    const int qb = (int)(tile % nqb);
    const long long bh = tile / nqb;  // b * Hq + h
    const int b = (int)(bh / Hq), h = (int)(bh % Hq);
    const size_t bhk = (size_t)b * Hkv + h / (Hq / Hkv);
#pragma unroll
    for (int pp = 0; pp < NP; ++pp) {
      const int t = qb * kTok + rs + pp * RPP;
      raw[pp] = t < Nq ? *reinterpret_cast<const uint4*>(q + ((size_t)bh * Nq + t) * D + vc * 8)
                       : make_uint4(0, 0, 0, 0);
    }
    pdl_wait();  // kbar (the raw Q loads above are already in flight)
    float kb[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) kb[i] = kbar[bhk * D + vc * 8 + i];
    float amax = 0.0f;
#pragma unroll
    for (int pp = 0; pp < NP; ++pp) {
      float x[8];
      unpack8(raw[pp], x);
#pragma unroll
      for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(x[i]));
    }
    amax = block_max256(amax, red);
    const float s = amax > 0.0f ? __fdiv_rn(amax, F8 ? 448.0f : 127.0f) : 1.0f;
    const float r_q = __frcp_rn(s);
#pragma unroll
    for (int pp = 0; pp < NP; ++pp) {
      const int t = qb * kTok + rs + pp * RPP;
      float x[8];
      unpack8(raw[pp], x);
      float dot = 0.0f;
#pragma unroll
      for (int i = 0; i < 8; ++i) dot = fmaf(x[i], kb[i], dot);
#pragma unroll
      for (int o = VPR / 2; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
      if (t < Nq) {
        *reinterpret_cast<uint2*>(q8 + ((size_t)bh * Nq + t) * D + vc * 8) = codes8<F8>(x, s, r_q);
        if (vc == 0) qk[(size_t)bh * Nq + t] = dot;
      }
    }
    if (tid == 0) sq[(size_t)bh * nqb + qb] = s;
  } else if (tile < n_q_tiles + n_k_tiles) {
    tile -= n_q_tiles;
    const int kb_i = (int)(tile % nkb);
    const size_t bh = (size_t)(tile / nkb);  // b * Hkv + h
#pragma unroll
    for (int pp = 0; pp < NP; ++pp) {
      const int t = kb_i * kTok + rs + pp * RPP;
      raw[pp] = t < Nkv ? *reinterpret_cast<const uint4*>(k + (bh * Nkv + t) * D + vc * 8) : make_uint4(0, 0, 0, 0);
    }
    pdl_wait();  // kbar
    float kb[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) kb[i] = kbar[bh * D + vc * 8 + i];
    float amax = 0.0f;
#pragma unroll
    for (int pp = 0; pp < NP; ++pp) {
      const int t = kb_i * kTok + rs + pp * RPP;
      if (t < Nkv) {
        float xk[8];
        unpack8(raw[pp], xk);
#pragma unroll
        for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(xk[i] - kb[i]));
      }
    }
    amax = block_max256(amax, red);
    const float s = amax > 0.0f ? __fdiv_rn(amax, F8 ? 448.0f : 127.0f) : 1.0f;
    const float r_s = __frcp_rn(s);
#pragma unroll
    for (int pp = 0; pp < NP; ++pp) {
      const int t = kb_i * kTok + rs + pp * RPP;
      if (t < Nkv) {
        float xk[8];
        unpack8(raw[pp], xk);
#pragma unroll
        for (int i = 0; i < 8; ++i) xk[i] = xk[i] - kb[i];
        *reinterpret_cast<uint2*>(k8 + (bh * Nkv + t) * D + vc * 8) = codes8<F8>(xk, s, r_s);
      }
    }
    if (tid == 0) sk[bh * nkb + kb_i] = s;
  } else {
    tile -= n_q_tiles + n_k_tiles;
    const int kb_i = (int)(tile % nkb);
    const size_t bh = (size_t)(tile / nkb);  // b * Hkv + h
#pragma unroll
    for (int pp = 0; pp < NP; ++pp) {
      const int t = kb_i * kTok + rs + pp * RPP;
      raw[pp] = t < Nkv ? *reinterpret_cast<const uint4*>(v + (bh * Nkv + t) * D + vc * 8) : make_uint4(0, 0, 0, 0);
    }
    pdl_wait();  // sv
    float svc[8], rsv[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      svc[i] = sv[bh * D + vc * 8 + i];
      rsv[i] = __frcp_rn(svc[i]);
    }
#pragma unroll
    for (int pp = 0; pp < NP; ++pp) {
      const int t = kb_i * kTok + rs + pp * RPP;
      if (t < Nkv) {
        float vf[8], y[8];
        unpack8(raw[pp], vf);
#pragma unroll
        for (int i = 0; i < 8; ++i) y[i] = div_rn(vf[i], svc[i], rsv[i]);
        const uint32_t w0 = pack_e4m3x2(y[0], y[1]) | (pack_e4m3x2(y[2], y[3]) << 16);
        const uint32_t w1 = pack_e4m3x2(y[4], y[5]) | (pack_e4m3x2(y[6], y[7]) << 16);
        *reinterpret_cast<uint2*>(v8 + (bh * Nkv + t) * D + vc * 8) = make_uint2(w0, w1);
      }
    }
  }
}

// ----------------------------------------------------------------- main kernel
template <int D>
struct Q8Cfg {
  static constexpr int kTileBytes = kTok * D;  // 8-bit tile: 128 rows x D bytes
  static constexpr int kStages = 8;
  static constexpr int kOffQ = 0;
  static constexpr int kOffRing = 2 * kTileBytes;
  static constexpr int kOffBar = kOffRing + kStages * kTileBytes;
  static constexpr int kOffSv = kOffBar + 512;
  static constexpr int kSmemBytes = kOffBar + 1024 + 1024;
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kColS0 = 0, kColS1 = 128;
  static constexpr uint32_t kColO0 = 256, kColO1 = 256 + D;
  static constexpr int kOutBoxBytes = 128 * 128;  // bf16 output box: 128 rows x 64 columns
};

struct Q8Bar {
  static constexpr int kFull = 0, kEmpty = 8, kQFull = 16, kSFull = 17, kPFull = 19,
                       kOFinal = 21, kEpi = 22, kDrain = 24, kSInit = 25;
  static constexpr int kTmemSlotByte = 8 * 32;
  static constexpr int kAbortByte = 8 * 32 + 4;
};

__device__ __forceinline__ void q8_flag_abort(volatile int* abort_flag, int* status, int where) {
  *abort_flag = 1;
  if (atomicCAS(status, 0, ATTN_ERR_TIMEOUT) == 0) status[1] = where;
}

__device__ __forceinline__ bool q8_warp_all(bool v) { return __all_sync(0xffffffffu, v) != 0; }

// Columns of an INT8 score tile that the MMA writes from zero: P (128 e4m3 per
// row) is stored over them, so they are in use until P.V has read P. The other
// kTok - kPCols columns are pre-set by the softmax threads to the bits of
// M = 1.5 * 2^23 and accumulated onto (see the softmax's s32 -> fp32 note).
constexpr int kPCols = kTok / 4;

// S = Q8 K8^T: INT8 (s32 accumulation) or, with F8, e4m3 (fp32 accumulation).
// INT8: keys [0, kPCols) into columns [0, kPCols) from zero, keys [kPCols, kTok)
// accumulated onto the pre-set columns [kPCols, kTok).
template <int D, bool F8>
__device__ __forceinline__ void issue_qk_i8(uint32_t d_tmem, uint32_t q_smem, uint32_t k_smem) {
  if constexpr (F8) {
    constexpr uint32_t idesc = idesc_e4m3_f32(128, 128);
#pragma unroll
    for (int kk = 0; kk < D / 32; ++kk) {
      const uint64_t a = smem_desc_sw(q_smem + kk * 32, 16, 8 * D, D);
      const uint64_t b = smem_desc_sw(k_smem + kk * 32, 16, 8 * D, D);
      mma_f8_ss(d_tmem, a, b, idesc, kk > 0 ? 1u : 0u);
    }
  } else {
    constexpr uint32_t idesc_p = idesc_s8_s32(128, kPCols);
    constexpr uint32_t idesc_rest = idesc_s8_s32(128, kTok - kPCols);
    // key row r of the tile starts at r * D bytes; kPCols rows are whole swizzle atoms
    const uint32_t k_rest = k_smem + kPCols * D;
#pragma unroll
    for (int kk = 0; kk < D / 32; ++kk) {
      const uint64_t a = smem_desc_sw(q_smem + kk * 32, 16, 8 * D, D);
      mma_i8_ss(d_tmem, a, smem_desc_sw(k_smem + kk * 32, 16, 8 * D, D), idesc_p, kk > 0 ? 1u : 0u);
      mma_i8_ss(d_tmem + kPCols, a, smem_desc_sw(k_rest + kk * 32, 16, 8 * D, D), idesc_rest, 1u);
    }
  }
}

template <int D>
__device__ __forceinline__ void issue_pv_f8(uint32_t o_tmem, uint32_t p_tmem, uint32_t v_smem,
                                            bool accumulate) {
  constexpr uint32_t idesc = idesc_e4m3_f32_bmn(128, D);
#pragma unroll
  for (int kk = 0; kk < kTok / 32; ++kk) {
    const uint64_t b = smem_desc_sw(v_smem + kk * 32 * D, kTok * D, 8 * D, D);
    mma_f8_ts(o_tmem, p_tmem + kk * 8, b, idesc, (accumulate || kk > 0) ? 1u : 0u);
  }
}

template <int D, bool F8>
__global__ void __launch_bounds__(kQ8Threads, 1)
    attn_fwd_q8_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                       const Q8Params p) {
  using C = Q8Cfg<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_base = smem_addr(smem_raw);
  const uint32_t base = (raw_base + 1023u) & ~1023u;
  uint8_t* const base_ptr = smem_raw + (base - raw_base);
  const uint32_t sQ = base + C::kOffQ;
  const uint32_t sRing = base + C::kOffRing;
  const uint32_t sBar = base + C::kOffBar;
  auto bar = [&](int slot) -> uint32_t { return sBar + 8u * slot; };
  uint32_t* const tmem_slot = reinterpret_cast<uint32_t*>(base_ptr + C::kOffBar + Q8Bar::kTmemSlotByte);
  volatile int* const abort_flag = reinterpret_cast<volatile int*>(base_ptr + C::kOffBar + Q8Bar::kAbortByte);
  float* const sv_smem = reinterpret_cast<float*>(base_ptr + C::kOffSv);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // causal: row blocks heaviest first across groups of heads (see grouped_heavy_first)
  int ux, hq, b;
  grouped_heavy_first(p.lpt_group, ux, hq, b);
  const int row_block = p.causal ? (p.num_row_blocks - 1 - ux) : ux;
  const int hk = hq / (p.Hq / p.Hkv);
  const int q0 = row_block * 2 * kTok;
  const int bh_q = b * p.Hq + hq;
  const int bh_kv = b * p.Hkv + hk;
  // causal mask aligned to the bottom right: key j visible to query i iff
  // j <= i + (Nkv - Nq); at least one K/V tile per unit (a row that sees no key
  // ends with l = 0, O = 0, LSE = -inf)
  const int diag = p.causal ? p.Nkv - p.Nq : 0;
  int n_tiles;
  if (p.causal) {
    const int last_key = min(min(q0 + 2 * kTok - 1, p.Nq - 1) + diag, p.Nkv - 1);
    n_tiles = last_key < 0 ? 1 : last_key / kTok + 1;
  } else {
    n_tiles = (p.Nkv + kTok - 1) / kTok;
  }
  const uint64_t budget = p.timeout_ns;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(bar(Q8Bar::kFull + s), 1);
      mbar_init(bar(Q8Bar::kEmpty + s), 1);
    }
    mbar_init(bar(Q8Bar::kQFull), 1);
    for (int t = 0; t < 2; ++t) {
      mbar_init(bar(Q8Bar::kSFull + t), 1);
      mbar_init(bar(Q8Bar::kPFull + t), 4);  // one arrival per softmax warp
      mbar_init(bar(Q8Bar::kEpi + t), 128);
    }
    mbar_init(bar(Q8Bar::kOFinal), 1);
    mbar_init(bar(Q8Bar::kDrain), 1);
    mbar_init(bar(Q8Bar::kSInit), 8);  // one arrival per softmax warp
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  pdl_wait();  // the prepass's codes, scales and q.kbar
  if (threadIdx.x < D) sv_smem[threadIdx.x] = p.sv[(size_t)bh_kv * D + threadIdx.x];
  if (warp == 8) {
    tmem_alloc(smem_addr(tmem_slot), C::kTmemCols);
    tmem_relinquish();
  }
  if (warp == 9 && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
    tma_prefetch_desc(&tm_o);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 9) {
    // ------------------------------------------------------------ TMA producer
    bool ok = true;
    uint32_t issued = 0;
    if (lane == 0) {
      mbar_arrive_expect_tx(bar(Q8Bar::kQFull), 2 * C::kTileBytes);
      for (int t = 0; t < 2; ++t)
        tma_load_3d(sQ + t * C::kTileBytes, &tm_q, bar(Q8Bar::kQFull), 0, q0 + t * kTok, bh_q);
    }
    for (int j = 0; j < n_tiles && ok; ++j) {
      for (int which = 0; which < 2; ++which) {
        const uint32_t stage = issued % C::kStages;
        const uint32_t phase = (issued / C::kStages) & 1u;
        ok = q8_warp_all(bounded_wait(bar(Q8Bar::kEmpty + stage), phase ^ 1u, abort_flag, budget));
        if (!ok) break;
        if (lane == 0) {
          const uint32_t fb = bar(Q8Bar::kFull + stage);
          mbar_arrive_expect_tx(fb, C::kTileBytes);
          tma_load_3d(sRing + stage * C::kTileBytes, which ? &tm_v : &tm_k, fb, 0, j * kTok, bh_kv);
        }
        __syncwarp();
        ++issued;
      }
    }
    if (!ok) {
      if (lane == 0) {
        q8_flag_abort(abort_flag, p.status, 0x1100);
        volatile int no_abort = 0;
        bounded_wait(bar(Q8Bar::kQFull), 0, &no_abort, budget);
        const uint32_t first = issued > (uint32_t)C::kStages ? issued - C::kStages : 0u;
        for (uint32_t i = first; i < issued; ++i)
          bounded_wait(bar(Q8Bar::kFull + i % C::kStages), (i / C::kStages) & 1u, &no_abort, budget);
      }
      __syncwarp();
    }
  } else if (warp == 8) {
    // ------------------------------------------------------------ MMA issuer
    const uint32_t tS[2] = {tmem + C::kColS0, tmem + C::kColS1};
    const uint32_t tO[2] = {tmem + C::kColO0, tmem + C::kColO1};
    const uint32_t q_smem[2] = {sQ, sQ + C::kTileBytes};
    bool ok = q8_warp_all(bounded_wait(bar(Q8Bar::kQFull), 0, abort_flag, budget));
    // INT8: the softmax threads pre-set the accumulated score columns before S(0)
    if (!F8 && ok) ok = q8_warp_all(bounded_wait(bar(Q8Bar::kSInit), 0, abort_flag, budget));
    uint32_t slot = 0, v_prev_stage = 0;
    int j = 0;
    for (; j < n_tiles && ok; ++j) {
      const uint32_t k_stage = slot % C::kStages, k_phase = (slot / C::kStages) & 1u;
      ++slot;
      const uint32_t v_stage = slot % C::kStages;
      ++slot;
      const uint32_t k_smem = sRing + k_stage * C::kTileBytes;
      ok = q8_warp_all(bounded_wait(bar(Q8Bar::kFull + k_stage), k_phase, abort_flag, budget));
      if (!ok) break;
      if (j > 0) {
        const uint32_t vp_slot = slot - 3;
        ok = q8_warp_all(bounded_wait(bar(Q8Bar::kPFull + 0), (j - 1) & 1, abort_flag, budget) &&
                         bounded_wait(bar(Q8Bar::kFull + v_prev_stage), (vp_slot / C::kStages) & 1u,
                                      abort_flag, budget));
        if (!ok) break;
        tc_fence_after();
        if (lane == 0) issue_pv_f8<D>(tO[0], tS[0], sRing + v_prev_stage * C::kTileBytes, j - 1 > 0);
      }
      tc_fence_after();
      if (lane == 0) {
        issue_qk_i8<D, F8>(tS[0], q_smem[0], k_smem);
        tc_commit(bar(Q8Bar::kSFull + 0));
      }
      __syncwarp();
      if (j > 0) {
        ok = q8_warp_all(bounded_wait(bar(Q8Bar::kPFull + 1), (j - 1) & 1, abort_flag, budget));
        if (!ok) break;
        tc_fence_after();
        if (lane == 0) {
          issue_pv_f8<D>(tO[1], tS[1], sRing + v_prev_stage * C::kTileBytes, j - 1 > 0);
          tc_commit(bar(Q8Bar::kEmpty + v_prev_stage));
        }
      }
      if (lane == 0) {
        issue_qk_i8<D, F8>(tS[1], q_smem[1], k_smem);
        tc_commit(bar(Q8Bar::kSFull + 1));
        tc_commit(bar(Q8Bar::kEmpty + k_stage));
      }
      __syncwarp();
      v_prev_stage = v_stage;
    }
    if (ok) {
      const int jl = n_tiles - 1;
      const uint32_t vp_slot = slot - 1;
      ok = q8_warp_all(bounded_wait(bar(Q8Bar::kPFull + 0), jl & 1, abort_flag, budget) &&
                       bounded_wait(bar(Q8Bar::kFull + v_prev_stage), (vp_slot / C::kStages) & 1u,
                                    abort_flag, budget));
      if (ok) {
        tc_fence_after();
        if (lane == 0) issue_pv_f8<D>(tO[0], tS[0], sRing + v_prev_stage * C::kTileBytes, jl > 0);
        __syncwarp();
        ok = q8_warp_all(bounded_wait(bar(Q8Bar::kPFull + 1), jl & 1, abort_flag, budget));
        if (ok) {
          tc_fence_after();
          if (lane == 0) {
            issue_pv_f8<D>(tO[1], tS[1], sRing + v_prev_stage * C::kTileBytes, jl > 0);
            tc_commit(bar(Q8Bar::kEmpty + v_prev_stage));
            tc_commit(bar(Q8Bar::kOFinal));
          }
          __syncwarp();
        }
      }
    }
    if (!ok) {
      if (lane == 0) {
        q8_flag_abort(abort_flag, p.status, 0x1200 | (j << 12));
        tc_commit(bar(Q8Bar::kDrain));
        volatile int no_abort = 0;
        bounded_wait(bar(Q8Bar::kDrain), 0, &no_abort, budget);
      }
      __syncwarp();
    }
  } else {
    // ------------------------------------------------------------ softmax / epilogue
    const int t = warp >> 2;
    const int wq = warp & 3;
    const int r = (wq << 5) | lane;
    const uint32_t lane_off = static_cast<uint32_t>(wq << 5) << 16;
    const uint32_t tS = tmem + (t ? C::kColS1 : C::kColS0) + lane_off;
    const uint32_t tO = tmem + (t ? C::kColO1 : C::kColO0) + lane_off;
    const int row = q0 + t * kTok + r;
    const int qtile = (q0 >> 7) + t;
    // a tile wholly past Nq has no scale; its rows are computed but never stored
    const float sq_t = qtile < p.nqb ? p.sq[(size_t)bh_q * p.nqb + qtile] : 1.0f;
    const float kLog2_448 = 8.807354922057604f;  // log2(448)
    // the reference maximum may lag the row maximum by up to kLag (log2 units):
    // P is encoded as 2^(t - m_ref) * 448 * 2^-kLag <= 448, and O is rescaled
    // only when a tile's maximum exceeds m_ref + kLag
    constexpr float kLag = 4.0f;

    // s32 -> fp32 without a conversion instruction: |s| <= 127 * 127 * d < 2^22,
    // so the bits of (s + 0x4B400000) are the float M + s exactly, M = 1.5 * 2^23.
    // The MMA adds s onto columns [kPCols, kTok) pre-set to 0x4B400000 (here for
    // S(0), after each read of S for the next tile); the columns P is stored over
    // get the integer add in registers. (The e4m3 MMA accumulates in fp32: no bias.)
    constexpr uint32_t kMagicBits = 0x4B400000u;
    if (!F8) {
#pragma unroll
      for (int c = kPCols; c < kTok; c += 32) tmem_fill32(tS + c, kMagicBits);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(Q8Bar::kSInit));
    }

    float m_run = -INFINITY;  // reference maximum of scale*log2(e)*S: within kLag below the row maximum
    float l_run = 0.0f;       // sum of 448 * 2^-kLag * 2^(. - m_run)
    bool ok = true;
    int j = 0;
    // the K block scale of the next tile is loaded a step ahead (off the chain)
    const float* const sk_row = p.sk + (size_t)bh_kv * p.nkb;
    float sk_next = __ldg(sk_row);
    for (; j < n_tiles; ++j) {
      const float sk_j = sk_next;
      if (j + 1 < n_tiles) sk_next = __ldg(sk_row + j + 1);
      ok = q8_warp_all(bounded_wait(bar(Q8Bar::kSFull + t), j & 1, abort_flag, budget));
      if (!ok) break;
      tc_fence_after();
      uint32_t sr[128];
#pragma unroll
      for (int c = 0; c < 4; ++c)
        tmem_ld32(tS + 32 * c, *reinterpret_cast<uint32_t(*)[32]>(&sr[32 * c]));
      tmem_wait_ld();
      const float f = sq_t * sk_j * p.scale_log2;
      // The floats M + s order like s (same binade), so the row maximum is taken
      // on them, and M * f is folded into the exponent's bias below.
      constexpr float kMagic = 12582912.0f;
      constexpr float kOff = F8 ? 0.0f : kMagic;
#pragma unroll
      for (int c = 0; c < (F8 ? 0 : kPCols); ++c) sr[c] += kMagicBits;
      const int kv0 = j * kTok;
      const bool tile_masked =
          (kv0 + kTok > p.Nkv) || (p.causal && kv0 + kTok - 1 > q0 + t * kTok + diag);
      if (tile_masked) {
        int lim = p.Nkv - kv0;
        if (p.causal) lim = min(lim, row + diag - kv0 + 1);
#pragma unroll
        for (int c = 0; c < kTok; ++c)
          if (c >= lim) sr[c] = __float_as_uint(-INFINITY);
      }
      float mx0 = -INFINITY, mx1 = -INFINITY, mx2 = -INFINITY, mx3 = -INFINITY;
#pragma unroll
      for (int c = 0; c < kTok; c += 8) {
        mx0 = fmax3(mx0, __uint_as_float(sr[c]), __uint_as_float(sr[c + 1]));
        mx1 = fmax3(mx1, __uint_as_float(sr[c + 2]), __uint_as_float(sr[c + 3]));
        mx2 = fmax3(mx2, __uint_as_float(sr[c + 4]), __uint_as_float(sr[c + 5]));
        mx3 = fmax3(mx3, __uint_as_float(sr[c + 6]), __uint_as_float(sr[c + 7]));
      }
      // f > 0 (all scales positive), so the max of s*f is f * max(s); M + max(s) - M is exact
      const float m_tile = (fmax3(mx0, mx1, fmaxf(mx2, mx3)) - kOff) * f;
      float alpha = 1.0f;
      if (m_tile > m_run + kLag) {
        alpha = ex2_approx(m_run - m_tile);
        m_run = m_tile;
      }
      const float mb = (m_run == -INFINITY) ? 0.0f : m_run;
      // p = 448 * 2^-kLag * 2^(s*f - m) = 2^(s*f - m + log2 448 - kLag) <= 448, evaluated
      // as (M + s) * f + (log2 448 - kLag - m - M * f): the bias is rounded once, by at
      // most half an ulp of M * f <= 0.75 f, i.e. below one unit of the integer score
      const float b0 = fmaf(-kOff, f, kLog2_448 - kLag - mb);
      const float2 slope = make_float2(f, f), bias = make_float2(b0, b0);
      float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                       make_float2(0.f, 0.f)};
#pragma unroll
      for (int qd = 0; qd < kTok / 4; ++qd) {
        const float2 x0 = fma2(make_float2(__uint_as_float(sr[4 * qd]), __uint_as_float(sr[4 * qd + 1])),
                               slope, bias);
        const float2 x1 = fma2(make_float2(__uint_as_float(sr[4 * qd + 2]), __uint_as_float(sr[4 * qd + 3])),
                               slope, bias);
        float2 e0, e1;
        if ((qd & 7) < kPolyOf8) {  // arguments <= log2 448; masked ones (-inf) give ~2^-125
          e0 = exp2_poly2(x0);
          e1 = exp2_poly2(x1);
        } else {
          e0 = make_float2(ex2_approx(x0.x), ex2_approx(x0.y));
          e1 = make_float2(ex2_approx(x1.x), ex2_approx(x1.y));
        }
        acc[qd & 3] = add2(acc[qd & 3], add2(e0, e1));
        sr[qd] = pack_e4m3x2(e0.x, e0.y) | (pack_e4m3x2(e1.x, e1.y) << 16);
      }
      const float2 acc01 = add2(acc[0], acc[1]), acc23 = add2(acc[2], acc[3]);
      const float row_sum = (acc01.x + acc01.y) + (acc23.x + acc23.y);
      tmem_st32(tS, *reinterpret_cast<const uint32_t(*)[32]>(&sr[0]));
      if (!F8) {
        // S(j) has been read: pre-set the accumulated columns for S(j + 1) (the
        // MMA writes them only after this step's P-full arrival)
#pragma unroll
        for (int c = kPCols; c < kTok; c += 32) tmem_fill32(tS + c, kMagicBits);
      }
      const bool rescale = (j > 0) && (alpha != 1.0f);
      if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
          uint32_t o[32];
          tmem_ld32(tO + 32 * c, o);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
          tmem_st32(tO + 32 * c, o);
        }
      }
      l_run = l_run * alpha + row_sum;
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(Q8Bar::kPFull + t));
    }

    if (ok) ok = q8_warp_all(bounded_wait(bar(Q8Bar::kOFinal), 0, abort_flag, budget));
    if (ok) {
      tc_fence_after();
      const float inv_l = l_run > 0.0f ? 1.0f / l_run : 0.0f;
      // The K/V ring is idle once every MMA has completed; stage the bf16 O
      // tile of query tile t in it (32 KiB at d = 128).
      uint8_t* const stage_ptr = base_ptr + C::kOffRing + t * (D / 64) * C::kOutBoxBytes;
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        uint32_t o[32];
        tmem_ld32(tO + 32 * c, o);
        tmem_wait_ld();
#pragma unroll
        for (int qd = 0; qd < 4; ++qd) {
          const int col16 = c * 4 + qd;
          const int bx = col16 >> 3;
          const int ch = col16 & 7;
          float y[8];
#pragma unroll
          for (int i = 0; i < 8; ++i)
            y[i] = __uint_as_float(o[8 * qd + i]) * sv_smem[col16 * 8 + i] * inv_l;
          uint4 v;
          v.x = pack_bf16x2(y[0], y[1]);
          v.y = pack_bf16x2(y[2], y[3]);
          v.z = pack_bf16x2(y[4], y[5]);
          v.w = pack_bf16x2(y[6], y[7]);
          *reinterpret_cast<uint4*>(stage_ptr + bx * C::kOutBoxBytes + r * 128 + ((ch ^ (r & 7)) << 4)) = v;
        }
      }
      fence_proxy_async_smem();
      mbar_arrive(bar(Q8Bar::kEpi + t));
      if (row < p.Nq) {
        // l_run carries the factor 448 * 2^-kLag, which O's numerator also carries
        const float lse2 = m_run + log2f(l_run) - (kLog2_448 - kLag);
        p.lse[(size_t)bh_q * p.Nq + row] =
            lse2 * 0.69314718055994530942f + p.scale * p.qk[(size_t)bh_q * p.Nq + row];
      }
      if (r == 0) {
        volatile int no_abort = 0;
        if (bounded_wait(bar(Q8Bar::kEpi + t), 0, &no_abort, budget)) {
          for (int bx = 0; bx < D / 64; ++bx)
            tma_store_3d(&tm_o, smem_addr(stage_ptr) + bx * C::kOutBoxBytes, bx * 64, q0 + t * kTok, bh_q);
          tma_store_commit();
          tma_store_wait_all();
        } else {
          q8_flag_abort(abort_flag, p.status, 0x1400 | t);
        }
      }
    } else if (lane == 0) {
      q8_flag_abort(abort_flag, p.status, 0x1300 | (t << 8) | (j << 12));
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 8) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

// Launch that may start while the previous kernel on the stream finishes
// (programmatic dependent launch; the kernel waits with pdl_wait before it
// reads the previous kernel's output).
template <typename... KArgs, typename... Args>
cudaError_t launch_dependent(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                             cudaStream_t stream, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

template <int D, bool F8>
cudaError_t launch_q8_d(const Q8Launch& L, cudaStream_t stream) {
  const int nqb = L.p.nqb, nkb = L.p.nkb;
  // the first launch waits for everything before it on the stream (a previous
  // call's main kernel may still read the workspace this call rewrites)
  dim3 g1(nkb, L.Hkv, L.B);
  q8_kv_stats_kernel<D, F8><<<g1, kPrepThreads, 0, stream>>>(
      static_cast<const uint16_t*>(L.k), static_cast<const uint16_t*>(L.v), L.p.Nkv, nkb,
      L.ksum_part, L.vmax_part);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  dim3 g2((unsigned)((long long)L.B * L.Hkv), D / 32);
  e = launch_dependent(q8_kv_final_kernel<D, F8>, g2, dim3(32 * kFinalSlices), 0, stream,
                       (const double*)L.ksum_part, (const float*)L.vmax_part, L.p.Nkv, nkb, L.kbar,
                       const_cast<float*>(L.p.sv));
  if (e != cudaSuccess) return e;
  const long long tiles = (long long)L.B * L.p.Hq * nqb + 2LL * L.B * L.Hkv * nkb;
  e = launch_dependent(q8_quantize_kernel<D, F8>, dim3((unsigned)tiles), dim3(kPrepThreads), 0, stream,
                       static_cast<const uint16_t*>(L.q), static_cast<const uint16_t*>(L.k),
                       static_cast<const uint16_t*>(L.v), L.B, L.p.Hq, L.Hkv, L.p.Nq, L.p.Nkv, nqb,
                       nkb, (const float*)L.kbar, L.p.sv, L.q8, L.k8, L.v8,
                       const_cast<float*>(L.p.sq), const_cast<float*>(L.p.sk),
                       const_cast<float*>(L.p.qk));
  if (e != cudaSuccess || L.prepass_only) return e;
  e = max_dynamic_smem_once<attn_fwd_q8_kernel<D, F8>>(Q8Cfg<D>::kSmemBytes);
  if (e != cudaSuccess) return e;
  dim3 grid(L.p.num_row_blocks, L.p.Hq, L.B);
  return launch_dependent(attn_fwd_q8_kernel<D, F8>, grid, dim3(kQ8Threads), Q8Cfg<D>::kSmemBytes,
                          stream, L.tq, L.tk, L.tv, L.to, L.p);
}

}  // namespace

cudaError_t launch_q8(const Q8Launch& L, int d, cudaStream_t stream) {
  if (L.fp8_qk)
    return d == 128 ? launch_q8_d<128, true>(L, stream) : launch_q8_d<64, true>(L, stream);
  return d == 128 ? launch_q8_d<128, false>(L, stream) : launch_q8_d<64, false>(L, stream);
}

}  // namespace attn_sm100
