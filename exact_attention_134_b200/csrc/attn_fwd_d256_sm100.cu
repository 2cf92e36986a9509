// attn_fwd_d256_sm100.cu — bf16 fused exact attention forward for head dim
// 256 on B200 (sm_100a).
//
// Same computation as attn_fwd_sm100.cu (the definition on "FlashAttention
// (TR)", "Standart Attention Mekanizmasının Sorunları", computed tile by tile
// with the online softmax of "Çevrimiçi Softmax Hesaplama"); that page's
// "FlashAttention-2 (2023)" section extends the head dimension to 256.
//
// At d = 256 one query tile's O accumulator (128 x 256 fp32) fills half of
// tensor memory, so the two-tile layout of the d <= 128 kernel does not fit.
// Layout here, one 128-row query tile per CTA:
//   TMEM (512 columns): Q [0,128) (bf16 pairs, the A operand of S = Q K^T),
//                       S0 [128,192), S1 [192,256) (64 keys each, fp32; P_t
//                       as bf16 over the first 32 columns of S_t),
//                       O [256,512) (fp32, one N = 256 accumulator).
//   Shared memory: a ring of 64-key K/V tiles (32 KB each). Q never touches
//   shared memory: the softmax threads load their rows into registers and
//   store them to TMEM, so S is a TS MMA that reads only K from shared memory.
// Roles (192 threads): warps 0-3 softmax, correction and epilogue (thread =
// query row = TMEM lane), warp 4 MMA issuer, warp 5 TMA producer.
// MMA order: S(0), S(1), PV(0), S(2), PV(1), ... — S(j+1) runs while the
// softmax works on tile j; S(j+1) overwrites P(j-1) only after PV(j-1), which
// was issued before it (tcgen05 MMAs from one thread execute in order). O is
// rescaled only when a row's running maximum moves by more than 2^8, and only
// then does the softmax wait for PV(j-1).
// VL = true: packed variable-length sequences [total, H, d] (grid x = query
// head, (y, z) = the 128-row units of all sequences, see packed_unit; rows
// from cu_seqlens, per-sequence bottom-right causal mask). A K/V tile that
// runs past its sequence reads the next sequence's rows (or the map's zero
// fill past the end); those columns are masked to -inf, so P = 0 there.
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "attn_internal.h"
#include "sm100_ptx.cuh"

namespace attn_sm100 {
namespace {

constexpr int kD = 256;
constexpr int kBM = 128;         // query rows per CTA
constexpr int kBN = 64;          // keys per K/V tile
constexpr int kThreads = 192;
constexpr int kMmaWarp = 4;
constexpr int kLoadWarp = 5;
constexpr int kStages = 6;       // ring slots (K and V tiles alternate)
constexpr int kTileBytes = kBN * kD * 2;   // 32 KB
constexpr int kBoxBytes = kBN * 128;       // 64 rows x 64 columns bf16, 128-byte swizzle
constexpr int kBoxes = kD / 64;
constexpr int kOffBar = kStages * kTileBytes;
constexpr int kSmemBytes = kOffBar + 256 + 1024;  // + base alignment slack
constexpr uint32_t kColQ = 0, kColS0 = 128, kColS1 = 192, kColO = 256;
constexpr float kRescaleThreshold = 8.0f;  // log2 units

struct Bars {
  static constexpr int kFull = 0;     // [kStages]
  static constexpr int kEmpty = 8;    // [kStages]
  static constexpr int kQFull = 16;   // Q stored into TMEM (128 arrivals)
  static constexpr int kSFull = 17;   // [2]
  static constexpr int kPFull = 19;   // [2] (128 arrivals)
  static constexpr int kPVDone = 21;  // one phase per PV(j), j < n - 1
  static constexpr int kOFinal = 22;
  static constexpr int kDrain = 23;
  static constexpr int kTmemSlotByte = 8 * 24;
  static constexpr int kAbortByte = 8 * 24 + 4;
};

__device__ __forceinline__ void flag_abort(volatile int* abort_flag, int* status, int where) {
  *abort_flag = 1;
  if (atomicCAS(status, 0, ATTN_ERR_TIMEOUT) == 0) status[1] = where;
}

__device__ __forceinline__ bool warp_all(bool v) { return __all_sync(0xffffffffu, v) != 0; }

// S[128 x 64] = Q (TMEM, 128 x 256) . K_j^T (K tile: 64 key rows, K-major).
__device__ __forceinline__ void issue_s(uint32_t s_tmem, uint32_t q_tmem, uint32_t k_smem) {
  constexpr uint32_t idesc = idesc_bf16_f32(kBM, kBN, 0);
#pragma unroll
  for (int kk = 0; kk < kD / 16; ++kk) {
    const uint64_t b = smem_desc_sw128(k_smem + (kk / 4) * kBoxBytes + (kk % 4) * 32, 16, 1024);
    mma_bf16_ts(s_tmem, q_tmem + kk * 8, b, idesc, kk > 0 ? 1u : 0u);
  }
}

// O[128 x 256] (+)= P (TMEM, 128 x 64) . V_j (64 key rows, MN-major: d spans 4 boxes).
__device__ __forceinline__ void issue_pv(uint32_t o_tmem, uint32_t p_tmem, uint32_t v_smem,
                                         bool accumulate) {
  constexpr uint32_t idesc = idesc_bf16_f32(kBM, kD, 1);
#pragma unroll
  for (int kk = 0; kk < kBN / 16; ++kk) {
    const uint64_t b = smem_desc_sw128(v_smem + kk * 16 * 128, kBoxBytes, 1024);
    mma_bf16_ts(o_tmem, p_tmem + kk * 8, b, idesc, (accumulate || kk > 0) ? 1u : 0u);
  }
}

template <bool VL>
__global__ void __launch_bounds__(kThreads, 1)
    attn_fwd_d256_kernel(const __grid_constant__ CUtensorMap tm_k,
                         const __grid_constant__ CUtensorMap tm_v, const void* __restrict__ q,
                         const FwdParams p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_base = smem_addr(smem_raw);
  const uint32_t base = (raw_base + 1023u) & ~1023u;
  uint8_t* const base_ptr = smem_raw + (base - raw_base);
  const uint32_t sBar = base + kOffBar;
  auto bar = [&](int slot) -> uint32_t { return sBar + 8u * slot; };
  uint32_t* const tmem_slot = reinterpret_cast<uint32_t*>(base_ptr + kOffBar + Bars::kTmemSlotByte);
  volatile int* const abort_flag = reinterpret_cast<volatile int*>(base_ptr + kOffBar + Bars::kAbortByte);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // ---- work unit: 128 query rows of one (batch entry or sequence, query head)
  // dense causal: row blocks heaviest first across groups of heads (see grouped_heavy_first)
  int ux, hq, b;
  grouped_heavy_first(VL ? 0 : p.lpt_group, ux, hq, b);
  int Lq = p.Nq, Lk = p.Nkv, q_start = 0, k_start = 0;
  if (VL) {
    // grid (head, item % rows, item / rows): consecutive CTAs are the heads of
    // one unit, and a sequence's units come heaviest first
    hq = blockIdx.x;
    const int item = (int)(blockIdx.y + (long long)blockIdx.z * gridDim.y);
    const int sq = packed_unit(p.cu_q, p.B, p.Nq, kBM, item, ux);
    q_start = min(max(p.cu_q[sq], 0), p.Nq);
    Lq = min(max(p.cu_q[sq + 1], q_start), p.Nq) - q_start;
    k_start = min(max(p.cu_k[sq], 0), p.Nkv);
    Lk = min(max(p.cu_k[sq + 1], k_start), p.Nkv) - k_start;
    b = 0;
  }
  const int nrb = (Lq + kBM - 1) / kBM;
  if (ux < 0 || ux >= nrb) return;  // no unit for this item (the whole CTA leaves)
  const int row_block = p.causal ? (nrb - 1 - ux) : ux;
  const int hk = hq / (p.Hq / p.Hkv);
  const int q0 = row_block * kBM;
  const int bh_q = b * p.Hq + hq;
  const int bh_kv = b * p.Hkv + hk;
  const int diag = p.causal ? Lk - Lq : 0;  // key j visible to query i iff j <= i + diag
  int n_tiles = (Lk + kBN - 1) / kBN;
  if (p.causal) {
    const int last_key = min(min(q0 + kBM - 1, Lq - 1) + diag, Lk - 1);
    n_tiles = last_key < 0 ? 1 : last_key / kBN + 1;
  }
  n_tiles = max(n_tiles, 1);  // a row that sees no key ends with l = 0
  const uint64_t budget = p.timeout_ns;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bar(Bars::kFull + s), 1);
      mbar_init(bar(Bars::kEmpty + s), 1);
    }
    mbar_init(bar(Bars::kQFull), 128);
    for (int t = 0; t < 2; ++t) {
      mbar_init(bar(Bars::kSFull + t), 1);
      mbar_init(bar(Bars::kPFull + t), 128);
    }
    mbar_init(bar(Bars::kPVDone), 1);
    mbar_init(bar(Bars::kOFinal), 1);
    mbar_init(bar(Bars::kDrain), 1);
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(smem_addr(tmem_slot), 512);
    tmem_relinquish();
  }
  if (warp == kLoadWarp && lane == 0) {
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == kLoadWarp) {
    // ================================================================ TMA producer
    bool ok = true;
    uint32_t issued = 0;
    for (int j = 0; j < n_tiles && ok; ++j) {
      for (int which = 0; which < 2; ++which) {  // 0 = K_j, 1 = V_j
        const uint32_t stage = issued % kStages;
        const uint32_t phase = (issued / kStages) & 1u;
        ok = warp_all(bounded_wait(bar(Bars::kEmpty + stage), phase ^ 1u, abort_flag, budget));
        if (!ok) break;
        if (lane == 0) {
          const uint32_t fb = bar(Bars::kFull + stage);
          mbar_arrive_expect_tx(fb, kTileBytes);
          for (int bx = 0; bx < kBoxes; ++bx)
            tma_load_3d(base + stage * kTileBytes + bx * kBoxBytes, which ? &tm_v : &tm_k, fb, bx * 64,
                        VL ? hk : j * kBN, VL ? k_start + j * kBN : bh_kv);
        }
        __syncwarp();
        ++issued;
      }
    }
    if (!ok) {
      if (lane == 0) {
        flag_abort(abort_flag, p.status, 0x100);
        volatile int no_abort = 0;
        const uint32_t first = issued > (uint32_t)kStages ? issued - kStages : 0u;
        for (uint32_t i = first; i < issued; ++i)
          bounded_wait(bar(Bars::kFull + i % kStages), (i / kStages) & 1u, &no_abort, budget);
      }
      __syncwarp();
    }
  } else if (warp == kMmaWarp) {
    // ================================================================ MMA issuer
    const uint32_t tQ = tmem + kColQ, tO = tmem + kColO;
    const uint32_t tS[2] = {tmem + kColS0, tmem + kColS1};
    bool ok = warp_all(bounded_wait(bar(Bars::kQFull), 0, abort_flag, budget));
    int j = 0;
    for (; j <= n_tiles && ok; ++j) {
      if (j < n_tiles) {
        const uint32_t ks = (2 * j) % kStages;
        ok = warp_all(bounded_wait(bar(Bars::kFull + ks), ((2 * j) / kStages) & 1u, abort_flag, budget));
        if (!ok) break;
        tc_fence_after();
        if (lane == 0) {
          issue_s(tS[j & 1], tQ, base + ks * kTileBytes);
          tc_commit(bar(Bars::kSFull + (j & 1)));
          tc_commit(bar(Bars::kEmpty + ks));
        }
        __syncwarp();
      }
      if (j >= 1) {
        const int jp = j - 1;
        const uint32_t vs = (2 * jp + 1) % kStages;
        ok = warp_all(bounded_wait(bar(Bars::kPFull + (jp & 1)), (jp >> 1) & 1, abort_flag, budget) &&
                      bounded_wait(bar(Bars::kFull + vs), ((2 * jp + 1) / kStages) & 1u, abort_flag, budget));
        if (!ok) break;
        tc_fence_after();
        if (lane == 0) {
          issue_pv(tO, tS[jp & 1], base + vs * kTileBytes, jp > 0);
          tc_commit(bar(Bars::kEmpty + vs));
          tc_commit(bar(jp + 1 < n_tiles ? Bars::kPVDone : Bars::kOFinal));
        }
        __syncwarp();
      }
    }
    if (!ok) {
      if (lane == 0) {
        flag_abort(abort_flag, p.status, 0x200 | (j << 12));
        tc_commit(bar(Bars::kDrain));
        volatile int no_abort = 0;
        bounded_wait(bar(Bars::kDrain), 0, &no_abort, budget);
      }
      __syncwarp();
    }
  } else {
    // ================================================================ softmax / correction / epilogue
    const int r = threadIdx.x;  // query row within the tile == TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>(warp << 5) << 16;
    const int row = q0 + r;  // within the sequence
    const bool row_valid = row < Lq;
    // element offset of a valid row (row 0 of the unit's sequence otherwise) in Q and O
    const size_t row_off = VL ? ((size_t)(q_start + (row_valid ? row : 0)) * p.Hq + hq) * kD
                              : ((size_t)bh_q * p.Nq + (row_valid ? row : 0)) * kD;
    // Q row -> registers -> TMEM (bf16 pairs: column c holds elements 2c, 2c+1)
    {
      const uint4* src = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(q) + row_off);
#pragma unroll 1
      for (int c = 0; c < kD / 64; ++c) {
        uint32_t w[32];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const uint4 v = row_valid ? src[8 * c + i] : make_uint4(0, 0, 0, 0);
          w[4 * i] = v.x;
          w[4 * i + 1] = v.y;
          w[4 * i + 2] = v.z;
          w[4 * i + 3] = v.w;
        }
        tmem_st32(tmem + kColQ + lane_off + 32 * c, w);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar(Bars::kQFull));
    }
    const float sl2 = p.scale_log2;
    float m_run = -INFINITY;
    float l_run = 0.0f;
    bool ok = true;
    int j = 0;
    for (; j < n_tiles; ++j) {
      const int t = j & 1;
      ok = warp_all(bounded_wait(bar(Bars::kSFull + t), (j >> 1) & 1, abort_flag, budget));
      if (!ok) break;
      tc_fence_after();
      const uint32_t tS = tmem + (t ? kColS1 : kColS0) + lane_off;
      uint32_t sr[kBN];
      tmem_ld32(tS, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
      tmem_ld32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
      tmem_wait_ld();
      const int kv0 = j * kBN;
      int lim = Lk - kv0;
      if (p.causal) lim = min(lim, row + diag - kv0 + 1);
      if (lim < kBN) {
#pragma unroll
        for (int c = 0; c < kBN; ++c)
          if (c >= lim) sr[c] = __float_as_uint(-INFINITY);
      }
      float mx0 = __uint_as_float(sr[0]), mx1 = __uint_as_float(sr[1]);
#pragma unroll
      for (int c = 2; c < kBN; c += 2) {
        mx0 = fmaxf(mx0, __uint_as_float(sr[c]));
        mx1 = fmaxf(mx1, __uint_as_float(sr[c + 1]));
      }
      const float m_tile = fmaxf(mx0, mx1) * sl2;
      float alpha = 1.0f;
      if (m_tile > m_run + kRescaleThreshold) {
        alpha = ex2_approx(m_run - m_tile);  // 0 on the first visible tile
        m_run = m_tile;
      }
      const float mb = (m_run == -INFINITY) ? 0.0f : m_run;
      float sum0 = 0.f, sum1 = 0.f;
#pragma unroll
      for (int c = 0; c < kBN; c += 2) {
        const float p0 = ex2_approx(fmaf(__uint_as_float(sr[c]), sl2, -mb));
        const float p1 = ex2_approx(fmaf(__uint_as_float(sr[c + 1]), sl2, -mb));
        sum0 += p0;
        sum1 += p1;
        sr[c >> 1] = pack_bf16x2(p0, p1);
      }
      // correction: O *= alpha on rows whose reference maximum moved; O holds
      // PV(0..j-1), so wait for PV(j-1) first
      const bool rescale = (j > 0) && (alpha != 1.0f);
      if (__any_sync(0xffffffffu, rescale)) {
        // PV(j-1) (j - 1 < n_tiles - 1) is phase j-1 of kPVDone; PV(j-2) is
        // complete already (the commit of S(j) covered it), so the parity
        // cannot alias an older phase
        ok = warp_all(bounded_wait(bar(Bars::kPVDone), (j - 1) & 1, abort_flag, budget));
        if (!ok) break;
        tc_fence_after();
#pragma unroll 1
        for (int c = 0; c < kD / 32; ++c) {
          uint32_t o[32];
          tmem_ld32(tmem + kColO + lane_off + 32 * c, o);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
          tmem_st32(tmem + kColO + lane_off + 32 * c, o);
        }
      }
      l_run = l_run * alpha + (sum0 + sum1);
      tmem_st32(tS, *reinterpret_cast<const uint32_t(*)[32]>(&sr[0]));  // P over S columns 0..31
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar(Bars::kPFull + t));
    }
    if (ok) ok = warp_all(bounded_wait(bar(Bars::kOFinal), 0, abort_flag, budget));
    if (ok) {
      // ---- epilogue: O / l -> bf16, row stores; LSE
      tc_fence_after();
      const float inv_l = l_run > 0.0f ? 1.0f / l_run : 0.0f;
      uint4* const orow = reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.o) + row_off);
#pragma unroll 1
      for (int c = 0; c < kD / 32; ++c) {
        uint32_t o[32];
        tmem_ld32(tmem + kColO + lane_off + 32 * c, o);
        tmem_wait_ld();
        if (row_valid) {
#pragma unroll
          for (int g = 0; g < 4; ++g) {
            uint4 v;
            v.x = pack_bf16x2(__uint_as_float(o[8 * g + 0]) * inv_l, __uint_as_float(o[8 * g + 1]) * inv_l);
            v.y = pack_bf16x2(__uint_as_float(o[8 * g + 2]) * inv_l, __uint_as_float(o[8 * g + 3]) * inv_l);
            v.z = pack_bf16x2(__uint_as_float(o[8 * g + 4]) * inv_l, __uint_as_float(o[8 * g + 5]) * inv_l);
            v.w = pack_bf16x2(__uint_as_float(o[8 * g + 6]) * inv_l, __uint_as_float(o[8 * g + 7]) * inv_l);
            orow[c * 4 + g] = v;
          }
        }
      }
      if (row_valid)
        p.lse[VL ? (size_t)hq * p.Nq + q_start + row : (size_t)bh_q * p.Nq + row] =
            (m_run + log2f(l_run)) * 0.69314718055994530942f;
    } else if (lane == 0) {
      flag_abort(abort_flag, p.status, 0x300 | (j << 12));
    }
  }

  // ---- teardown
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace

namespace {
template <bool VL>
cudaError_t launch_d256(const CUtensorMap& tk, const CUtensorMap& tv, const void* q,
                        const FwdParams& p, cudaStream_t stream) {
  cudaError_t e = max_dynamic_smem_once<attn_fwd_d256_kernel<VL>>(kSmemBytes);
  if (e != cudaSuccess) return e;
  dim3 grid((p.Nq + kBM - 1) / kBM, p.Hq, p.B);
  if (VL) {  // x = head, the units of all sequences over y (at most 65535) and z
    const unsigned items = (unsigned)p.num_row_blocks, gy = items < 65535u ? items : 65535u;
    grid = dim3((unsigned)p.Hq, gy, (items + gy - 1) / gy);
  }
  attn_fwd_d256_kernel<VL><<<grid, kThreads, kSmemBytes, stream>>>(tk, tv, q, p);
  return cudaGetLastError();
}
}  // namespace

cudaError_t launch_fwd_d256(const CUtensorMap& tk, const CUtensorMap& tv, const void* q,
                            const FwdParams& p, cudaStream_t stream) {
  return p.cu_q != nullptr ? launch_d256<true>(tk, tv, q, p, stream)
                           : launch_d256<false>(tk, tv, q, p, stream);
}

int fwd_rows_per_cta_d256() { return kBM; }

}  // namespace attn_sm100
