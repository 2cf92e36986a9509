// attn_fwd_sm100.cu — bf16 fused exact attention forward for B200 (sm_100a).
//
// What it computes is the definition on "FlashAttention (TR)"
// (systems-analysis.info), section "Standart Attention Mekanizmasının
// Sorunları": O = softmax(scale * Q K^T [+ causal mask]) V, plus the per-row
// log-sum-exp. How it computes it follows the same page's "Tiling ve Blok
// Tabanlı İşleme" (K/V streamed tile by tile through on-chip memory),
// "Çevrimiçi Softmax Hesaplama" (running row maximum and running sum of
// exponentials, updated per tile) and "İşlemlerin Tek Bir CUDA Çekirdeğinde
// Birleştirilmesi" (QK^T, masking, softmax and the product with V in one
// kernel; only O and LSE reach HBM). The asynchronous producer/consumer idea
// of "Makale Bülteni — FlashAttention-3" ("İddia ve Gerçeklik") is kept, but
// re-derived for Blackwell: TMA loads into a shared-memory ring, tcgen05 MMAs
// accumulating S and O in tensor memory (TMEM), P written back into TMEM as
// the A operand of the second MMA.
//
// CTA = 2 query tiles of 128 rows (same batch and head) sharing every K/V
// tile. Roles (320 threads):
//   warps 0-3   softmax + correction + epilogue of query tile 0 (thread = row)
//   warps 4-7   the same for query tile 1
//   warp  8     MMA issuer (one lane issues tcgen05.mma / commit)
//   warp  9     TMA producer (one lane issues cp.async.bulk.tensor)
// TMEM (512 columns): S0 [0,128) S1 [128,256) O0 [256,256+d) O1 [256+d, 256+2d);
// P_t (bf16, 64 columns) aliases the first half of S_t.
//
// MMA order per KV tile j:  PV0(j-1), S0(j), PV1(j-1), S1(j). Each S_t(j) is
// issued after PV_t(j-1), which read P_t from the same TMEM columns; tcgen05
// MMAs from one thread execute in issue order, and the commit that signals
// S_t(j) also covers PV_t(j-1), so the softmax role may rescale O_t as soon as
// it sees S_t(j).
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "attn_internal.h"
#include "sm100_ptx.cuh"

namespace attn_sm100 {

constexpr int kBM = 128;  // query rows per tile
constexpr int kBN = 128;  // keys per K/V tile
constexpr int kThreads = 320;
constexpr int kMmaWarp = 8;
constexpr int kLoadWarp = 9;
// TMA boxes: 128 rows x kBoxCols bf16. d = 64 / 128 use 64-column boxes with
// the 128-byte swizzle; d = 96 (192-byte rows) uses three 32-column boxes with
// the 64-byte swizzle. The tcgen05 descriptors describe the same layouts.
constexpr float kRescaleThreshold = 8.0f;  // log2 units: rescale O only when the max grows by > 2^8

template <int D>
struct FwdCfg {
  static constexpr int kTileBytes = kBM * D * 2;
  static constexpr int kBoxCols = (D == 96) ? 32 : 64;
  static constexpr int kRowBytes = kBoxCols * 2;           // swizzle width (64 or 128 B)
  static constexpr int kBoxBytes = kBM * kRowBytes;
  static constexpr int kBoxes = D / kBoxCols;
  static constexpr int kAtomBytes = 8 * kRowBytes;         // 8-row swizzle atom
  static constexpr int kStages = (D == 128) ? 4 : (D == 96 ? 6 : 8);
  static constexpr bool kRowStores = (D == 96);            // O stored row by row (no TMA box)
  static constexpr int kOffQ = 0;
  static constexpr int kOffRing = 2 * kTileBytes;
  static_assert(kTileBytes % 1024 == 0, "tiles must keep the 1024-byte swizzle alignment");
  static constexpr int kOffBar = kOffRing + kStages * kTileBytes;
  static constexpr int kBarBytes = 512;
  static constexpr int kSmemBytes = kOffBar + kBarBytes + 1024;  // + base alignment slack
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kColS0 = 0, kColS1 = 128;
  static constexpr uint32_t kColO0 = 256, kColO1 = 256 + D;
};

// Barrier slots (8 bytes each) inside the barrier block.
struct BarLayout {
  static constexpr int kFull = 0;        // [kMaxStages]
  static constexpr int kEmpty = 8;       // [kMaxStages]
  static constexpr int kQFull = 16;
  static constexpr int kSFull = 17;      // [2]
  static constexpr int kPFull = 19;      // [2]
  static constexpr int kOFinal = 21;
  static constexpr int kEpi = 22;        // [2]
  static constexpr int kDrain = 24;
  static constexpr int kCount = 25;
  static constexpr int kTmemSlotByte = 8 * 32;   // uint32 TMEM base address
  static constexpr int kAbortByte = 8 * 32 + 4;  // int abort flag
};

// Record a failed wait once: status[0] = code, status[1] = where (role, tile).
__device__ __forceinline__ void flag_abort(volatile int* abort_flag, int* status, int where) {
  *abort_flag = 1;
  if (atomicCAS(status, 0, ATTN_ERR_TIMEOUT) == 0) status[1] = where;
}

__device__ __forceinline__ bool warp_all(bool v) { return __all_sync(0xffffffffu, v) != 0; }

template <int D>
__device__ __forceinline__ void issue_qk(uint32_t d_tmem, uint32_t q_smem, uint32_t k_smem) {
  constexpr uint32_t idesc = idesc_bf16_f32(kBM, kBN, 0);
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    // 16 columns (32 bytes) per MMA step: box kk / steps-per-box, then 32 B in
    constexpr int kSteps = FwdCfg<D>::kBoxCols / 16;
    const uint32_t off = (kk / kSteps) * FwdCfg<D>::kBoxBytes + (kk % kSteps) * 32;
    const uint64_t a = smem_desc_sw(q_smem + off, 16, FwdCfg<D>::kAtomBytes, FwdCfg<D>::kRowBytes);
    const uint64_t b = smem_desc_sw(k_smem + off, 16, FwdCfg<D>::kAtomBytes, FwdCfg<D>::kRowBytes);
    mma_bf16_ss(d_tmem, a, b, idesc, kk > 0 ? 1u : 0u);
  }
}

template <int D>
__device__ __forceinline__ void issue_pv(uint32_t o_tmem, uint32_t p_tmem, uint32_t v_smem,
                                         bool accumulate) {
  constexpr uint32_t idesc = idesc_bf16_f32(kBM, D, 1);
#pragma unroll
  for (int kk = 0; kk < kBN / 16; ++kk) {
    // V is the MN-major B operand: 16 keys = 16 rows per step; d spans boxes (LBO)
    const uint64_t b = smem_desc_sw(v_smem + kk * 16 * FwdCfg<D>::kRowBytes, FwdCfg<D>::kBoxBytes,
                                    FwdCfg<D>::kAtomBytes, FwdCfg<D>::kRowBytes);
    mma_bf16_ts(o_tmem, p_tmem + kk * 8, b, idesc, (accumulate || kk > 0) ? 1u : 0u);
  }
}

// VL = false: dense [B, H, N, d] tensors, one grid z-slice per batch entry.
// VL = true : packed variable-length sequences [total, H, d]; grid x = query
//             head, (y, z) run over the units of all sequences (packed_unit);
//             the query/key rows of a unit's sequence come from cu_seqlens; O
//             and LSE are stored row by row (a TMA box could cross into the
//             next sequence).
// PART = true (dense only): a partial result over key ranges — grid z = batch
//             entry x range, fp32 O rows and LSE per range, the causal mask
//             aligned to the end of the full key sequence (p.kv_tail keys
//             after the tensor). A separate instantiation, so the plain
//             forward carries none of it.
// PAIR = true (dense, Nq <= 128, an even number of query heads per kv head):
//             the two query tiles are the same rows of two query heads that
//             share a kv head (2 * blockIdx.y and 2 * blockIdx.y + 1), so a
//             short query block does not leave the second tile empty.
template <int D, bool VL, bool PART, bool PAIR>
__global__ void __launch_bounds__(kThreads, 1)
    attn_fwd_bf16_kernel(const __grid_constant__ CUtensorMap tm_q,
                         const __grid_constant__ CUtensorMap tm_k,
                         const __grid_constant__ CUtensorMap tm_v,
                         const __grid_constant__ CUtensorMap tm_o, const FwdParams p) {
  using C = FwdCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_base = smem_addr(smem_raw);
  const uint32_t base = (raw_base + 1023u) & ~1023u;
  uint8_t* const base_ptr = smem_raw + (base - raw_base);

  const uint32_t sQ = base + C::kOffQ;
  const uint32_t sRing = base + C::kOffRing;
  const uint32_t sBar = base + C::kOffBar;
  auto bar = [&](int slot) -> uint32_t { return sBar + 8u * slot; };
  uint32_t* const tmem_slot = reinterpret_cast<uint32_t*>(base_ptr + C::kOffBar + BarLayout::kTmemSlotByte);
  volatile int* const abort_flag =
      reinterpret_cast<volatile int*>(base_ptr + C::kOffBar + BarLayout::kAbortByte);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // ---- work unit: 256 query rows of one (sequence, query head)
  // Dense causal launches dispatch the row blocks heaviest first across
  // groups of p.lpt_group (batch, query head) pairs whose K/V stay in L2:
  // (row-block rank ux, head uy, batch uz).
  int ux, uy, uz;
  grouped_heavy_first((!VL && !PART) ? p.lpt_group : 0, ux, uy, uz);
  int Lq = p.Nq, Lk = p.Nkv, q_start = 0, k_start = 0;
  constexpr int kUnitRows = PAIR ? kBM : 2 * kBM;  // query rows of a work unit
  if (VL) {
    // grid (head, item % rows, item / rows): consecutive CTAs are the heads of
    // one unit, and a sequence's units come heaviest first
    uy = blockIdx.x;
    const int item = (int)(blockIdx.y + (long long)blockIdx.z * gridDim.y);
    const int sq = packed_unit(p.cu_q, p.B, p.Nq, kUnitRows, item, ux);
    q_start = min(max(p.cu_q[sq], 0), p.Nq);
    Lq = min(max(p.cu_q[sq + 1], q_start), p.Nq) - q_start;
    k_start = min(max(p.cu_k[sq], 0), p.Nkv);
    Lk = min(max(p.cu_k[sq + 1], k_start), p.Nkv) - k_start;
  } else if (PART && p.num_splits > 1) {
    // key range (blockIdx.z % num_splits) of a partial-result launch
    k_start = ((int)blockIdx.z % p.num_splits) * p.kv_chunk;  // < Nkv: only non-empty ranges are launched
    Lk = min(p.Nkv - k_start, p.kv_chunk);
  }
  constexpr int kTileRowStep = PAIR ? 0 : kBM;    // first row of tile 1 - of tile 0
  const int nrb = (Lq + kUnitRows - 1) / kUnitRows;
  if (ux < 0 || ux >= nrb) return;  // no unit for this item (the whole CTA leaves)
  const int row_block = p.causal ? (nrb - 1 - ux) : ux;
  const int hq = PAIR ? 2 * uy : uy;  // query head of tile 0
  const int b = VL ? 0 : (PART ? uz / p.num_splits : uz);
  const int hk = hq / (p.Hq / p.Hkv);
  const int q0 = row_block * kUnitRows;  // first query row of the unit, within its sequence
  const int bh_q = b * p.Hq + hq;        // (tile 1: bh_q + 1 when PAIR)
  const int bh_kv = b * p.Hkv + hk;
  // causal mask aligned to the bottom right of the full key sequence: key j
  // (of this unit's range) is visible to query i iff j <= i + (Lk + tail - Lq),
  // tail = the keys after the range (0 unless the keys are split)
  const int tail = PART ? p.kv_tail + (p.Nkv - k_start - Lk) : 0;
  const int diag = p.causal ? Lk + tail - Lq : 0;
  // K/V tiles a query tile needs (at least one, so every pipeline runs; a row
  // that sees no key ends with l = 0): all of them, or (causal) up to the key
  // its last row sees. Query tile 0 of a causal CTA thus skips the last tile.
  auto tiles_for = [&](int last_row) -> int {
    if (!p.causal) return max(1, (Lk + kBN - 1) / kBN);
    const int last_key = min(last_row + diag, Lk - 1);
    return last_key < 0 ? 1 : last_key / kBN + 1;
  };
  const int n_tiles = tiles_for(min(q0 + kUnitRows - 1, Lq - 1));
  const int n_tiles0 = PAIR ? n_tiles : tiles_for(min(q0 + kBM - 1, Lq - 1));
  // TMA coordinates (rows, outer) of a query tile / a K/V tile
  const int q_c1 = VL ? hq : 0, kv_c1 = VL ? hk : 0;
  auto q_row = [&](int t) { return VL ? q_start + q0 + t * kBM : q0 + t * kTileRowStep; };
  auto kv_row = [&](int j) { return k_start + j * kBN; };
  const uint64_t budget = p.timeout_ns;

  // ---- setup: barriers (thread 0), TMEM (MMA warp)
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(bar(BarLayout::kFull + s), 1);
      mbar_init(bar(BarLayout::kEmpty + s), 1);
    }
    mbar_init(bar(BarLayout::kQFull), 1);
    for (int t = 0; t < 2; ++t) {
      mbar_init(bar(BarLayout::kSFull + t), 1);
      mbar_init(bar(BarLayout::kPFull + t), 128);
      mbar_init(bar(BarLayout::kEpi + t), 128);
    }
    mbar_init(bar(BarLayout::kOFinal), 1);
    mbar_init(bar(BarLayout::kDrain), 1);
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(smem_addr(tmem_slot), C::kTmemCols);
    tmem_relinquish();
  }
  if (warp == kLoadWarp && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
    tma_prefetch_desc(&tm_o);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == kLoadWarp) {
    // ================================================================ TMA producer
    bool ok = true;
    uint32_t issued = 0;  // ring slots filled so far
    if (lane == 0) {
      mbar_arrive_expect_tx(bar(BarLayout::kQFull), 2 * C::kTileBytes);
      for (int t = 0; t < 2; ++t)
        for (int bx = 0; bx < C::kBoxes; ++bx)
          tma_load_3d(sQ + t * C::kTileBytes + bx * C::kBoxBytes, &tm_q, bar(BarLayout::kQFull),
                      bx * C::kBoxCols, VL ? q_c1 : q_row(t), VL ? q_row(t) : bh_q + (PAIR ? t : 0));
    }
    for (int j = 0; j < n_tiles && ok; ++j) {
      for (int which = 0; which < 2; ++which) {  // 0 = K_j, 1 = V_j
        const uint32_t stage = issued % C::kStages;
        const uint32_t phase = (issued / C::kStages) & 1u;
        ok = warp_all(bounded_wait(bar(BarLayout::kEmpty + stage), phase ^ 1u, abort_flag, budget));
        if (!ok) break;
        if (lane == 0) {
          const uint32_t fb = bar(BarLayout::kFull + stage);
          mbar_arrive_expect_tx(fb, C::kTileBytes);
          const CUtensorMap* tm = which ? &tm_v : &tm_k;
          for (int bx = 0; bx < C::kBoxes; ++bx)
            tma_load_3d(sRing + stage * C::kTileBytes + bx * C::kBoxBytes, tm, fb, bx * C::kBoxCols,
                        VL ? kv_c1 : kv_row(j), VL ? kv_row(j) : bh_kv);
        }
        __syncwarp();
        ++issued;
      }
    }
    if (!ok) {
      if (lane == 0) flag_abort(abort_flag, p.status, 0x100);
      // Let the loads already in flight land before the CTA can exit.
      if (lane == 0) {
        volatile int no_abort = 0;
        bounded_wait(bar(BarLayout::kQFull), 0, &no_abort, budget);
        const uint32_t first = issued > (uint32_t)C::kStages ? issued - C::kStages : 0u;
        for (uint32_t i = first; i < issued; ++i)
          bounded_wait(bar(BarLayout::kFull + i % C::kStages), (i / C::kStages) & 1u, &no_abort,
                       budget);
      }
      __syncwarp();
    }
  } else if (warp == kMmaWarp) {
    // ================================================================ MMA issuer
    const uint32_t tS[2] = {tmem + C::kColS0, tmem + C::kColS1};
    const uint32_t tO[2] = {tmem + C::kColO0, tmem + C::kColO1};
    const uint32_t q_smem[2] = {sQ, sQ + C::kTileBytes};
    bool ok = warp_all(bounded_wait(bar(BarLayout::kQFull), 0, abort_flag, budget));
    uint32_t slot = 0;
    uint32_t v_prev_stage = 0;
    int j = 0;
    for (; j < n_tiles && ok; ++j) {
      const uint32_t k_stage = slot % C::kStages, k_phase = (slot / C::kStages) & 1u;
      ++slot;
      const uint32_t v_stage = slot % C::kStages;
      ++slot;
      const uint32_t k_smem = sRing + k_stage * C::kTileBytes;
      ok = warp_all(bounded_wait(bar(BarLayout::kFull + k_stage), k_phase, abort_flag, budget));
      if (!ok) break;
      if (j > 0 && j - 1 < n_tiles0) {
        const uint32_t vp_slot = slot - 3;  // V_{j-1}
        ok = warp_all(bounded_wait(bar(BarLayout::kPFull + 0), (j - 1) & 1, abort_flag, budget) &&
                      bounded_wait(bar(BarLayout::kFull + v_prev_stage),
                                   (vp_slot / C::kStages) & 1u, abort_flag, budget));
        if (!ok) break;
        tc_fence_after();
        if (lane == 0)
          issue_pv<D>(tO[0], tS[0], sRing + v_prev_stage * C::kTileBytes, j - 1 > 0);
      }
      tc_fence_after();
      if (lane == 0 && j < n_tiles0) {
        issue_qk<D>(tS[0], q_smem[0], k_smem);
        tc_commit(bar(BarLayout::kSFull + 0));
      }
      __syncwarp();
      if (j > 0) {
        ok = warp_all(bounded_wait(bar(BarLayout::kPFull + 1), (j - 1) & 1, abort_flag, budget));
        if (!ok) break;
        tc_fence_after();
        if (lane == 0) {
          issue_pv<D>(tO[1], tS[1], sRing + v_prev_stage * C::kTileBytes, j - 1 > 0);
          tc_commit(bar(BarLayout::kEmpty + v_prev_stage));
        }
      }
      if (lane == 0) {
        issue_qk<D>(tS[1], q_smem[1], k_smem);
        tc_commit(bar(BarLayout::kSFull + 1));
        tc_commit(bar(BarLayout::kEmpty + k_stage));
      }
      __syncwarp();
      v_prev_stage = v_stage;
    }
    if (ok) {
      // tail: PV of the last tile for both query tiles (tile 0 only if it needs it)
      const int jl = n_tiles - 1;
      const uint32_t vp_slot = slot - 1;
      ok = warp_all(bounded_wait(bar(BarLayout::kFull + v_prev_stage), (vp_slot / C::kStages) & 1u,
                                 abort_flag, budget) &&
                    (n_tiles0 < n_tiles ||
                     bounded_wait(bar(BarLayout::kPFull + 0), jl & 1, abort_flag, budget)));
      if (ok) {
        tc_fence_after();
        if (lane == 0 && n_tiles0 == n_tiles)
          issue_pv<D>(tO[0], tS[0], sRing + v_prev_stage * C::kTileBytes, jl > 0);
        __syncwarp();
        ok = warp_all(bounded_wait(bar(BarLayout::kPFull + 1), jl & 1, abort_flag, budget));
        if (ok) {
          tc_fence_after();
          if (lane == 0) {
            issue_pv<D>(tO[1], tS[1], sRing + v_prev_stage * C::kTileBytes, jl > 0);
            tc_commit(bar(BarLayout::kEmpty + v_prev_stage));
            tc_commit(bar(BarLayout::kOFinal));
          }
          __syncwarp();
        }
      }
    }
    if (!ok) {
      if (lane == 0) {
        flag_abort(abort_flag, p.status, 0x200 | (j << 12));
        // Wait until every MMA already issued has finished before TMEM is freed.
        tc_commit(bar(BarLayout::kDrain));
        volatile int no_abort = 0;
        bounded_wait(bar(BarLayout::kDrain), 0, &no_abort, budget);
      }
      __syncwarp();
    }
  } else {
    // ================================================================ softmax / correction / epilogue
    const int t = warp >> 2;          // query tile 0 or 1
    const int wq = warp & 3;          // TMEM lane quadrant this warp may access
    const int r = (wq << 5) | lane;   // row within the tile == TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>(wq << 5) << 16;
    const uint32_t tS = tmem + (t ? C::kColS1 : C::kColS0) + lane_off;
    const uint32_t tO = tmem + (t ? C::kColO1 : C::kColO0) + lane_off;
    const int row = q0 + t * kTileRowStep + r;
    const int bh_qt = bh_q + (PAIR ? t : 0);  // this tile's (batch, query head)
    const float sl2 = p.scale_log2;

    float m_run = -INFINITY;  // reference maximum of scale*log2(e)*S over the row, so far
    float l_run = 0.0f;       // sum of 2^(scale*log2(e)*S - m_run)
    bool ok = true;
    int j = 0;
    const int my_tiles = t ? n_tiles : n_tiles0;
    for (; j < my_tiles; ++j) {
      ok = warp_all(bounded_wait(bar(BarLayout::kSFull + t), j & 1, abort_flag, budget));
      if (!ok) break;
      tc_fence_after();
      uint32_t sr[128];
#pragma unroll
      for (int c = 0; c < 4; ++c)
        tmem_ld32(tS + 32 * c, *reinterpret_cast<uint32_t(*)[32]>(&sr[32 * c]));
      tmem_wait_ld();

      // mask: keys >= Nkv, and (causal) keys after this row
      const int kv0 = j * kBN;
      int lim = Lk - kv0;
      if (p.causal) lim = min(lim, row + diag - kv0 + 1);
      if (lim < kBN) {
#pragma unroll
        for (int c = 0; c < kBN; ++c)
          if (c >= lim) sr[c] = __float_as_uint(-INFINITY);
      }
      float mx0 = __uint_as_float(sr[0]), mx1 = __uint_as_float(sr[1]);
      float mx2 = __uint_as_float(sr[2]), mx3 = __uint_as_float(sr[3]);
#pragma unroll
      for (int c = 4; c < kBN; c += 4) {
        mx0 = fmaxf(mx0, __uint_as_float(sr[c]));
        mx1 = fmaxf(mx1, __uint_as_float(sr[c + 1]));
        mx2 = fmaxf(mx2, __uint_as_float(sr[c + 2]));
        mx3 = fmaxf(mx3, __uint_as_float(sr[c + 3]));
      }
      const float m_tile = fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3)) * sl2;
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
        sr[c >> 1] = pack_bf16x2(p0, p1);  // P packed in place (index c/2 <= c already read)
      }
      tmem_st32(tS, *reinterpret_cast<const uint32_t(*)[32]>(&sr[0]));
      tmem_st32(tS + 32, *reinterpret_cast<const uint32_t(*)[32]>(&sr[32]));

      // correction: O_t *= alpha on rows whose reference maximum moved
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
      l_run = l_run * alpha + (sum0 + sum1);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar(BarLayout::kPFull + t));
    }

    if (ok) ok = warp_all(bounded_wait(bar(BarLayout::kOFinal), 0, abort_flag, budget));
    if (PART && ok) {
      // ---- epilogue of a partial result: O = O_acc / l in fp32, row by row;
      // a row that saw no key of the range gets O = 0, LSE = -inf
      tc_fence_after();
      const float inv_l = l_run > 0.0f ? 1.0f / l_run : 0.0f;
      const bool valid = row < Lq;
      const int split = p.num_splits > 1 ? (int)blockIdx.z % p.num_splits : 0;
      const size_t prow = ((size_t)split * p.B * p.Hq + bh_qt) * p.Nq + (valid ? row : 0);
      float4* const orow = reinterpret_cast<float4*>(p.o_part + prow * D);
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        uint32_t o[32];
        tmem_ld32(tO + 32 * c, o);
        tmem_wait_ld();
        if (valid) {
#pragma unroll
          for (int q = 0; q < 8; ++q)
            orow[c * 8 + q] = make_float4(__uint_as_float(o[4 * q]) * inv_l, __uint_as_float(o[4 * q + 1]) * inv_l,
                                          __uint_as_float(o[4 * q + 2]) * inv_l, __uint_as_float(o[4 * q + 3]) * inv_l);
        }
      }
      if (valid) p.lse[prow] = (m_run + log2f(l_run)) * 0.69314718055994530942f;
    } else if (ok && (VL || C::kRowStores)) {
      // ---- epilogue (packed sequences, d = 96): O = O_acc / l -> bf16 stored row by row
      tc_fence_after();
      const float inv_l = l_run > 0.0f ? 1.0f / l_run : 0.0f;
      const bool valid = row < Lq;  // q_start + row < total holds by the clamping above
      const size_t orow_idx = VL ? (size_t)(q_start + (valid ? row : 0)) * p.Hq + hq
                                 : (size_t)bh_qt * p.Nq + (valid ? row : 0);
      uint4* const orow = reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.o) + orow_idx * D);
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        uint32_t o[32];
        tmem_ld32(tO + 32 * c, o);
        tmem_wait_ld();
        if (valid) {
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint4 v;
            v.x = pack_bf16x2(__uint_as_float(o[8 * q + 0]) * inv_l, __uint_as_float(o[8 * q + 1]) * inv_l);
            v.y = pack_bf16x2(__uint_as_float(o[8 * q + 2]) * inv_l, __uint_as_float(o[8 * q + 3]) * inv_l);
            v.z = pack_bf16x2(__uint_as_float(o[8 * q + 4]) * inv_l, __uint_as_float(o[8 * q + 5]) * inv_l);
            v.w = pack_bf16x2(__uint_as_float(o[8 * q + 6]) * inv_l, __uint_as_float(o[8 * q + 7]) * inv_l);
            orow[c * 4 + q] = v;
          }
        }
      }
      if (valid)  // LSE: packed sequences [Hq, total_q], dense [B, Hq, Nq]
        p.lse[VL ? (size_t)hq * p.Nq + q_start + row : (size_t)bh_qt * p.Nq + row] =
            (m_run + log2f(l_run)) * 0.69314718055994530942f;
    } else if (ok) {
      // ---- epilogue: O = O_acc / l -> bf16 into the (now free) Q_t buffer, then TMA store
      tc_fence_after();
      const float inv_l = l_run > 0.0f ? 1.0f / l_run : 0.0f;
      uint8_t* const stage_ptr = base_ptr + C::kOffQ + t * C::kTileBytes;
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        uint32_t o[32];
        tmem_ld32(tO + 32 * c, o);
        tmem_wait_ld();
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int col16 = c * 4 + q;   // 16-byte chunk (8 columns) index within the row
          const int bx = col16 >> 3;
          const int ch = col16 & 7;
          uint4 v;
          v.x = pack_bf16x2(__uint_as_float(o[8 * q + 0]) * inv_l, __uint_as_float(o[8 * q + 1]) * inv_l);
          v.y = pack_bf16x2(__uint_as_float(o[8 * q + 2]) * inv_l, __uint_as_float(o[8 * q + 3]) * inv_l);
          v.z = pack_bf16x2(__uint_as_float(o[8 * q + 4]) * inv_l, __uint_as_float(o[8 * q + 5]) * inv_l);
          v.w = pack_bf16x2(__uint_as_float(o[8 * q + 6]) * inv_l, __uint_as_float(o[8 * q + 7]) * inv_l);
          *reinterpret_cast<uint4*>(stage_ptr + bx * C::kBoxBytes + r * 128 + ((ch ^ (r & 7)) << 4)) = v;
        }
      }
      fence_proxy_async_smem();
      mbar_arrive(bar(BarLayout::kEpi + t));
      if (row < Lq) p.lse[(size_t)bh_qt * p.Nq + row] = (m_run + log2f(l_run)) * 0.69314718055994530942f;
      if (r == 0) {
        volatile int no_abort = 0;
        if (bounded_wait(bar(BarLayout::kEpi + t), 0, &no_abort, budget)) {
          for (int bx = 0; bx < C::kBoxes; ++bx)
            tma_store_3d(&tm_o, sQ + t * C::kTileBytes + bx * C::kBoxBytes, bx * 64, q0 + t * kTileRowStep,
                         bh_qt);
          tma_store_commit();
          // the CTA may exit once the store has read shared memory; its global
          // writes complete on their own (visible when the kernel ends)
          tma_store_wait_read();
        } else {
          flag_abort(abort_flag, p.status, 0x400 | t);
        }
      }
    } else if (lane == 0) {
      flag_abort(abort_flag, p.status, 0x300 | (t << 8) | (j << 12));
    }
  }

  // ---- teardown
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

// ------------------------------------------------------------------ host side
template <int D>
static int smem_bytes() { return FwdCfg<D>::kSmemBytes; }

template <int D, bool VL, bool PART = false, bool PAIR = false>
static cudaError_t launch_fwd_d(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                                const CUtensorMap& to, const FwdParams& p, cudaStream_t stream) {
  cudaError_t e = max_dynamic_smem_once<attn_fwd_bf16_kernel<D, VL, PART, PAIR>>(smem_bytes<D>());
  if (e != cudaSuccess) return e;
  // head pairs: Hq / 2 units of 128 rows; packed sequences: x = head, the units
  // of all sequences over y (at most 65535) and z
  dim3 grid(p.num_row_blocks, PAIR ? p.Hq / 2 : p.Hq, p.B * p.num_splits);
  if (VL) {
    const unsigned items = (unsigned)p.num_row_blocks, gy = items < 65535u ? items : 65535u;
    grid = dim3((unsigned)p.Hq, gy, (items + gy - 1) / gy);
  }
  attn_fwd_bf16_kernel<D, VL, PART, PAIR><<<grid, kThreads, smem_bytes<D>(), stream>>>(tq, tk, tv, to, p);
  return cudaGetLastError();
}

cudaError_t launch_fwd_bf16(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                            const CUtensorMap& to, const FwdParams& p, int d, cudaStream_t stream) {
  const bool vl = p.cu_q != nullptr;
  if (!vl && p.pair_heads) {  // dense, Nq <= 128, query-head pairs share a kv head
    if (p.o_part != nullptr) {
      if (d == 128) return launch_fwd_d<128, false, true, true>(tq, tk, tv, to, p, stream);
      if (d == 96) return launch_fwd_d<96, false, true, true>(tq, tk, tv, to, p, stream);
      return launch_fwd_d<64, false, true, true>(tq, tk, tv, to, p, stream);
    }
    if (d == 128) return launch_fwd_d<128, false, false, true>(tq, tk, tv, to, p, stream);
    if (d == 96) return launch_fwd_d<96, false, false, true>(tq, tk, tv, to, p, stream);
    return launch_fwd_d<64, false, false, true>(tq, tk, tv, to, p, stream);
  }
  if (p.o_part != nullptr) {  // partial results (dense tensors)
    if (d == 128) return launch_fwd_d<128, false, true>(tq, tk, tv, to, p, stream);
    if (d == 96) return launch_fwd_d<96, false, true>(tq, tk, tv, to, p, stream);
    return launch_fwd_d<64, false, true>(tq, tk, tv, to, p, stream);
  }
  if (d == 128)
    return vl ? launch_fwd_d<128, true>(tq, tk, tv, to, p, stream)
              : launch_fwd_d<128, false>(tq, tk, tv, to, p, stream);
  if (d == 96)
    return vl ? launch_fwd_d<96, true>(tq, tk, tv, to, p, stream)
              : launch_fwd_d<96, false>(tq, tk, tv, to, p, stream);
  return vl ? launch_fwd_d<64, true>(tq, tk, tv, to, p, stream)
            : launch_fwd_d<64, false>(tq, tk, tv, to, p, stream);
}

int fwd_rows_per_cta() { return 2 * kBM; }
int fwd_rows_per_cta_paired() { return kBM; }

}  // namespace attn_sm100
