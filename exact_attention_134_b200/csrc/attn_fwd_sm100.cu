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
// Persistent kernel: one CTA per SM walks a static list of work units (256
// query rows of one batch/head = two 128-row tiles sharing every K/V tile),
// heads in groups of 8 so the K/V of the heads in flight stay in L2, and
// within a group the heaviest causal row blocks first. Roles (512 threads):
//   warps 0-3   softmax of query tile 0 (thread = row = TMEM lane), 192 regs
//   warps 4-7   softmax of query tile 1, 192 regs
//   warps 8-11  correction (rescale O when a row maximum moved) and epilogue
//               (O / l -> bf16 -> TMA store, LSE), 64 regs
//   warp 12     MMA issuer (one lane issues tcgen05.mma / commit), 64 regs
//   warp 13     TMA producer (one lane issues cp.async.bulk.tensor), 64 regs
//   warps 14-15 idle
// TMEM (512 columns): S0 [0,128) S1 [128,256) O0 [256,256+d) O1 [256+d,256+2d);
// P_t (bf16, 64 columns) aliases the first half of S_t.
//
// MMA order per KV tile j: PV0(j-1), S0(j), PV1(j-1), S1(j). Each S_t(j) is
// issued after PV_t(j-1), which read P_t from the same TMEM columns; tcgen05
// MMAs from one thread execute in issue order. PV_t(j) waits for the softmax
// (P_t(j) written) and for the correction warpgroup (O_t rescaled for j); the
// first PV_t of a unit also waits until the epilogue has drained O_t of the
// previous unit.
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "attn_internal.h"
#include "sm100_ptx.cuh"

namespace attn_sm100 {

constexpr int kBM = 128;  // query rows per tile
constexpr int kBN = 128;  // keys per K/V tile
constexpr int kThreads = 512;
constexpr int kCorrWarp0 = 8;
constexpr int kMmaWarp = 12;
constexpr int kLoadWarp = 13;
constexpr int kBoxBytes = 128 * 128;  // one TMA box: 128 rows x 64 bf16 (128 B, swizzled)
constexpr float kRescaleThreshold = 8.0f;  // log2 units: rescale O only when the max grows by > 2^8
constexpr int kHeadGroup = 8;

template <int D>
struct FwdCfg {
  static constexpr int kTileBytes = kBM * D * 2;
  static constexpr int kBoxes = D / 64;
  static constexpr int kStages = (D == 128) ? 4 : 8;
  // of every 4 pairs of exponentials, this many are evaluated by the FMA-pipe
  // polynomial instead of MUFU (MUFU is the co-bottleneck with the tensor pipe;
  // a half split also keeps the softmax inside its 192 registers)
  static constexpr int kEmuPairs = 2;
  static constexpr int kOffQ = 0;
  static constexpr int kOffRing = 2 * kTileBytes;
  static constexpr int kOffStage = kOffRing + kStages * kTileBytes;  // one output box
  static constexpr int kOffBar = kOffStage + kBoxBytes;
  static constexpr int kOffStats = kOffBar + 512;  // alpha, m, l: [2][128] fp32 each
  static constexpr int kSmemBytes = kOffStats + 3 * 2 * 128 * 4 + 1024;  // + alignment slack
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kColS0 = 0, kColS1 = 128;
  static constexpr uint32_t kColO0 = 256, kColO1 = 256 + D;
};

// Barrier slots (8 bytes each); [2] = one per query tile.
struct Bar {
  static constexpr int kFull = 0;       // [8] ring slot loaded          (TMA tx)
  static constexpr int kEmpty = 8;      // [8] ring slot consumed        (MMA commit)
  static constexpr int kQFull = 16;     // [2] Q tile loaded             (TMA tx)
  static constexpr int kQFree = 18;     // [2] last S MMA of a unit done (MMA commit)
  static constexpr int kSFull = 20;     // [2] S_t(j) in TMEM            (MMA commit)
  static constexpr int kPFull = 22;     // [2] P_t(j) in TMEM            (128 softmax threads)
  static constexpr int kStats = 24;     // [2] alpha_t(j) in smem        (128 softmax threads)
  static constexpr int kOCorr = 26;     // [2] O_t rescaled for j        (128 correction threads)
  static constexpr int kPvDone = 28;    // [2] PV_t(j) complete          (MMA commit)
  static constexpr int kFin = 30;       // [2] final m, l of a unit      (128 softmax threads)
  static constexpr int kOFree = 32;     // [2] O_t drained by epilogue   (128 correction threads)
  static constexpr int kEpiFull = 34;   // output box staged             (128 correction threads)
  static constexpr int kStageFree = 35; // output box staging reusable   (1 thread)
  static constexpr int kDrain = 36;     // abort path: MMAs drained      (MMA commit)
  static constexpr int kTmemSlotByte = 320;
  static constexpr int kAbortByte = 324;
};

// Record a failed wait once: status[0] = code, status[1] = where (role, tile).
__device__ __forceinline__ void flag_abort(volatile int* abort_flag, int* status, int where) {
  *abort_flag = 1;
  if (atomicCAS(status, 0, ATTN_ERR_TIMEOUT) == 0) status[1] = where;
}

__device__ __forceinline__ bool warp_all(bool v) { return __all_sync(0xffffffffu, v) != 0; }

struct Unit {
  int q0, b, hq, n_tiles;
};

// Work unit u -> (row block, batch, head). Heads go in groups of kHeadGroup;
// inside a group the row blocks run heaviest-first when causal.
__device__ __forceinline__ Unit decode_unit(int u, const FwdParams& p) {
  const int BH = p.B * p.Hq;
  const int nrb = p.num_row_blocks;
  const int full = BH / kHeadGroup, rem = BH - full * kHeadGroup;
  const int span = kHeadGroup * nrb;
  int rb_idx, bh;
  if (u < full * span) {
    const int g = u / span, r = u - g * span;
    rb_idx = r / kHeadGroup;
    bh = g * kHeadGroup + r % kHeadGroup;
  } else {
    const int r = u - full * span;
    rb_idx = r / rem;
    bh = full * kHeadGroup + r % rem;
  }
  Unit x;
  const int rb = p.causal ? nrb - 1 - rb_idx : rb_idx;
  x.q0 = rb * 2 * kBM;
  x.b = bh / p.Hq;
  x.hq = bh - x.b * p.Hq;
  if (p.causal) {
    const int last_row = min(x.q0 + 2 * kBM - 1, p.Nq - 1);
    x.n_tiles = min(last_row, p.Nkv - 1) / kBN + 1;
  } else {
    x.n_tiles = (p.Nkv + kBN - 1) / kBN;
  }
  return x;
}

template <int D>
__device__ __forceinline__ void issue_qk(uint32_t d_tmem, uint32_t q_smem, uint32_t k_smem) {
  constexpr uint32_t idesc = idesc_bf16_f32(kBM, kBN, 0);
#pragma unroll 1
  for (int kk = 0; kk < D / 16; ++kk) {
    const uint32_t off = (kk >> 2) * kBoxBytes + (kk & 3) * 32;
    const uint64_t a = smem_desc_sw128(q_smem + off, 16, 1024);
    const uint64_t b = smem_desc_sw128(k_smem + off, 16, 1024);
    mma_bf16_ss(d_tmem, a, b, idesc, kk > 0 ? 1u : 0u);
  }
}

template <int D>
__device__ __forceinline__ void issue_pv(uint32_t o_tmem, uint32_t p_tmem, uint32_t v_smem,
                                         bool accumulate) {
  constexpr uint32_t idesc = idesc_bf16_f32(kBM, D, 1);
#pragma unroll 1
  for (int kk = 0; kk < kBN / 16; ++kk) {
    const uint64_t b = smem_desc_sw128(v_smem + kk * 16 * 128, kBoxBytes, 1024);
    mma_bf16_ts(o_tmem, p_tmem + kk * 8, b, idesc, (accumulate || kk > 0) ? 1u : 0u);
  }
}

template <int D>
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
  const uint32_t sStage = base + C::kOffStage;
  const uint32_t sBar = base + C::kOffBar;
  auto bar = [&](int slot) -> uint32_t { return sBar + 8u * slot; };
  uint32_t* const tmem_slot = reinterpret_cast<uint32_t*>(base_ptr + C::kOffBar + Bar::kTmemSlotByte);
  volatile int* const abort_flag = reinterpret_cast<volatile int*>(base_ptr + C::kOffBar + Bar::kAbortByte);
  float* const st_alpha = reinterpret_cast<float*>(base_ptr + C::kOffStats);  // [2][128]
  float* const st_m = st_alpha + 256;                                         // [2][128]
  float* const st_l = st_alpha + 512;                                         // [2][128]

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint64_t budget = p.timeout_ns;

  // ---- setup: barriers (thread 0), TMEM (MMA warp)
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(bar(Bar::kFull + s), 1);
      mbar_init(bar(Bar::kEmpty + s), 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(bar(Bar::kQFull + t), 1);
      mbar_init(bar(Bar::kQFree + t), 1);
      mbar_init(bar(Bar::kSFull + t), 1);
      mbar_init(bar(Bar::kPFull + t), 128);
      mbar_init(bar(Bar::kStats + t), 128);
      mbar_init(bar(Bar::kOCorr + t), 128);
      mbar_init(bar(Bar::kPvDone + t), 1);
      mbar_init(bar(Bar::kFin + t), 128);
      mbar_init(bar(Bar::kOFree + t), 128);
    }
    mbar_init(bar(Bar::kEpiFull), 128);
    mbar_init(bar(Bar::kStageFree), 1);
    mbar_init(bar(Bar::kDrain), 1);
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

  // Register split per sub-partition: 192 + 192 + 64 + 64 = 512 registers per
  // lane, i.e. the 16384-register file of each of the four sub-partitions
  // (each holds one warp of every warpgroup). Each role re-splits at its entry.
  const int wg = warp >> 2;
  if (wg == 3) regs_decrease<64>();
  if (warp == kLoadWarp) {
    // ================================================================ TMA producer
    bool ok = true;
    uint32_t issued = 0;  // ring slots filled so far
    int it = 0;
    int q_loaded_it = -1;
    for (int u = blockIdx.x; u < p.num_units && ok; u += gridDim.x, ++it) {
      const Unit w = decode_unit(u, p);
      const int bh_q = w.b * p.Hq + w.hq;
      const int bh_kv = w.b * p.Hkv + w.hq / (p.Hq / p.Hkv);
      for (int t = 0; t < 2 && ok; ++t) {
        ok = warp_all(bounded_wait(bar(Bar::kQFree + t), (it & 1) ^ 1, abort_flag, budget));
        if (!ok) break;
        if (lane == 0) {
          mbar_arrive_expect_tx(bar(Bar::kQFull + t), C::kTileBytes);
          for (int bx = 0; bx < C::kBoxes; ++bx)
            tma_load_3d(sQ + t * C::kTileBytes + bx * kBoxBytes, &tm_q, bar(Bar::kQFull + t),
                        bx * 64, w.q0 + t * kBM, bh_q);
        }
        __syncwarp();
        q_loaded_it = it;
      }
      for (int j = 0; j < w.n_tiles && ok; ++j) {
        for (int which = 0; which < 2; ++which) {  // 0 = K_j, 1 = V_j
          const uint32_t stage = issued % C::kStages;
          const uint32_t phase = (issued / C::kStages) & 1u;
          ok = warp_all(bounded_wait(bar(Bar::kEmpty + stage), phase ^ 1u, abort_flag, budget));
          if (!ok) break;
          if (lane == 0) {
            const uint32_t fb = bar(Bar::kFull + stage);
            mbar_arrive_expect_tx(fb, C::kTileBytes);
            const CUtensorMap* tm = which ? &tm_v : &tm_k;
            for (int bx = 0; bx < C::kBoxes; ++bx)
              tma_load_3d(sRing + stage * C::kTileBytes + bx * kBoxBytes, tm, fb, bx * 64, j * kBN,
                          bh_kv);
          }
          __syncwarp();
          ++issued;
        }
      }
    }
    if (!ok) {
      if (lane == 0) {
        flag_abort(abort_flag, p.status, 0x100 | (it << 12));
        // Let the loads already in flight land before the CTA can exit.
        volatile int no_abort = 0;
        if (q_loaded_it >= 0)
          for (int t = 0; t < 2; ++t)
            bounded_wait(bar(Bar::kQFull + t), q_loaded_it & 1, &no_abort, budget);
        const uint32_t first = issued > (uint32_t)C::kStages ? issued - C::kStages : 0u;
        for (uint32_t i = first; i < issued; ++i)
          bounded_wait(bar(Bar::kFull + i % C::kStages), (i / C::kStages) & 1u, &no_abort, budget);
      }
      __syncwarp();
    }
  } else if (warp == kMmaWarp) {
    // ================================================================ MMA issuer
    const uint32_t tS[2] = {tmem + C::kColS0, tmem + C::kColS1};
    const uint32_t tO[2] = {tmem + C::kColO0, tmem + C::kColO1};
    const uint32_t q_smem[2] = {sQ, sQ + C::kTileBytes};
    bool ok = true;
    uint32_t slot = 0;
    uint32_t base = 0;  // K/V iterations of earlier units (phase index of per-iteration barriers)
    int it = 0;
    int where = 0;
    // PV_t(jj) of the current unit: waits for P_t(jj), O_t corrected, V_jj loaded,
    // and (jj == 0) the previous unit's epilogue having drained O_t.
    auto pv = [&](int t, int jj, uint32_t v_stage, uint32_t v_slot) -> bool {
      const uint32_t ph = (base + jj) & 1u;
      bool r = bounded_wait(bar(Bar::kPFull + t), ph, abort_flag, budget) &&
               bounded_wait(bar(Bar::kOCorr + t), ph, abort_flag, budget) &&
               bounded_wait(bar(Bar::kFull + v_stage), (v_slot / C::kStages) & 1u, abort_flag, budget);
      if (r && jj == 0) r = bounded_wait(bar(Bar::kOFree + t), (it & 1) ^ 1, abort_flag, budget);
      r = warp_all(r);
      if (!r) return false;
      tc_fence_after();
      if (lane == 0) {
        issue_pv<D>(tO[t], tS[t], sRing + v_stage * C::kTileBytes, jj > 0);
        tc_commit(bar(Bar::kPvDone + t));
      }
      __syncwarp();
      return true;
    };
    for (int u = blockIdx.x; u < p.num_units && ok; u += gridDim.x, ++it) {
      const Unit w = decode_unit(u, p);
      const int n = w.n_tiles;
      ok = warp_all(bounded_wait(bar(Bar::kQFull + 0), it & 1, abort_flag, budget) &&
                    bounded_wait(bar(Bar::kQFull + 1), it & 1, abort_flag, budget));
      if (!ok) { where = 1; break; }
      uint32_t v_prev_stage = 0, v_prev_slot = 0;
      for (int j = 0; j < n; ++j) {
        const uint32_t k_slot = slot++;
        const uint32_t v_slot = slot++;
        const uint32_t k_stage = k_slot % C::kStages, v_stage = v_slot % C::kStages;
        const uint32_t k_smem = sRing + k_stage * C::kTileBytes;
        ok = warp_all(bounded_wait(bar(Bar::kFull + k_stage), (k_slot / C::kStages) & 1u, abort_flag, budget));
        if (!ok) { where = 2; break; }
        if (j > 0 && !(ok = pv(0, j - 1, v_prev_stage, v_prev_slot))) { where = 3; break; }
        tc_fence_after();
        if (lane == 0) {
          issue_qk<D>(tS[0], q_smem[0], k_smem);
          tc_commit(bar(Bar::kSFull + 0));
        }
        __syncwarp();
        if (j > 0) {
          if (!(ok = pv(1, j - 1, v_prev_stage, v_prev_slot))) { where = 4; break; }
          if (lane == 0) tc_commit(bar(Bar::kEmpty + v_prev_stage));
        }
        if (lane == 0) {
          issue_qk<D>(tS[1], q_smem[1], k_smem);
          tc_commit(bar(Bar::kSFull + 1));
          tc_commit(bar(Bar::kEmpty + k_stage));
          if (j == n - 1) {  // every S MMA of this unit issued: Q buffers free once they finish
            tc_commit(bar(Bar::kQFree + 0));
            tc_commit(bar(Bar::kQFree + 1));
          }
        }
        __syncwarp();
        v_prev_stage = v_stage;
        v_prev_slot = v_slot;
      }
      if (!ok) break;
      if (!(ok = pv(0, n - 1, v_prev_stage, v_prev_slot))) { where = 5; break; }
      if (!(ok = pv(1, n - 1, v_prev_stage, v_prev_slot))) { where = 6; break; }
      if (lane == 0) tc_commit(bar(Bar::kEmpty + v_prev_stage));
      __syncwarp();
      base += n;
    }
    if (!ok) {
      if (lane == 0) {
        flag_abort(abort_flag, p.status, 0x200 | where | (it << 12));
        // Wait until every MMA already issued has finished before TMEM is freed.
        tc_commit(bar(Bar::kDrain));
        volatile int no_abort = 0;
        bounded_wait(bar(Bar::kDrain), 0, &no_abort, budget);
      }
      __syncwarp();
    }
  } else if (wg < 2) {
    // ================================================================ softmax of query tile t
    regs_increase<192>();
    const int t = wg;
    const int wq = warp & 3;          // TMEM lane quadrant this warp may access
    const int r = (wq << 5) | lane;   // row within the tile == TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>(wq << 5) << 16;
    const uint32_t tS = tmem + (t ? C::kColS1 : C::kColS0) + lane_off;
    const float sl2 = p.scale_log2;
    bool ok = true;
    uint32_t base = 0;
    int it = 0;
    int j = 0;
    for (int u = blockIdx.x; u < p.num_units && ok; u += gridDim.x, ++it) {
      const Unit w = decode_unit(u, p);
      const int row = w.q0 + t * kBM + r;
      float m_run = -INFINITY;  // reference maximum of scale*log2(e)*S over the row, so far
      float l_run = 0.0f;       // sum of 2^(scale*log2(e)*S - m_run)
      for (j = 0; j < w.n_tiles; ++j) {
        ok = warp_all(bounded_wait(bar(Bar::kSFull + t), (base + j) & 1u, abort_flag, budget));
        if (!ok) break;
        tc_fence_after();
        uint32_t sr[128];
#pragma unroll
        for (int c = 0; c < 4; ++c)
          tmem_ld32(tS + 32 * c, *reinterpret_cast<uint32_t(*)[32]>(&sr[32 * c]));
        tmem_wait_ld();

        // mask keys >= Nkv and (causal) keys after the row, only on tiles that need it
        const int kv0 = j * kBN;
        const bool tile_masked =
            (kv0 + kBN > p.Nkv) || (p.causal && kv0 + kBN - 1 > w.q0 + t * kBM);
        if (tile_masked) {
          int lim = p.Nkv - kv0;
          if (p.causal) lim = min(lim, row - kv0 + 1);
#pragma unroll
          for (int c = 0; c < kBN; ++c)
            if (c >= lim) sr[c] = __float_as_uint(-INFINITY);
        }
        float mx0 = -INFINITY, mx1 = -INFINITY, mx2 = -INFINITY, mx3 = -INFINITY;
#pragma unroll
        for (int c = 0; c < kBN; c += 8) {
          mx0 = fmax3(mx0, __uint_as_float(sr[c]), __uint_as_float(sr[c + 1]));
          mx1 = fmax3(mx1, __uint_as_float(sr[c + 2]), __uint_as_float(sr[c + 3]));
          mx2 = fmax3(mx2, __uint_as_float(sr[c + 4]), __uint_as_float(sr[c + 5]));
          mx3 = fmax3(mx3, __uint_as_float(sr[c + 6]), __uint_as_float(sr[c + 7]));
        }
        const float m_tile = fmax3(mx0, mx1, fmaxf(mx2, mx3)) * sl2;
        float alpha = 1.0f;
        if (m_tile > m_run + kRescaleThreshold) {
          alpha = ex2_approx(m_run - m_tile);  // 0 on the first visible tile
          m_run = m_tile;
        }
        st_alpha[t * 128 + r] = alpha;
        mbar_arrive(bar(Bar::kStats + t));  // the correction warpgroup rescales O_t meanwhile

        const float mb = (m_run == -INFINITY) ? 0.0f : m_run;
        const float2 slope = make_float2(sl2, sl2), bias = make_float2(-mb, -mb);
        float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                         make_float2(0.f, 0.f)};
        // p = 2^(s * scale * log2(e) - m); P packed to bf16 in place (index pi <= 2 pi)
        if (tile_masked) {
#pragma unroll
          for (int pi = 0; pi < kBN / 2; ++pi) {
            const float2 x = fma2(make_float2(__uint_as_float(sr[2 * pi]), __uint_as_float(sr[2 * pi + 1])),
                                  slope, bias);
            const float2 e = make_float2(ex2_approx(x.x), ex2_approx(x.y));
            acc[pi & 3] = add2(acc[pi & 3], e);
            sr[pi] = pack_bf16x2(e.x, e.y);
          }
        } else {
          // a fixed share of the exponentials runs on the FMA pipe, the rest on MUFU
#pragma unroll
          for (int pi = 0; pi < kBN / 2; ++pi) {
            const float2 x = fma2(make_float2(__uint_as_float(sr[2 * pi]), __uint_as_float(sr[2 * pi + 1])),
                                  slope, bias);
            const float2 e = ((pi & 3) < C::kEmuPairs) ? exp2_poly2(x)
                                                       : make_float2(ex2_approx(x.x), ex2_approx(x.y));
            acc[pi & 3] = add2(acc[pi & 3], e);
            sr[pi] = pack_bf16x2(e.x, e.y);
          }
        }
        tmem_st32(tS, *reinterpret_cast<const uint32_t(*)[32]>(&sr[0]));
        tmem_st32(tS + 32, *reinterpret_cast<const uint32_t(*)[32]>(&sr[32]));
        const float2 acc01 = add2(acc[0], acc[1]), acc23 = add2(acc[2], acc[3]);
        l_run = l_run * alpha + ((acc01.x + acc01.y) + (acc23.x + acc23.y));
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(bar(Bar::kPFull + t));
      }
      if (!ok) break;
      st_m[t * 128 + r] = m_run;
      st_l[t * 128 + r] = l_run;
      mbar_arrive(bar(Bar::kFin + t));
      base += w.n_tiles;
    }
    if (!ok && lane == 0) flag_abort(abort_flag, p.status, 0x300 | (t << 8) | (it << 12));
  } else if (wg == 2) {
    // ================================================================ correction + epilogue
    regs_decrease<64>();
    const int wq = warp & 3;
    const int r = (wq << 5) | lane;
    const uint32_t lane_off = static_cast<uint32_t>(wq << 5) << 16;
    const uint32_t tO[2] = {tmem + C::kColO0 + lane_off, tmem + C::kColO1 + lane_off};
    uint8_t* const stage_ptr = base_ptr + C::kOffStage;
    bool ok = true;
    uint32_t base = 0;
    uint32_t stage_uses = 0;
    int it = 0;
    int where = 0;
    for (int u = blockIdx.x; u < p.num_units && ok; u += gridDim.x, ++it) {
      const Unit w = decode_unit(u, p);
      const int n = w.n_tiles;
      const int bh_q = w.b * p.Hq + w.hq;
      for (int j = 0; j < n && ok; ++j) {
        for (int t = 0; t < 2; ++t) {
          ok = warp_all(bounded_wait(bar(Bar::kStats + t), (base + j) & 1u, abort_flag, budget));
          if (!ok) { where = 1; break; }
          const float alpha = st_alpha[t * 128 + r];
          if (j > 0 && __any_sync(0xffffffffu, alpha != 1.0f)) {
            // PV_t(j-1) must have finished writing O_t
            ok = warp_all(bounded_wait(bar(Bar::kPvDone + t), (base + j - 1) & 1u, abort_flag, budget));
            if (!ok) { where = 2; break; }
            tc_fence_after();
#pragma unroll 1
            for (int c = 0; c < D / 32; ++c) {
              uint32_t o[32];
              tmem_ld32(tO[t] + 32 * c, o);
              tmem_wait_ld();
#pragma unroll
              for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
              tmem_st32(tO[t] + 32 * c, o);
            }
            tmem_wait_st();
          }
          tc_fence_before();
          mbar_arrive(bar(Bar::kOCorr + t));
        }
      }
      if (!ok) break;
      // ---- epilogue: O = O_acc / l -> bf16 -> one 64-column box at a time -> TMA store
      for (int t = 0; t < 2 && ok; ++t) {
        ok = warp_all(bounded_wait(bar(Bar::kFin + t), it & 1, abort_flag, budget) &&
                      bounded_wait(bar(Bar::kPvDone + t), (base + n - 1) & 1u, abort_flag, budget));
        if (!ok) { where = 3; break; }
        tc_fence_after();
        const float m_fin = st_m[t * 128 + r];
        const float l_fin = st_l[t * 128 + r];
        const float inv_l = l_fin > 0.0f ? 1.0f / l_fin : 0.0f;
        for (int bx = 0; bx < C::kBoxes; ++bx) {
          ok = warp_all(bounded_wait(bar(Bar::kStageFree), (stage_uses & 1u) ^ 1u, abort_flag, budget));
          if (!ok) { where = 4; break; }
#pragma unroll 1
          for (int half = 0; half < 2; ++half) {
            uint32_t o[32];
            tmem_ld32(tO[t] + 64 * bx + 32 * half, o);
            tmem_wait_ld();
            if (bx == C::kBoxes - 1 && half == 1) {  // O_t fully read: the next unit may overwrite it
              tc_fence_before();
              mbar_arrive(bar(Bar::kOFree + t));
            }
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const int ch = half * 4 + q;  // 16-byte chunk of the 128-byte box row
              uint4 v;
              v.x = pack_bf16x2(__uint_as_float(o[8 * q + 0]) * inv_l, __uint_as_float(o[8 * q + 1]) * inv_l);
              v.y = pack_bf16x2(__uint_as_float(o[8 * q + 2]) * inv_l, __uint_as_float(o[8 * q + 3]) * inv_l);
              v.z = pack_bf16x2(__uint_as_float(o[8 * q + 4]) * inv_l, __uint_as_float(o[8 * q + 5]) * inv_l);
              v.w = pack_bf16x2(__uint_as_float(o[8 * q + 6]) * inv_l, __uint_as_float(o[8 * q + 7]) * inv_l);
              *reinterpret_cast<uint4*>(stage_ptr + r * 128 + ((ch ^ (r & 7)) << 4)) = v;
            }
          }
          fence_proxy_async_smem();
          mbar_arrive(bar(Bar::kEpiFull));
          if (r == 0) {
            if (bounded_wait(bar(Bar::kEpiFull), stage_uses & 1u, abort_flag, budget)) {
              tma_store_3d(&tm_o, sStage, bx * 64, w.q0 + t * kBM, bh_q);
              tma_store_commit();
              tma_store_wait_read();
            } else {
              flag_abort(abort_flag, p.status, 0x400 | (t << 8) | (it << 12));
            }
            mbar_arrive(bar(Bar::kStageFree));
          }
          ++stage_uses;
        }
        const int row = w.q0 + t * kBM + r;
        if (ok && row < p.Nq)
          p.lse[(size_t)bh_q * p.Nq + row] = (m_fin + log2f(l_fin)) * 0.69314718055994530942f;
      }
      base += n;
    }
    if (!ok && lane == 0) flag_abort(abort_flag, p.status, 0x500 | where | (it << 12));
    if (r == 0) tma_store_wait_all();
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
static cudaError_t launch_fwd_d(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                                const CUtensorMap& to, const FwdParams& p, cudaStream_t stream) {
  cudaError_t e = cudaFuncSetAttribute(attn_fwd_bf16_kernel<D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       FwdCfg<D>::kSmemBytes);
  if (e != cudaSuccess) return e;
  const int grid = p.num_units < p.num_ctas ? p.num_units : p.num_ctas;
  attn_fwd_bf16_kernel<D><<<grid, kThreads, FwdCfg<D>::kSmemBytes, stream>>>(tq, tk, tv, to, p);
  return cudaGetLastError();
}

cudaError_t launch_fwd_bf16(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                            const CUtensorMap& to, const FwdParams& p, int d, cudaStream_t stream) {
  if (d == 128) return launch_fwd_d<128>(tq, tk, tv, to, p, stream);
  return launch_fwd_d<64>(tq, tk, tv, to, p, stream);
}

int fwd_rows_per_cta() { return 2 * kBM; }

}  // namespace attn_sm100
