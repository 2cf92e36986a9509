// attn_bwd_sm100.cu — bf16 exact attention backward for B200 (sm_100a).
//
// The glossary page "FlashAttention" (aisaas-seo) states that the backward
// pass recomputes a few cheap intermediates instead of storing them: here the
// probabilities P are recomputed tile by tile from Q, K and the per-row
// log-sum-exp the forward wrote, so neither S nor P is ever stored. The
// gradients are the derivative of the definition on "FlashAttention (TR)"
// ("Standart Attention Mekanizmasının Sorunları"), O = softmax(scale*Q K^T) V:
//
//   dV = P^T dO,  dP = dO V^T,  dS = P * (dP - D) with D_i = sum_c dO_ic O_ic,
//   dQ = scale * dS K,  dK = scale * dS^T Q.
//
// The work is tiled as in "Tiling ve Blok Tabanlı İşleme" of the same page,
// with the roles of Q and K/V exchanged: a CTA owns 128 keys of one
// (batch, kv head), keeps K and V in shared memory and dK, dV in tensor memory
// (TMEM), and streams the query blocks of every query head of its group past
// them. Three kernels:
//   attn_bwd_pre   D = rowsum(dO * O), LSE in log2 units, zeroed dQ accumulator
//   attn_bwd_main  everything else; each key block's dQ partial sums are
//                  staged in shared memory and added into an fp32 accumulator
//                  by the TMA unit (cp.reduce.async.bulk .add.f32)
//   attn_bwd_post  dQ = bf16(scale * accumulator)
//
// Main kernel, per iteration (one 128-row query block of one query head):
//   S^T  = K Q^T                (SS MMA, keys in TMEM lanes)
//   dP^T = V dO^T               (SS MMA)
//   P^T  = 2^(S^T * scale*log2e - LSE_2)        softmax warps, bf16 into TMEM
//   dV  += P^T dO               (TS MMA, A = P^T from TMEM)
//   dS^T = P^T * (dP^T - D)                     softmax warps, bf16 into TMEM
//                                               and into a swizzled smem tile
//   dK  += dS^T Q               (TS MMA, A = dS^T from TMEM)
//   dQ_j = dS K                 (SS MMA, A = the dS tile read MN-major)
// Roles (384 threads, three warpgroups):
//   warps 0-3  P and dS (thread = key row = TMEM lane), then the dK epilogue
//   warps 4-7  dQ drain (thread = query row): TMEM -> registers -> the dO
//              buffer of the finished query block, 16 KB at a time -> bulk
//              reduce-add into the accumulator; then the dV epilogue
//   warp  8    MMA issuer
//   warp  9    TMA producer (K, V once; Q, dO, LSE_2, D per query block)
//   warps 10-11 idle (they complete the third warpgroup, which the register
//              re-split needs)
// TMEM (512 columns): S^T [0,128) with P^T (bf16) over [0,64);
//   dP^T [128,256) with dS^T (bf16) over [128,192), then dQ_j (fp32) over
//   [128,128+d); dV [256,256+d); dK [256+d,256+2d).
// MMA issue order per iteration it:
//   dV(it), S(it+1), dK(it), dQ(it), dP(it+1)
// tcgen05 MMAs from one thread execute in issue order, so S(it+1) overwrites
// P^T(it) only after dV(it) read it, and dQ(it) overwrites dS^T(it) only after
// dK(it) read it; dP(it+1) waits until the dQ drain has read dQ(it).
// Each query-block stage has two halves with their own barriers: Q and LSE_2
// are released when dK(it) completes, dO and D only when the dQ drain's bulk
// reductions have read the dO buffer (it doubles as their staging area).
// Measured on B200: vector atomics (red.global.add.v4.f32) from registers for
// the same 64 KB per iteration stalled the tensor core's shared-memory
// operand reads while they drained; the bulk reduce does not.
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "attn_internal.h"
#include "sm100_ptx.cuh"

namespace attn_sm100 {
namespace {

constexpr int kBK = 128;  // keys per CTA (MMA M)
constexpr int kBQ = 128;  // query rows per iteration
constexpr int kThreads = 384;  // three full warpgroups (setmaxnreg is per warpgroup)
constexpr int kMmaWarp = 8;
constexpr int kLoadWarp = 9;
constexpr int kMaxSmem = 232448;  // 227 KB opt-in limit per CTA

// Q, K, V, dO tiles: 128 rows x kBoxCols bf16 per TMA box; d = 64 / 128 use
// 64-column boxes with the 128-byte swizzle, d = 96 three 32-column boxes with
// the 64-byte swizzle (the descriptors below describe the same layouts). The
// dS tile always uses 64-column boxes with the 128-byte swizzle.
template <int D>
struct BwdCfg {
  static constexpr int kTileBytes = 128 * D * 2;  // a 128-row bf16 tile
  static constexpr int kBoxCols = (D == 96) ? 32 : 64;
  static constexpr int kRowBytes = kBoxCols * 2;   // swizzle width (64 or 128 B)
  static constexpr int kBoxBytes = 128 * kRowBytes;
  static constexpr int kBoxes = D / kBoxCols;
  static constexpr int kAtomBytes = 8 * kRowBytes; // 8-row swizzle atom
  static constexpr int kDSBoxBytes = 128 * 128;    // dS^T tile box: 128 keys x 64 queries
  static_assert(kTileBytes % 1024 == 0, "tiles must keep the 1024-byte swizzle alignment");
  static constexpr int kOffK = 0;
  static constexpr int kOffV = kTileBytes;
  static constexpr int kOffQ = 2 * kTileBytes;     // + stage * 2 * kTileBytes
  static constexpr int kOffDO = 3 * kTileBytes;    // + stage * 2 * kTileBytes
  static constexpr int kOffDS = 6 * kTileBytes;    // dS^T tile: 128 keys x 128 queries bf16
  static constexpr int kOffVec = kOffDS + 2 * kDSBoxBytes;  // LSE_2[2][128], D[2][128] (fp32)
  static constexpr int kOffBar = kOffVec + 4 * kBQ * 4;
  static constexpr int kBytes = kOffBar + 128;
  // dynamic shared memory is requested with up to 1 KB of slack for aligning
  // the tiles to the 1024-byte swizzle atom; the kernel checks the base it got
  static constexpr int kSlack = (kBytes + 1024 <= kMaxSmem) ? 1024 : (kMaxSmem - kBytes);
  static constexpr int kSmemBytes = kBytes + kSlack;
  static constexpr int kHalfBytes = kTileBytes + kBQ * 4;  // TMA bytes of Q + LSE_2 (or dO + D)
  static constexpr int kStageBufs = kTileBytes / 16384;      // 16 KB dQ staging buffers in a dO tile
  static constexpr uint32_t kColS = 0, kColDP = 128, kColDV = 256, kColDK = 256 + D;
  static_assert(kBytes <= kMaxSmem, "shared memory layout too large");
};

// Barrier slots (8 bytes each).
struct Bars {
  static constexpr int kKV = 0;
  static constexpr int kFull = 1;    // [2] Q + LSE_2 of stage s landed
  static constexpr int kEmpty = 3;   // [2] Q + LSE_2 of stage s released (dK done)
  static constexpr int kS = 5;       // S^T(it) in TMEM
  static constexpr int kDP = 6;      // dP^T(it) in TMEM
  static constexpr int kP = 7;       // P^T(it) written (128 arrivals)
  static constexpr int kDS = 8;      // dS^T(it) written (128 arrivals)
  static constexpr int kDQ = 9;      // dQ(it) in TMEM
  static constexpr int kDQFree = 10; // dQ(it) read out of TMEM (128 arrivals)
  static constexpr int kAcc = 11;    // dK, dV final
  static constexpr int kDrain = 12;
  static constexpr int kFullDO = 13;  // [2] dO + D of stage s landed
  static constexpr int kEmptyDO = 15; // [2] dO buffer of stage s released (dQ staged out)
  static constexpr int kTmemSlotByte = 8 * 17;
  static constexpr int kAbortByte = 8 * 17 + 4;
};

__device__ __forceinline__ void flag_abort(volatile int* abort_flag, int* status, int where) {
  *abort_flag = 1;
  if (atomicCAS(status, 0, ATTN_ERR_TIMEOUT) == 0) status[1] = where;
}

__device__ __forceinline__ bool warp_all(bool v) { return __all_sync(0xffffffffu, v) != 0; }

// D[128 x 128] = A[128 x d] . B[128 x d]^T, both K-major tiles as TMA writes them.
template <int D>
__device__ __forceinline__ void issue_ss_k(uint32_t d_tmem, uint32_t a_smem, uint32_t b_smem) {
  using C = BwdCfg<D>;
  constexpr uint32_t idesc = idesc_bf16_f32(kBK, kBQ, 0);
  constexpr int kSteps = C::kBoxCols / 16;  // 16-column MMA steps per box
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const uint32_t off = (kk / kSteps) * C::kBoxBytes + (kk % kSteps) * 32;
    mma_bf16_ss(d_tmem, smem_desc_sw(a_smem + off, 16, C::kAtomBytes, C::kRowBytes),
                smem_desc_sw(b_smem + off, 16, C::kAtomBytes, C::kRowBytes), idesc, kk > 0 ? 1u : 0u);
  }
}

// D[128 x d] (+)= A[128 x 128] (TMEM, bf16) . B[128 x d] (MN-major tile: rows = K).
template <int D>
__device__ __forceinline__ void issue_ts_mn(uint32_t d_tmem, uint32_t a_tmem, uint32_t b_smem,
                                            bool accumulate) {
  using C = BwdCfg<D>;
  constexpr uint32_t idesc = idesc_bf16_f32(kBK, D, 1);
#pragma unroll
  for (int kk = 0; kk < kBQ / 16; ++kk) {
    const uint64_t b = smem_desc_sw(b_smem + kk * 16 * C::kRowBytes, C::kBoxBytes, C::kAtomBytes, C::kRowBytes);
    mma_bf16_ts(d_tmem, a_tmem + kk * 8, b, idesc, (accumulate || kk > 0) ? 1u : 0u);
  }
}

// dQ[128 queries x d] = dS[queries x keys] . K[keys x d]; the dS^T tile (rows =
// keys, columns = queries) is read as an MN-major A, the K tile as an MN-major B.
template <int D>
__device__ __forceinline__ void issue_dq(uint32_t d_tmem, uint32_t ds_smem, uint32_t k_smem) {
  using C = BwdCfg<D>;
  constexpr uint32_t idesc = idesc_bf16_f32_major(kBQ, D, 1, 1);
#pragma unroll
  for (int kk = 0; kk < kBK / 16; ++kk) {
    const uint64_t a = smem_desc_sw128(ds_smem + kk * 16 * 128, C::kDSBoxBytes, 1024);
    const uint64_t b = smem_desc_sw(k_smem + kk * 16 * C::kRowBytes, C::kBoxBytes, C::kAtomBytes, C::kRowBytes);
    mma_bf16_ss(d_tmem, a, b, idesc, kk > 0 ? 1u : 0u);
  }
}

// Writes one row of 128 keys: dK or dV (fp32 in TMEM) * mul -> bf16 -> global.
template <int D>
__device__ __forceinline__ void store_row(uint32_t t_row, float mul, uint16_t* dst, bool valid) {
#pragma unroll 1
  for (int c = 0; c < D / 32; ++c) {
    uint32_t v[32];
    tmem_ld32(t_row + 32 * c, v);
    tmem_wait_ld();
    if (valid) {
      uint4* out = reinterpret_cast<uint4*>(dst + 32 * c);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint4 w;
        w.x = pack_bf16x2(__uint_as_float(v[8 * q + 0]) * mul, __uint_as_float(v[8 * q + 1]) * mul);
        w.y = pack_bf16x2(__uint_as_float(v[8 * q + 2]) * mul, __uint_as_float(v[8 * q + 3]) * mul);
        w.z = pack_bf16x2(__uint_as_float(v[8 * q + 4]) * mul, __uint_as_float(v[8 * q + 5]) * mul);
        w.w = pack_bf16x2(__uint_as_float(v[8 * q + 6]) * mul, __uint_as_float(v[8 * q + 7]) * mul);
        out[q] = w;
      }
    }
  }
}

// VL = false: dense [B, H, N, d] tensors, grid z = batch entry.
// VL = true : packed variable-length sequences [total, H, d]; grid x = kv
//             head, (y, z) run over the 128-key units of all sequences
//             (packed_unit: consecutive CTAs are the kv heads of one unit, a
//             sequence's first, heaviest key blocks come first); rows past a
//             sequence's end (the next sequence's) are loaded but contribute
//             nothing: their keys are masked and their queries carry
//             LSE_2 = +inf (P = dS = 0).
template <int D, bool VL>
__global__ void __launch_bounds__(kThreads, 1)
    attn_bwd_main_kernel(const __grid_constant__ CUtensorMap tm_q,
                         const __grid_constant__ CUtensorMap tm_k,
                         const __grid_constant__ CUtensorMap tm_v,
                         const __grid_constant__ CUtensorMap tm_do, const BwdParams p) {
  using C = BwdCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_base = smem_addr(smem_raw);
  const uint32_t base = (raw_base + 1023u) & ~1023u;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // ---- work unit: 128 keys of one (batch, kv head)
  // Causal launches dispatch key blocks heaviest first (the first keys are
  // seen by the most queries) across groups of p.lpt_group (kv head, batch or
  // sequence) pairs whose Q, dO and dQ accumulator stay in L2.
  int kb, hk, b;  // b: batch entry, or sequence (VL)
  grouped_heavy_first(VL ? 0 : p.lpt_group, kb, hk, b);
  if (VL) {
    hk = blockIdx.x;
    const int item = (int)(blockIdx.y + (long long)blockIdx.z * gridDim.y);
    b = packed_unit(p.cu_k, p.num_seqs, p.Nkv, kBK, item, kb);
  }
  const int G = p.Hq / p.Hkv;
  const int k0 = kb * kBK;
  int Lq = p.Nq, Lk = p.Nkv, q_start = 0, k_start = 0;
  if (VL) {
    q_start = min(max(p.cu_q[b], 0), p.Nq);
    // rows past max_seqlen_q (nq_pad) are not computed: they have no
    // accumulator rows
    Lq = min(min(max(p.cu_q[b + 1], q_start), p.Nq) - q_start, p.nq_pad);
    k_start = min(max(p.cu_k[b], 0), p.Nkv);
    Lk = min(max(p.cu_k[b + 1], k_start), p.Nkv) - k_start;
    if (kb < 0 || k0 >= Lk) return;  // no key unit for this item (the whole CTA leaves)
  }
  // row of key k0 + r in dK / dV, and TMA coordinates of K/V and Q/dO tiles
  auto kv_row_off = [&](int r) -> size_t {
    return VL ? ((size_t)(k_start + k0 + r) * p.Hkv + hk) * D
              : ((size_t)(b * p.Hkv + hk) * p.Nkv + k0 + r) * D;
  };
  // causal mask aligned to the bottom right: key j is visible to query i iff
  // j <= i + (Lk - Lq). The first query block with a visible pair:
  const int diag = p.causal ? Lk - Lq : 0;
  const int nqb = (Lq + kBQ - 1) / kBQ;
  int j_begin = 0;
  if (p.causal) j_begin = max(0, k0 - diag) / kBQ;
  const int n_iter = max(0, nqb - j_begin) * G;

  if (n_iter == 0 || base - raw_base > (uint32_t)C::kSlack) {
    // no query sees these keys: dK = dV = 0 (or, never expected, a shared
    // memory base that cannot be aligned within the slack: report it)
    if (n_iter != 0) {
      if (threadIdx.x == 0 && atomicCAS(p.status, 0, ATTN_ERR_CUDA) == 0) p.status[1] = 0x800;
      return;
    }
    for (int r = threadIdx.x; r < kBK; r += kThreads) {
      if (k0 + r >= Lk) break;
      const size_t off = kv_row_off(r);
      uint4* dk = reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.dk) + off);
      uint4* dv = reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.dv) + off);
      for (int i = 0; i < D / 8; ++i) dk[i] = dv[i] = make_uint4(0, 0, 0, 0);
    }
    return;
  }

  uint8_t* const base_ptr = smem_raw + (base - raw_base);
  const uint32_t sK = base + C::kOffK, sV = base + C::kOffV, sDS = base + C::kOffDS;
  const uint32_t sBar = base + C::kOffBar;
  auto bar = [&](int slot) -> uint32_t { return sBar + 8u * slot; };
  auto sQ = [&](int s) -> uint32_t { return base + C::kOffQ + s * 2 * C::kTileBytes; };
  auto sDO = [&](int s) -> uint32_t { return base + C::kOffDO + s * 2 * C::kTileBytes; };
  const float* const vec = reinterpret_cast<const float*>(base_ptr + C::kOffVec);  // [lse2 s0, lse2 s1, D s0, D s1]
  uint32_t* const tmem_slot = reinterpret_cast<uint32_t*>(base_ptr + C::kOffBar + Bars::kTmemSlotByte);
  volatile int* const abort_flag = reinterpret_cast<volatile int*>(base_ptr + C::kOffBar + Bars::kAbortByte);
  const uint64_t budget = p.timeout_ns;
  auto q_block = [&](int it) { return j_begin + it / G; };
  auto q_head = [&](int it) { return hk * G + it % G; };

  if (threadIdx.x == 0) {
    mbar_init(bar(Bars::kKV), 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(Bars::kFull + s), 1);
      mbar_init(bar(Bars::kEmpty + s), 1);
      mbar_init(bar(Bars::kFullDO + s), 1);
      mbar_init(bar(Bars::kEmptyDO + s), 1);
    }
    mbar_init(bar(Bars::kS), 1);
    mbar_init(bar(Bars::kDP), 1);
    mbar_init(bar(Bars::kP), 128);
    mbar_init(bar(Bars::kDS), 128);
    mbar_init(bar(Bars::kDQ), 1);
    mbar_init(bar(Bars::kDQFree), 128);
    mbar_init(bar(Bars::kAcc), 1);
    mbar_init(bar(Bars::kDrain), 1);
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(smem_addr(tmem_slot), 512);
    tmem_relinquish();
  }
  if (warp == kLoadWarp && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
    tma_prefetch_desc(&tm_do);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // Register re-split by warpgroup: 224 + 160 + 120 = 3 x 168, the launch
  // allocation (each sub-partition holds one warp of each warpgroup). Every
  // warp of a warpgroup executes the same setmaxnreg.
  if (warp >= kMmaWarp) {
  regs_decrease<120>();
  if (warp == kLoadWarp) {
    // ================================================================ TMA producer
    bool ok = true;
    int it = 0;
    if (lane == 0) {
      mbar_arrive_expect_tx(bar(Bars::kKV), 2 * C::kTileBytes);
      for (int bx = 0; bx < C::kBoxes; ++bx) {
        const int c1 = VL ? hk : k0, c2 = VL ? k_start + k0 : b * p.Hkv + hk;
        tma_load_3d(sK + bx * C::kBoxBytes, &tm_k, bar(Bars::kKV), bx * C::kBoxCols, c1, c2);
        tma_load_3d(sV + bx * C::kBoxBytes, &tm_v, bar(Bars::kKV), bx * C::kBoxCols, c1, c2);
      }
    }
    int half = 0;  // 0: Q + LSE_2 of query block it; 1: its dO + D
    for (; it < n_iter && ok; half ^= 1, it += half ^ 1) {
      const int s = it & 1;
      ok = warp_all(bounded_wait(bar((half ? Bars::kEmptyDO : Bars::kEmpty) + s),
                                 ((it >> 1) & 1) ^ 1, abort_flag, budget));
      if (!ok) break;
      if (lane == 0) {
        const int q0 = q_block(it) * kBQ;
        const int h = q_head(it);
        const int bh_q = b * p.Hq + h;  // (batch or sequence, head): row of LSE_2 / D
        const uint32_t fb = bar((half ? Bars::kFullDO : Bars::kFull) + s);
        mbar_arrive_expect_tx(fb, C::kHalfBytes);
        for (int bx = 0; bx < C::kBoxes; ++bx)
          tma_load_3d((half ? sDO(s) : sQ(s)) + bx * C::kBoxBytes, half ? &tm_do : &tm_q, fb, bx * C::kBoxCols,
                      VL ? h : q0, VL ? q_start + q0 : bh_q);
        const size_t voff = (size_t)bh_q * p.nq_pad + q0;
        bulk_load(base + C::kOffVec + (2 * half + s) * kBQ * 4, (half ? p.dvec : p.lse2) + voff,
                  kBQ * 4, fb);
      }
      __syncwarp();
    }
    if (!ok) {
      if (lane == 0) {
        flag_abort(abort_flag, p.status, 0x100 | (it << 12));
        // let the loads in flight land before the CTA exits (loads issued:
        // both halves of blocks < it, and the Q half of block it if half = 1)
        volatile int no_abort = 0;
        bounded_wait(bar(Bars::kKV), 0, &no_abort, budget);
        for (int i = max(0, it - 2); i <= it && i < n_iter; ++i) {
          if (i < it || half) bounded_wait(bar(Bars::kFull + (i & 1)), (i >> 1) & 1, &no_abort, budget);
          if (i < it) bounded_wait(bar(Bars::kFullDO + (i & 1)), (i >> 1) & 1, &no_abort, budget);
        }
      }
      __syncwarp();
    }
  } else if (warp == kMmaWarp) {
    // ================================================================ MMA issuer
    const uint32_t tS = tmem + C::kColS, tDP = tmem + C::kColDP;
    const uint32_t tDV = tmem + C::kColDV, tDK = tmem + C::kColDK;
    int it = 0;
    bool ok = warp_all(bounded_wait(bar(Bars::kKV), 0, abort_flag, budget) &&
                       bounded_wait(bar(Bars::kFull + 0), 0, abort_flag, budget) &&
                       bounded_wait(bar(Bars::kFullDO + 0), 0, abort_flag, budget));
    if (ok) {
      tc_fence_after();
      if (lane == 0) {
        issue_ss_k<D>(tS, sK, sQ(0));
        tc_commit(bar(Bars::kS));
        issue_ss_k<D>(tDP, sV, sDO(0));
        tc_commit(bar(Bars::kDP));
      }
      __syncwarp();
    }
    for (; it < n_iter && ok; ++it) {
      const int s = it & 1;
      const bool more = it + 1 < n_iter;
      ok = warp_all(bounded_wait(bar(Bars::kP), it & 1, abort_flag, budget));
      if (!ok) break;
      tc_fence_after();
      if (lane == 0) issue_ts_mn<D>(tDV, tS, sDO(s), it > 0);
      __syncwarp();
      if (more) {
        ok = warp_all(bounded_wait(bar(Bars::kFull + (s ^ 1)), ((it + 1) >> 1) & 1, abort_flag, budget));
        if (!ok) break;
        tc_fence_after();
        if (lane == 0) {
          issue_ss_k<D>(tS, sK, sQ(s ^ 1));
          tc_commit(bar(Bars::kS));
        }
        __syncwarp();
      }
      ok = warp_all(bounded_wait(bar(Bars::kDS), it & 1, abort_flag, budget));
      if (!ok) break;
      tc_fence_after();
      if (lane == 0) {
        issue_ts_mn<D>(tDK, tDP, sQ(s), it > 0);
        tc_commit(bar(Bars::kEmpty + s));
        issue_dq<D>(tDP, sDS, sK);
        tc_commit(bar(Bars::kDQ));
      }
      __syncwarp();
      if (more) {
        ok = warp_all(bounded_wait(bar(Bars::kDQFree), it & 1, abort_flag, budget) &&
                      bounded_wait(bar(Bars::kFullDO + (s ^ 1)), ((it + 1) >> 1) & 1, abort_flag, budget));
        if (!ok) break;
        tc_fence_after();
        if (lane == 0) {
          issue_ss_k<D>(tDP, sV, sDO(s ^ 1));
          tc_commit(bar(Bars::kDP));
        }
        __syncwarp();
      }
    }
    if (ok) {
      if (lane == 0) tc_commit(bar(Bars::kAcc));
      __syncwarp();
    } else {
      if (lane == 0) {
        flag_abort(abort_flag, p.status, 0x200 | (it << 12));
        // every MMA already issued must finish before TMEM is freed
        tc_commit(bar(Bars::kDrain));
        volatile int no_abort = 0;
        bounded_wait(bar(Bars::kDrain), 0, &no_abort, budget);
      }
      __syncwarp();
    }
  }
  } else if (warp < 4) {
    // ================================================================ P and dS (thread = key row)
    regs_increase<224>();
    const int kr = threadIdx.x;  // key row within the block == TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>(warp << 5) << 16;
    const uint32_t tS = tmem + C::kColS + lane_off, tDP = tmem + C::kColDP + lane_off;
    const bool key_valid = k0 + kr < Lk;
    const float sl2 = p.scale_log2;
    uint8_t* const ds_row = base_ptr + C::kOffDS + kr * 128;
    bool ok = true;
    int it = 0;
    for (; it < n_iter; ++it) {
      const int s = it & 1;
      const int q0 = q_block(it) * kBQ;
      // columns c < cmin are masked for this key: key k0+kr sees query q0+c
      // iff k0+kr <= q0+c+diag; keys past Nkv see nothing
      int cmin = 0;
      if (!key_valid) cmin = kBQ;
      else if (p.causal) cmin = min(kBQ, max(0, k0 + kr - q0 - diag));
      const float* lse2 = vec + s * kBQ;
      const float* dvec = vec + (2 + s) * kBQ;

      // LSE_2 and D of this stage were written by the bulk copies counted on
      // the stage's full barrier; S^T(it) is ready when its commit arrives
      ok = warp_all(bounded_wait(bar(Bars::kFull + s), (it >> 1) & 1, abort_flag, budget) &&
                    bounded_wait(bar(Bars::kS), it & 1, abort_flag, budget));
      if (!ok) break;
      tc_fence_after();
      float pr[kBQ];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t sr[32];
        tmem_ld32(tS + 32 * c, sr);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; i += 4) {
          const float4 l4 = *reinterpret_cast<const float4*>(lse2 + 32 * c + i);
          pr[32 * c + i + 0] = ex2_approx(fmaf(__uint_as_float(sr[i + 0]), sl2, -l4.x));
          pr[32 * c + i + 1] = ex2_approx(fmaf(__uint_as_float(sr[i + 1]), sl2, -l4.y));
          pr[32 * c + i + 2] = ex2_approx(fmaf(__uint_as_float(sr[i + 2]), sl2, -l4.z));
          pr[32 * c + i + 3] = ex2_approx(fmaf(__uint_as_float(sr[i + 3]), sl2, -l4.w));
        }
        if (cmin > 32 * c) {
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (32 * c + i < cmin) pr[32 * c + i] = 0.0f;
        }
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) pk[i] = pack_bf16x2(pr[32 * c + 2 * i], pr[32 * c + 2 * i + 1]);
        tmem_st16(tS + 16 * c, pk);  // P^T chunk c over S^T columns already read
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar(Bars::kP));

      ok = warp_all(bounded_wait(bar(Bars::kFullDO + s), (it >> 1) & 1, abort_flag, budget) &&
                    bounded_wait(bar(Bars::kDP), it & 1, abort_flag, budget));
      if (!ok) break;
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t dr[32];
        tmem_ld32(tDP + 32 * c, dr);
        tmem_wait_ld();
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; i += 2) {
          const float4 d4 = *reinterpret_cast<const float4*>(dvec + 32 * c + 2 * i);
          pk[i] = pack_bf16x2(pr[32 * c + 2 * i] * (__uint_as_float(dr[2 * i]) - d4.x),
                              pr[32 * c + 2 * i + 1] * (__uint_as_float(dr[2 * i + 1]) - d4.y));
          pk[i + 1] = pack_bf16x2(pr[32 * c + 2 * i + 2] * (__uint_as_float(dr[2 * i + 2]) - d4.z),
                                  pr[32 * c + 2 * i + 3] * (__uint_as_float(dr[2 * i + 3]) - d4.w));
        }
        tmem_st16(tDP + 16 * c, pk);  // dS^T chunk c over dP^T columns already read
        // the same 32 values into the dS^T tile: box c/2, 16-byte chunks (c%2)*4 + q
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int ch = (c & 1) * 4 + q;
          *reinterpret_cast<uint4*>(ds_row + (c >> 1) * C::kDSBoxBytes + ((ch ^ (kr & 7)) << 4)) =
              make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
        }
      }
      tmem_wait_st();
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(bar(Bars::kDS));
    }
    if (ok) ok = warp_all(bounded_wait(bar(Bars::kAcc), 0, abort_flag, budget));
    if (ok) {
      tc_fence_after();
      uint16_t* dst = static_cast<uint16_t*>(p.dk) + kv_row_off(key_valid ? kr : 0);
      store_row<D>(tmem + C::kColDK + lane_off, p.scale, dst, key_valid);
    } else if (lane == 0) {
      flag_abort(abort_flag, p.status, 0x300 | (it << 12));
    }
  } else {
    // ================================================================ dQ drain (thread = query row)
    regs_decrease<160>();
    const int wq = warp & 3;
    const uint32_t lane_off = static_cast<uint32_t>(wq << 5) << 16;
    const uint32_t tDQ = tmem + C::kColDP + lane_off;
    bool ok = true;
    int it = 0;
    for (; it < n_iter; ++it) {
      // the four drain warps meet at named barriers below, which cannot time
      // out: they decide together whether to go on
      ok = named_bar_and(1, 128, bounded_wait(bar(Bars::kDQ), it & 1, abort_flag, budget));
      if (!ok) break;
      tc_fence_after();
      uint32_t v[D];
#pragma unroll
      for (int c = 0; c < D / 32; ++c) tmem_ld32(tDQ + 32 * c, *reinterpret_cast<uint32_t(*)[32]>(&v[32 * c]));
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(bar(Bars::kDQFree));
      // Stage dQ(it) in the dO buffer of its stage (free: dP(it) and dV(it)
      // completed before dQ(it)) 16 KB = 32 columns at a time, alternating
      // kStageBufs buffers, each chunk added into the accumulator by one bulk
      // reduce. Accumulator layout per 128-row block: [d/4][128 rows][4].
      const int s = it & 1;
      const int q0 = q_block(it) * kBQ;
      const int bh_q = b * p.Hq + q_head(it);
      float* const acc = p.dq_acc + ((size_t)bh_q * (p.nq_pad / kBQ) + q0 / kBQ) * kBQ * D;
      uint8_t* const stage = base_ptr + C::kOffDO + s * 2 * C::kTileBytes;
      const int r = wq * 32 + lane;
      const bool leader = warp == 4 && lane == 0;
#pragma unroll
      for (int q = 0; q < D / 32; ++q) {
        uint8_t* const buf = stage + (q % C::kStageBufs) * 16384;
        if (q >= C::kStageBufs) {
          // the chunk that used this buffer must have been read
          if (leader) bulk_wait_read<C::kStageBufs - 1>();
          named_bar_sync(1, 128);
        }
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const int g = 8 * q + c;
          *reinterpret_cast<float4*>(buf + c * 2048 + r * 16) =
              make_float4(__uint_as_float(v[4 * g]), __uint_as_float(v[4 * g + 1]),
                          __uint_as_float(v[4 * g + 2]), __uint_as_float(v[4 * g + 3]));
        }
        fence_proxy_async_smem();
        named_bar_sync(1, 128);
        if (leader) {
          bulk_reduce_add_f32(acc + q * 4096, smem_addr(buf), 16384);
          tma_store_commit();
        }
      }
      if (leader) {
        bulk_wait_read<0>();
        mbar_arrive(bar(Bars::kEmptyDO + s));
      }
    }
    if (ok) ok = warp_all(bounded_wait(bar(Bars::kAcc), 0, abort_flag, budget));
    if (ok) {
      tc_fence_after();
      const int kr = wq * 32 + lane;
      const bool key_valid = k0 + kr < Lk;
      uint16_t* dst = static_cast<uint16_t*>(p.dv) + kv_row_off(key_valid ? kr : 0);
      store_row<D>(tmem + C::kColDV + lane_off, 1.0f, dst, key_valid);
    } else if (lane == 0) {
      flag_abort(abort_flag, p.status, 0x500 | (it << 12));
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

// Rows of one (batch entry or sequence, head): their count, and the offsets of
// row r in the [.., H, d]-shaped tensors and in LSE ([B, H, N] dense,
// [H, total] packed).
template <int D, bool VL>
struct RowMap {
  int L, start;
  size_t head_base;  // dense: (s * H + h) * N
  int h, H;
  __device__ RowMap(const int* cu, int s, int h_, int H_, int N) : h(h_), H(H_) {
    if (VL) {
      start = min(max(cu[s], 0), N);
      L = min(max(cu[s + 1], start), N) - start;
      head_base = 0;
    } else {
      start = 0;
      L = N;
      head_base = ((size_t)s * H + h_) * N;
    }
  }
  __device__ size_t row(int r) const {  // element offset of row r, column 0
    return VL ? ((size_t)(start + r) * H + h) * D : (head_base + r) * D;
  }
  __device__ size_t lse(int r, int N) const {
    return VL ? (size_t)h * N + start + r : head_base + r;
  }
};

// D_i = sum_c dO_ic O_ic (fp32), LSE_2 = LSE * log2(e) (+inf for padding rows
// and for rows that saw no key, so their P is 0), and the dQ accumulator rows
// zeroed. Grid (nq_pad / 32, Hq, batch entries or sequences); block = 256
// threads = 32 rows x 8 threads per row.
template <int D, bool VL>
__global__ void __launch_bounds__(256) attn_bwd_pre_kernel(const BwdPreParams p) {
  const int g = blockIdx.x;  // 32-row group
  const int h = blockIdx.y, sq = blockIdx.z;
  const RowMap<D, VL> m(p.cu_q, sq, h, p.Hq, p.Nq);
  const size_t bh = (size_t)sq * p.Hq + h;
  // only the sequence's own 128-row blocks are read or reduced into
  if (VL && g * 32 >= (m.L + kBQ - 1) / kBQ * kBQ) return;
  const int r = g * 32 + (threadIdx.x >> 3);
  const int part = threadIdx.x & 7;   // D/8 columns each
  float acc = 0.0f;
  if (r < m.L) {
    // D/8 columns per thread, read 4 at a time (8-byte loads: at d = 96 a
    // thread's 12 columns start at a multiple of 24 bytes)
    const size_t row = m.row(r) + part * (D / 8);
    const uint2* o = reinterpret_cast<const uint2*>(static_cast<const uint16_t*>(p.o) + row);
    const uint2* g2 = reinterpret_cast<const uint2*>(static_cast<const uint16_t*>(p.dout) + row);
#pragma unroll
    for (int i = 0; i < D / 32; ++i) {
      const uint2 a = o[i], c = g2[i];
      const uint32_t aw[2] = {a.x, a.y}, cw[2] = {c.x, c.y};
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        acc = fmaf(__uint_as_float(aw[k] << 16), __uint_as_float(cw[k] << 16), acc);
        acc = fmaf(__uint_as_float(aw[k] & 0xffff0000u), __uint_as_float(cw[k] & 0xffff0000u), acc);
      }
    }
  }
  acc += __shfl_xor_sync(0xffffffffu, acc, 1);
  acc += __shfl_xor_sync(0xffffffffu, acc, 2);
  acc += __shfl_xor_sync(0xffffffffu, acc, 4);
  if (part == 0) {
    const size_t v = bh * p.nq_pad + r;
    p.dvec[v] = acc;
    float l2 = INFINITY;
    if (r < m.L) {
      const float l = p.lse[m.lse(r, p.Nq)];
      if (l != -INFINITY) l2 = l * 1.4426950408889634f;
    }
    p.lse2[v] = l2;
  }
  // zero the accumulator's floats [32 D g, 32 D (g + 1)) of this (sequence,
  // head) (the groups together cover its nq_pad * D floats, whatever the layout)
  float4* acc_rows = reinterpret_cast<float4*>(p.dq_acc + (bh * p.nq_pad + g * 32) * D);
  for (int i = threadIdx.x; i < 8 * D; i += 256) acc_rows[i] = make_float4(0.f, 0.f, 0.f, 0.f);
}

// dQ = bf16(scale * accumulator), through a shared-memory transpose so both
// the accumulator reads and the dQ row writes are contiguous. The accumulator
// holds each 128-row block as [d/4][128 rows][4]; a CTA converts 32 rows.
template <int D, bool VL>
__global__ void __launch_bounds__(256) attn_bwd_post_kernel(const BwdPostParams p) {
  constexpr int kPitch = D + 8;  // bf16 elements per staged row (breaks bank conflicts)
  __shared__ __align__(16) uint16_t tile[32 * kPitch];
  const int g = blockIdx.x;
  const int h = blockIdx.y, sq = blockIdx.z;
  const RowMap<D, VL> m(p.cu_q, sq, h, p.Hq, p.Nq);
  const size_t bh = (size_t)sq * p.Hq + h;
  if (g * 32 >= m.L) return;  // nothing of this sequence in these rows
  const float4* src = reinterpret_cast<const float4*>(p.dq_acc + (bh * p.nq_pad + (g >> 2) * kBQ) * D) +
                      (g & 3) * 32;
  for (int i = threadIdx.x; i < 8 * D; i += 256) {
    const int c4 = i >> 5, row = i & 31;
    const float4 a = src[c4 * kBQ + row];
    uint2 w;
    w.x = pack_bf16x2(a.x * p.scale, a.y * p.scale);
    w.y = pack_bf16x2(a.z * p.scale, a.w * p.scale);
    *reinterpret_cast<uint2*>(&tile[row * kPitch + 4 * c4]) = w;
  }
  __syncthreads();
  for (int i = threadIdx.x; i < 32 * (D / 8); i += 256) {
    const int row = i / (D / 8), c8 = i % (D / 8);
    const int r = g * 32 + row;
    if (r < m.L)
      *reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.dq) + m.row(r) + 8 * c8) =
          *reinterpret_cast<const uint4*>(&tile[row * kPitch + 8 * c8]);
  }
}

template <int D, bool VL>
cudaError_t launch_bwd_d(const BwdLaunch& L, cudaStream_t stream) {
  const dim3 rows_grid(L.pre.nq_pad / 32, L.main.Hq, L.B);  // B: batch entries or sequences
  attn_bwd_pre_kernel<D, VL><<<rows_grid, 256, 0, stream>>>(L.pre);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  e = max_dynamic_smem_once<attn_bwd_main_kernel<D, VL>>(BwdCfg<D>::kSmemBytes);
  if (e != cudaSuccess) return e;
  dim3 grid((L.max_kv + kBK - 1) / kBK, L.main.Hkv, L.B);
  if (VL) {  // x = kv head, the key units of all sequences over y (at most 65535) and z
    const unsigned items = (unsigned)(L.main.Nkv / kBK + L.B), gy = items < 65535u ? items : 65535u;
    grid = dim3((unsigned)L.main.Hkv, gy, (items + gy - 1) / gy);
  }
  attn_bwd_main_kernel<D, VL><<<grid, kThreads, BwdCfg<D>::kSmemBytes, stream>>>(L.tq, L.tk, L.tv, L.tdo,
                                                                              L.main);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  attn_bwd_post_kernel<D, VL><<<rows_grid, 256, 0, stream>>>(L.post);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_bwd(const BwdLaunch& L, int d, cudaStream_t stream) {
  const bool vl = L.main.cu_q != nullptr;
  if (d == 128) return vl ? launch_bwd_d<128, true>(L, stream) : launch_bwd_d<128, false>(L, stream);
  if (d == 96) return vl ? launch_bwd_d<96, true>(L, stream) : launch_bwd_d<96, false>(L, stream);
  return vl ? launch_bwd_d<64, true>(L, stream) : launch_bwd_d<64, false>(L, stream);
}

}  // namespace attn_sm100
