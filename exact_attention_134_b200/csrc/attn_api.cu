// attn_api.cu — the C ABI declared in include/attn.h: argument validation,
// tensor-map (TMA descriptor) construction, launch, device status word.
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstring>
#include <mutex>

#include "attn_internal.h"
#include "sm100_ptx.cuh"

namespace {

constexpr int kMaxDevices = 64;

// Device status word: [0] = attn_status_t code of the first failure since the
// last read, [1] = where it happened (role / tile, for diagnostics).
__device__ int g_status[4];

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;
std::mutex g_dev_mutex;
int* g_status_ptr[kMaxDevices] = {nullptr};
std::atomic<long long> g_timeout_ns{1000000000LL};
thread_local cudaError_t g_last_cuda_error = cudaSuccess;

// Map a CUDA runtime result to the ABI status, remembering the runtime's code
// for attn_last_cuda_error().
attn_status_t cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return ATTN_OK;
  g_last_cuda_error = e;
  return ATTN_ERR_CUDA;
}

void load_encode() {
  void* fn = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault,
                                       &q) == cudaSuccess &&
      q == cudaDriverEntryPointSuccess)
    g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
}

// Per-device one-time set-up with that device current: the driver's tensor-map
// encoder and the device address of the status word.
int* device_status_ptr() {
  std::call_once(g_encode_once, load_encode);
  if (!g_encode) return nullptr;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_dev_mutex);
  if (!g_status_ptr[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_status) != cudaSuccess) return nullptr;
    g_status_ptr[dev] = static_cast<int*>(ptr);
  }
  return g_status_ptr[dev];
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// d = 96 is supported by the bf16 kernels only (allow96 = false for the 8-bit
// paths); d = 256 by the bf16 forward only, dense and packed (allow256).
attn_status_t check_args(const void* q, const void* k, const void* v, const void* o,
                         const void* lse, int B, int Hq, int Hkv, int Nq, int Nkv, int d,
                         int causal, float scale, bool allow96 = true, bool allow256 = false) {
  if (!q || !k || !v || !o || !lse) return ATTN_ERR_INVALID_ARG;
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || Nq <= 0 || Nkv <= 0 || d <= 0) return ATTN_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return ATTN_ERR_INVALID_ARG;
  if (!std::isfinite(scale) || !(scale > 0.0f)) return ATTN_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return ATTN_ERR_INVALID_ARG;
  if (d != 64 && d != 128 && !(allow96 && d == 96) && !(allow256 && d == 256))
    return ATTN_ERR_UNSUPPORTED;
  if (B > 65535 || Hq > 65535) return ATTN_ERR_UNSUPPORTED;
  // TMA global strides must stay below 2^40 bytes.
  const unsigned long long head_bytes_q = 2ull * (unsigned long long)Nq * d;
  const unsigned long long head_bytes_kv = 2ull * (unsigned long long)Nkv * d;
  if (head_bytes_q >= (1ull << 40) || head_bytes_kv >= (1ull << 40)) return ATTN_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse))
    return ATTN_ERR_ALIGNMENT;
  return ATTN_OK;
}

// bf16 tensor [BH, N, d] as a 3-D map {d, N, BH}; box = 64 columns x 128 rows,
// 128-byte swizzle (the layout the tcgen05 descriptors expect).
// (d = 96: 32-column boxes with the 64-byte swizzle, three per 96-column row.)
// (d = 256 K/V: 64-row boxes, the d = 256 kernel's 64-key tiles.)
bool encode_map(CUtensorMap* m, const void* ptr, int d, int N, long long BH) {
  cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)N, (cuuint64_t)BH};
  cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)N * (cuuint64_t)d * 2};
  cuuint32_t box[3] = {d == 96 ? 32u : 64u, d == 256 ? 64u : 128u, 1};
  cuuint32_t elem_strides[3] = {1, 1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims,
                        strides, box, elem_strides, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        d == 96 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Packed bf16 tensor [total, H, d] as {d, H, total}; box = 64 columns x 1 head x
// 128 rows (the same shared-memory layout as the dense box; d = 256: 64 rows).
bool encode_map_packed(CUtensorMap* m, const void* ptr, int d, int H, int total) {
  cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)total};
  cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)H * (cuuint64_t)d * 2};
  cuuint32_t box[3] = {d == 96 ? 32u : 64u, 1, d == 256 ? 64u : 128u};
  cuuint32_t elem_strides[3] = {1, 1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims,
                        strides, box, elem_strides, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        d == 96 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// 8-bit tensor [BH, N, d] as {d, N, BH}; box = d bytes x 128 rows, swizzle = d bytes.
bool encode_map_u8(CUtensorMap* m, const void* ptr, int d, int N, long long BH) {
  cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)N, (cuuint64_t)BH};
  cuuint64_t strides[2] = {(cuuint64_t)d, (cuuint64_t)N * (cuuint64_t)d};
  cuuint32_t box[3] = {(cuuint32_t)d, 128, 1};
  cuuint32_t elem_strides[3] = {1, 1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(ptr), dims, strides,
                        box, elem_strides, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        d == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}


// Encoded tensor maps, cached per calling thread: a map depends only on the
// pointer, the shape and the layout kind, so a hit returns exactly what the
// encoder would. Direct-mapped, kMapCacheSlots entries per thread.
constexpr int kMapCacheSlots = 64;
struct MapCacheEntry {
  int kind = -1;  // 0 dense bf16, 1 packed bf16, 2 8-bit
  const void* ptr = nullptr;
  long long a = 0, b = 0, c = 0;
  alignas(64) CUtensorMap map;
};
thread_local MapCacheEntry g_map_cache[kMapCacheSlots];

template <typename Encode>
bool cached_map(CUtensorMap* m, int kind, const void* ptr, long long a, long long b, long long c,
                Encode encode) {
  uint64_t h = reinterpret_cast<uintptr_t>(ptr) ^ (uint64_t)kind * 0x9E3779B97F4A7C15ull;
  h = (h ^ (uint64_t)a * 0xBF58476D1CE4E5B9ull) ^ ((uint64_t)b * 0x94D049BB133111EBull) ^ (uint64_t)c;
  h ^= h >> 31;
  MapCacheEntry& e = g_map_cache[h % kMapCacheSlots];
  if (e.kind == kind && e.ptr == ptr && e.a == a && e.b == b && e.c == c) {
    *m = e.map;
    return true;
  }
  if (!encode(m)) return false;
  e.kind = kind;
  e.ptr = ptr;
  e.a = a;
  e.b = b;
  e.c = c;
  e.map = *m;
  return true;
}

bool make_map(CUtensorMap* m, const void* ptr, int d, int N, long long BH) {
  return cached_map(m, 0, ptr, d, N, BH, [&](CUtensorMap* x) { return encode_map(x, ptr, d, N, BH); });
}
bool make_map_packed(CUtensorMap* m, const void* ptr, int d, int H, int total) {
  return cached_map(m, 1, ptr, d, H, total, [&](CUtensorMap* x) { return encode_map_packed(x, ptr, d, H, total); });
}
bool make_map_u8(CUtensorMap* m, const void* ptr, int d, int N, long long BH) {
  return cached_map(m, 2, ptr, d, N, BH, [&](CUtensorMap* x) { return encode_map_u8(x, ptr, d, N, BH); });
}

// Key-range partial results (dense bf16 kernel only): o_part != null makes the
// kernel write fp32 O rows [num_splits, B, Hq, Nq, d] and lse [num_splits, B,
// Hq, Nq]; num_splits > 1 splits the keys into ranges of kv_chunk keys.
struct PartialArgs {
  float* o_part = nullptr;
  int num_splits = 1;
  int kv_chunk = 0;
  int kv_tail = 0;
};

// A CTA of the bf16 forward holds two 128-row query tiles: 256 rows of one
// query head, or — for Nq <= 128 with an even number of query heads per kv
// head — the same rows of two query heads that share their K/V tiles.
bool pairs_heads(int Hq, int Hkv, int Nq, int d) {
  return d != 256 && Nq <= attn_sm100::fwd_rows_per_cta_paired() && (Hq / Hkv) % 2 == 0;
}
long long fwd_ctas(int B, int Hq, int Hkv, int Nq, int d) {
  if (pairs_heads(Hq, Hkv, Nq, d)) return (long long)B * (Hq / 2);
  const int rows = attn_sm100::fwd_rows_per_cta();
  return (long long)B * Hq * ((Nq + rows - 1) / rows);
}

attn_status_t run_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                      int Hq, int Hkv, int Nq, int Nkv, int d, int causal, float scale,
                      cudaStream_t stream, const PartialArgs& part = PartialArgs()) {
  int* status = device_status_ptr();
  if (!status) return ATTN_ERR_CUDA;
  alignas(64) CUtensorMap tq, tk, tv, to;
  if (d == 256) {
    if (!make_map(&tk, k, d, Nkv, (long long)B * Hkv) || !make_map(&tv, v, d, Nkv, (long long)B * Hkv))
      return ATTN_ERR_CUDA;
  } else if (!make_map(&tq, q, d, Nq, (long long)B * Hq) ||
             !make_map(&tk, k, d, Nkv, (long long)B * Hkv) ||
             !make_map(&tv, v, d, Nkv, (long long)B * Hkv) ||
             // a partial result is stored row by row: the output map is unused
             !make_map(&to, part.o_part ? q : o, d, Nq, (long long)B * Hq)) {
    return ATTN_ERR_CUDA;
  }
  attn_sm100::FwdParams p;
  p.o = o;
  p.lse = lse;
  p.status = status;
  p.cu_q = nullptr;
  p.cu_k = nullptr;
  p.B = B;
  p.Nq = Nq;
  p.Nkv = Nkv;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.causal = causal;
  // short query blocks: pair the query heads of a kv head in one CTA
  p.pair_heads = pairs_heads(Hq, Hkv, Nq, d) ? 1 : 0;
  const int rows = p.pair_heads ? attn_sm100::fwd_rows_per_cta_paired() : attn_sm100::fwd_rows_per_cta();
  p.num_row_blocks = (Nq + rows - 1) / rows;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.timeout_ns = (unsigned long long)g_timeout_ns.load();
  // Causal row blocks differ in cost: dispatch the heaviest of a group of
  // (batch, query head) pairs first, the group's kv heads holding at most
  // 32 MiB of K and V so that they stay in L2 while the group runs.
  if (causal && !p.pair_heads && !part.o_part && Nq > 128) {
    const long long kv_head_bytes = 4LL * Nkv * d;
    const long long kv_heads = std::max(1LL, (32LL << 20) / kv_head_bytes);
    p.lpt_group = (int)std::min((long long)B * Hq, kv_heads * (Hq / Hkv));
  }
  p.o_part = part.o_part;
  p.num_splits = part.num_splits;
  p.kv_chunk = part.kv_chunk;
  p.kv_tail = part.kv_tail;
  if (d == 256) return cuda_status(attn_sm100::launch_fwd_d256(tk, tv, q, p, stream));
  return cuda_status(attn_sm100::launch_fwd_bf16(tq, tk, tv, to, p, d, stream));
}

attn_status_t run_fwd_varlen(const void* q, const void* k, const void* v, void* o, float* lse,
                             const int* cu_q, const int* cu_k, int num_seqs, int max_seqlen_q,
                             int total_q, int total_k, int Hq, int Hkv, int d, int causal,
                             float scale, cudaStream_t stream) {
  int* status = device_status_ptr();
  if (!status) return ATTN_ERR_CUDA;
  alignas(64) CUtensorMap tq, tk, tv;
  // d = 256: the d = 256 kernel reads Q rows directly (no Q map)
  if ((d != 256 && !make_map_packed(&tq, q, d, Hq, total_q)) || !make_map_packed(&tk, k, d, Hkv, total_k) ||
      !make_map_packed(&tv, v, d, Hkv, total_k))
    return ATTN_ERR_CUDA;
  attn_sm100::FwdParams p;
  p.o = o;
  p.lse = lse;
  p.status = status;
  p.cu_q = cu_q;
  p.cu_k = cu_k;
  p.B = num_seqs;
  p.Nq = total_q;
  p.Nkv = total_k;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.causal = causal;
  // grid x: the units of all sequences, at most one item per sequence without one
  // (packed_unit); max_seqlen_q is not needed for it
  const int rows = d == 256 ? attn_sm100::fwd_rows_per_cta_d256() : attn_sm100::fwd_rows_per_cta();
  p.num_row_blocks = total_q / rows + num_seqs;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.timeout_ns = (unsigned long long)g_timeout_ns.load();
  if (d == 256) return cuda_status(attn_sm100::launch_fwd_d256(tk, tv, q, p, stream));
  // the output map is unused by the packed path (rows are stored one by one)
  return cuda_status(attn_sm100::launch_fwd_bf16(tq, tk, tv, tq, p, d, stream));
}

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Failure-detection self-test: one thread waits, with the kernels' own bounded
// wait, on an mbarrier that nothing completes. The wait must give up after its
// budget and record ATTN_ERR_TIMEOUT (where = 0xF00) in the status word; the
// kernel then returns normally, so the context stays usable.
__global__ void selftest_wait_timeout_kernel(int* status, unsigned long long budget_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    attn_sm100::mbar_init(attn_sm100::smem_addr(&bar), 1);
    abort_flag = 0;
    attn_sm100::fence_mbarrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0 &&
      !attn_sm100::bounded_wait(attn_sm100::smem_addr(&bar), 0, &abort_flag, budget_ns)) {
    if (atomicCAS(status, 0, ATTN_ERR_TIMEOUT) == 0) status[1] = 0xF00;
  }
}

// Workspace of the 8-bit path, in this order, each region 256-byte aligned:
// q8, k8, v8 (1 byte per element), sq, sk, sv, kbar, qk (fp32), ksum partials
// (fp64), vmax partials (fp32).
constexpr int kQ8Regions = 10;

void q8_layout(int B, int Hq, int Hkv, int Nq, int Nkv, int d, size_t off[kQ8Regions + 1]) {
  const size_t nqb = (size_t)(Nq + 127) / 128, nkb = (size_t)(Nkv + 127) / 128;
  const size_t sz[kQ8Regions] = {
      (size_t)B * Hq * Nq * d,      (size_t)B * Hkv * Nkv * d,   (size_t)B * Hkv * Nkv * d,
      4ull * B * Hq * nqb,          4ull * B * Hkv * nkb,        4ull * B * Hkv * d,
      4ull * B * Hkv * d,           4ull * B * Hq * (size_t)Nq,  8ull * B * Hkv * nkb * d,
      4ull * B * Hkv * nkb * d};
  size_t o = 0;
  for (int i = 0; i < kQ8Regions; ++i) {
    off[i] = o;
    o = round_up(o + sz[i], 256);
  }
  off[kQ8Regions] = o;
}

attn_status_t run_q8(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                     int Hq, int Hkv, int Nq, int Nkv, int d, int causal, float scale,
                     void* workspace, size_t workspace_bytes, bool prepass_only,
                     cudaStream_t stream, bool fp8_qk = false) {
  if (!workspace || !aligned16(workspace)) return ATTN_ERR_WORKSPACE;
  size_t off[kQ8Regions + 1];
  q8_layout(B, Hq, Hkv, Nq, Nkv, d, off);
  if (workspace_bytes < off[kQ8Regions]) return ATTN_ERR_WORKSPACE;
  int* status = device_status_ptr();
  if (!status) return ATTN_ERR_CUDA;
  char* w = static_cast<char*>(workspace);
  attn_sm100::Q8Launch L;
  std::memset(static_cast<void*>(&L), 0, sizeof(L));
  L.q = q;
  L.k = k;
  L.v = v;
  L.q8 = reinterpret_cast<int8_t*>(w + off[0]);
  L.k8 = reinterpret_cast<int8_t*>(w + off[1]);
  L.v8 = reinterpret_cast<uint8_t*>(w + off[2]);
  L.kbar = reinterpret_cast<float*>(w + off[6]);
  L.ksum_part = reinterpret_cast<double*>(w + off[8]);
  L.vmax_part = reinterpret_cast<float*>(w + off[9]);
  L.B = B;
  L.Hkv = Hkv;
  L.prepass_only = prepass_only;
  L.fp8_qk = fp8_qk;
  attn_sm100::Q8Params& p = L.p;
  p.lse = lse;
  p.status = status;
  p.sq = reinterpret_cast<const float*>(w + off[3]);
  p.sk = reinterpret_cast<const float*>(w + off[4]);
  p.sv = reinterpret_cast<const float*>(w + off[5]);
  p.qk = reinterpret_cast<const float*>(w + off[7]);
  p.Nq = Nq;
  p.Nkv = Nkv;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.causal = causal;
  p.num_row_blocks = (Nq + 255) / 256;
  p.nqb = (Nq + 127) / 128;
  p.nkb = (Nkv + 127) / 128;
  if (causal && Nq > 256) {  // as the bf16 forward, for 8-bit K and V
    const long long kv_heads = std::max(1LL, (32LL << 20) / (2LL * Nkv * d));
    p.lpt_group = (int)std::min((long long)B * Hq, kv_heads * (Hq / Hkv));
  }
  p.scale_log2 = scale * 1.4426950408889634f;
  p.scale = scale;
  p.timeout_ns = (unsigned long long)g_timeout_ns.load();
  if (!prepass_only) {
    if (!make_map_u8(&L.tq, L.q8, d, Nq, (long long)B * Hq) ||
        !make_map_u8(&L.tk, L.k8, d, Nkv, (long long)B * Hkv) ||
        !make_map_u8(&L.tv, L.v8, d, Nkv, (long long)B * Hkv) ||
        !make_map(&L.to, o, d, Nq, (long long)B * Hq))
      return ATTN_ERR_CUDA;
  }
  return cuda_status(attn_sm100::launch_q8(L, d, stream));
}

struct HostLayout {
  size_t q, k, v, o, lse, total;
};

// Streams and events of the host-buffer entry point, created once per device
// (with that device current) and kept for the process: a copy-in stream, a
// copy-out stream and the per-chunk events that order them around the caller's
// stream, on which the kernels run.
constexpr int kHostChunks = 8;
struct HostPipe {
  cudaStream_t in = nullptr, out = nullptr;
  cudaEvent_t start = nullptr, done = nullptr;
  cudaEvent_t loaded[kHostChunks] = {}, computed[kHostChunks] = {};
  bool ready = false;
};
HostPipe g_pipe[kMaxDevices];
std::mutex g_pipe_mutex[kMaxDevices];  // one enqueue sequence at a time per device

HostPipe* host_pipe() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_dev_mutex);
  HostPipe& P = g_pipe[dev];
  if (!P.ready) {
    const unsigned f = cudaEventDisableTiming;
    bool ok = cudaStreamCreateWithFlags(&P.in, cudaStreamNonBlocking) == cudaSuccess &&
              cudaStreamCreateWithFlags(&P.out, cudaStreamNonBlocking) == cudaSuccess &&
              cudaEventCreateWithFlags(&P.start, f) == cudaSuccess &&
              cudaEventCreateWithFlags(&P.done, f) == cudaSuccess;
    for (int i = 0; ok && i < kHostChunks; ++i)
      ok = cudaEventCreateWithFlags(&P.loaded[i], f) == cudaSuccess &&
           cudaEventCreateWithFlags(&P.computed[i], f) == cudaSuccess;
    if (!ok) return nullptr;
    P.ready = true;
  }
  return &P;
}

HostLayout host_layout(int B, int Hq, int Hkv, int Nq, int Nkv, int d) {
  HostLayout L;
  const size_t qo = 2ull * B * Hq * (size_t)Nq * d;
  const size_t kv = 2ull * B * Hkv * (size_t)Nkv * d;
  L.q = 0;
  L.k = round_up(L.q + qo, 256);
  L.v = round_up(L.k + kv, 256);
  L.o = round_up(L.v + kv, 256);
  L.lse = round_up(L.o + qo, 256);
  L.total = round_up(L.lse + 4ull * B * Hq * (size_t)Nq, 256);
  return L;
}

// Backward workspace: fp32 dQ accumulator [B*Hq, nq_pad, d], then LSE*log2(e)
// and D, each [B*Hq, nq_pad] fp32; regions 256-byte aligned.
struct BwdLayout {
  size_t acc, lse2, dvec, total;
};

BwdLayout bwd_layout(int B, int Hq, int Nq, int d) {
  const size_t rows = (size_t)B * Hq * (size_t)((Nq + 127) / 128 * 128);
  BwdLayout L;
  L.acc = 0;
  L.lse2 = round_up(L.acc + 4 * rows * d, 256);
  L.dvec = round_up(L.lse2 + 4 * rows, 256);
  L.total = round_up(L.dvec + 4 * rows, 256);
  return L;
}

// Backward for dense tensors (cu_q == nullptr: B batch entries, Nq / Nkv rows
// each) or packed sequences (B = sequences, Nq / Nkv = total rows, rows of a
// sequence up to max_q / max_k).
attn_status_t run_bwd(const void* q, const void* k, const void* v, const void* o,
                      const float* lse, const void* dout, void* dq, void* dk, void* dv,
                      const int* cu_q, const int* cu_k, int B, int Hq, int Hkv, int Nq, int Nkv,
                      int max_q, int max_k, int d, int causal, float scale, void* workspace,
                      cudaStream_t stream) {
  int* status = device_status_ptr();
  if (!status) return ATTN_ERR_CUDA;
  const bool vl = cu_q != nullptr;
  const BwdLayout W = bwd_layout(B, Hq, max_q, d);
  char* w = static_cast<char*>(workspace);
  attn_sm100::BwdLaunch L;
  std::memset(static_cast<void*>(&L), 0, sizeof(L));
  const bool maps_ok =
      vl ? make_map_packed(&L.tq, q, d, Hq, Nq) && make_map_packed(&L.tk, k, d, Hkv, Nkv) &&
               make_map_packed(&L.tv, v, d, Hkv, Nkv) && make_map_packed(&L.tdo, dout, d, Hq, Nq)
         : make_map(&L.tq, q, d, Nq, (long long)B * Hq) &&
               make_map(&L.tk, k, d, Nkv, (long long)B * Hkv) &&
               make_map(&L.tv, v, d, Nkv, (long long)B * Hkv) &&
               make_map(&L.tdo, dout, d, Nq, (long long)B * Hq);
  if (!maps_ok) return ATTN_ERR_CUDA;
  const int nq_pad = (max_q + 127) / 128 * 128;
  float* acc = reinterpret_cast<float*>(w + W.acc);
  float* lse2 = reinterpret_cast<float*>(w + W.lse2);
  float* dvec = reinterpret_cast<float*>(w + W.dvec);
  L.B = B;
  L.max_kv = max_k;
  L.pre.o = o;
  L.pre.dout = dout;
  L.pre.lse = lse;
  L.pre.dvec = dvec;
  L.pre.lse2 = lse2;
  L.pre.dq_acc = acc;
  L.pre.cu_q = cu_q;
  L.pre.Nq = Nq;
  L.pre.Hq = Hq;
  L.pre.nq_pad = nq_pad;
  attn_sm100::BwdParams& p = L.main;
  p.dk = dk;
  p.dv = dv;
  p.dq_acc = acc;
  p.lse2 = lse2;
  p.dvec = dvec;
  p.status = status;
  p.cu_q = cu_q;
  p.cu_k = cu_k;
  p.Nq = Nq;
  p.Nkv = Nkv;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.causal = causal;
  p.nq_pad = nq_pad;
  p.scale = scale;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.timeout_ns = (unsigned long long)g_timeout_ns.load();
  if (causal && !vl && Nkv > 128) {
    // a group's Q, dO (bf16) and dQ accumulator (fp32) within 32 MiB
    const long long per_kv_head = 8LL * Nq * d * (Hq / Hkv);
    p.lpt_group = (int)std::min((long long)B * Hkv, std::max(1LL, (32LL << 20) / per_kv_head));
  }
  // packed sequences: the grid is (kv head, key units of all sequences), so the
  // kv heads of one unit run together and a sequence's heavy first keys first
  p.num_seqs = vl ? B : 0;
  L.post.dq_acc = acc;
  L.post.dq = dq;
  L.post.cu_q = cu_q;
  L.post.Nq = Nq;
  L.post.Hq = Hq;
  L.post.nq_pad = nq_pad;
  L.post.scale = scale;
  return cuda_status(attn_sm100::launch_bwd(L, d, stream));
}

}  // namespace

namespace attn_sm100 {

attn_status_t cuda_error_status(cudaError_t e) { return cuda_status(e); }

// Internal: the argument checks of attn_fwd / attn_fwd_q8.
attn_status_t validate_fwd_args(const void* q, const void* k, const void* v, const void* o,
                                const void* lse, int B, int Hq, int Hkv, int Nq, int Nkv, int d,
                                int causal, float scale) {
  return check_args(q, k, v, o, lse, B, Hq, Hkv, Nq, Nkv, d, causal, scale, false);
}

// Internal: validate arguments and run the 8-bit forward with a workspace the
// caller already has (used by the entry point whose workspace is a static
// device array).
attn_status_t q8_forward_with_workspace(const void* q, const void* k, const void* v, void* o,
                                        float* lse, int B, int Hq, int Hkv, int Nq, int Nkv, int d,
                                        int causal, float scale, void* workspace,
                                        size_t workspace_bytes, cudaStream_t stream) {
  attn_status_t s = check_args(q, k, v, o, lse, B, Hq, Hkv, Nq, Nkv, d, causal, scale, false);
  if (s != ATTN_OK) return s;
  return run_q8(q, k, v, o, lse, B, Hq, Hkv, Nq, Nkv, d, causal, scale, workspace, workspace_bytes,
                false, stream);
}

}  // namespace attn_sm100

namespace {

// Split of the keys for attn_fwd_splitkv: num_splits <= 0 picks as many ranges
// as fill one wave of CTAs (one per SM, the forward kernel's occupancy) without
// starting a second, partly empty one; ranges hold at least two 128-key tiles.
// The ranges are whole tiles, and only non-empty ones are launched.
constexpr int kMaxSplits = 64;

int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
    return 148;
  return n;
}

struct SplitPlan {
  int splits;
  int chunk;
};
SplitPlan plan_splits(int B, int Hq, int Hkv, int Nq, int Nkv, int d, int num_splits) {
  const int tiles = (Nkv + 127) / 128;
  long long s = num_splits;
  if (s <= 0) {
    const long long units = fwd_ctas(B, Hq, Hkv, Nq, d);
    const long long sms = sm_count();
    s = units >= sms ? 1 : sms / units;
    s = std::min<long long>(s, std::max(1, tiles / 2));
  }
  s = std::max<long long>(1, std::min<long long>({s, (long long)tiles, (long long)kMaxSplits}));
  const int chunk = (int)((tiles + s - 1) / s) * 128;
  return {(Nkv + chunk - 1) / chunk, chunk};
}

struct SplitLayout {
  size_t lse_off, total;
};
SplitLayout splitkv_layout(int splits, int B, int Hq, int Nq, int d) {
  const size_t rows = (size_t)splits * B * Hq * Nq;
  const size_t lse_off = round_up(rows * d * 4, 256);
  return {lse_off, round_up(lse_off + rows * 4, 256)};
}

}  // namespace

extern "C" {

attn_status_t attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                       int Hq, int Hkv, int Nq, int Nkv, int d, int causal, float scale,
                       void* stream) {
  attn_status_t s = check_args(q, k, v, o, lse, B, Hq, Hkv, Nq, Nkv, d, causal, scale, true, true);
  if (s != ATTN_OK) return s;
  return run_fwd(q, k, v, o, lse, B, Hq, Hkv, Nq, Nkv, d, causal, scale,
                 static_cast<cudaStream_t>(stream));
}

attn_status_t attn_fwd_partial(const void* q, const void* k, const void* v, float* o_part,
                               float* lse_part, int B, int Hq, int Hkv, int Nq, int Nkv, int d,
                               int causal, float scale, int kv_tail, void* stream) {
  attn_status_t s = check_args(q, k, v, o_part, lse_part, B, Hq, Hkv, Nq, Nkv, d, causal, scale);
  if (s != ATTN_OK) return s;
  if (kv_tail < 0 || (long long)Nkv + kv_tail > 0x7fffffffLL) return ATTN_ERR_INVALID_ARG;
  PartialArgs part;
  part.o_part = o_part;
  part.kv_tail = kv_tail;
  return run_fwd(q, k, v, nullptr, lse_part, B, Hq, Hkv, Nq, Nkv, d, causal, scale,
                 static_cast<cudaStream_t>(stream), part);
}

attn_status_t attn_merge_partials(const float* o_parts, const float* lse_parts, int num_parts,
                                  int B, int Hq, int Nq, int d, void* o, float* lse,
                                  void* stream) {
  if (!o_parts || !lse_parts || !o || !lse) return ATTN_ERR_INVALID_ARG;
  if (num_parts <= 0 || B <= 0 || Hq <= 0 || Nq <= 0 || d <= 0) return ATTN_ERR_INVALID_ARG;
  if (d != 64 && d != 96 && d != 128 && d != 256) return ATTN_ERR_UNSUPPORTED;
  if (!aligned16(o_parts) || !aligned16(lse_parts) || !aligned16(o) || !aligned16(lse))
    return ATTN_ERR_ALIGNMENT;
  return cuda_status(attn_sm100::launch_merge(o_parts, lse_parts, num_parts,
                                              (long long)B * Hq * Nq, d, o, lse,
                                              static_cast<cudaStream_t>(stream)));
}

long long attn_partial_packed_floats(int B, int Hq, int Nq, int d) {
  if (B <= 0 || Hq <= 0 || Nq <= 0 || d <= 0) return 0;
  const long long rows = (long long)B * Hq * Nq;
  return (rows * d + rows + 3) / 4 * 4;
}

attn_status_t attn_merge_partials_packed(const float* parts, int num_parts, int B, int Hq, int Nq,
                                         int d, void* o, float* lse, void* stream) {
  if (!parts || !o || !lse) return ATTN_ERR_INVALID_ARG;
  if (num_parts <= 0 || B <= 0 || Hq <= 0 || Nq <= 0 || d <= 0) return ATTN_ERR_INVALID_ARG;
  if (d != 64 && d != 96 && d != 128 && d != 256) return ATTN_ERR_UNSUPPORTED;
  if (!aligned16(parts) || !aligned16(o) || !aligned16(lse)) return ATTN_ERR_ALIGNMENT;
  const long long rows = (long long)B * Hq * Nq;
  const long long stride = attn_partial_packed_floats(B, Hq, Nq, d);
  return cuda_status(attn_sm100::launch_merge(parts, parts + rows * d, num_parts, rows, d, o, lse,
                                              static_cast<cudaStream_t>(stream), false, stride,
                                              stride));
}

int attn_fwd_splitkv_num_splits(int B, int Hq, int Hkv, int Nq, int Nkv, int d, int num_splits) {
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv || Nq <= 0 || Nkv <= 0 || d <= 0) return 0;
  return plan_splits(B, Hq, Hkv, Nq, Nkv, d, num_splits).splits;
}

size_t attn_fwd_splitkv_workspace_size(int B, int Hq, int Hkv, int Nq, int Nkv, int d,
                                       int num_splits) {
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv || Nq <= 0 || Nkv <= 0 || d <= 0) return 0;
  const SplitPlan plan = plan_splits(B, Hq, Hkv, Nq, Nkv, d, num_splits);
  return plan.splits == 1 ? 0 : splitkv_layout(plan.splits, B, Hq, Nq, d).total;
}

attn_status_t attn_fwd_partial_splitkv(const void* q, const void* k, const void* v, float* o_part,
                                       float* lse_part, int B, int Hq, int Hkv, int Nq, int Nkv,
                                       int d, int causal, float scale, int kv_tail, int num_splits,
                                       void* workspace, size_t workspace_bytes, void* stream) {
  attn_status_t s = check_args(q, k, v, o_part, lse_part, B, Hq, Hkv, Nq, Nkv, d, causal, scale);
  if (s != ATTN_OK) return s;
  if (kv_tail < 0 || (long long)Nkv + kv_tail > 0x7fffffffLL) return ATTN_ERR_INVALID_ARG;
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  const SplitPlan plan = plan_splits(B, Hq, Hkv, Nq, Nkv, d, num_splits);
  PartialArgs part;
  part.kv_tail = kv_tail;
  if (plan.splits == 1) {  // one range: the partial kernel writes the caller's buffers
    part.o_part = o_part;
    return run_fwd(q, k, v, nullptr, lse_part, B, Hq, Hkv, Nq, Nkv, d, causal, scale, st, part);
  }
  if ((long long)B * plan.splits > 65535) return ATTN_ERR_UNSUPPORTED;
  const SplitLayout lay = splitkv_layout(plan.splits, B, Hq, Nq, d);
  if (!workspace || !aligned16(workspace) || workspace_bytes < lay.total) return ATTN_ERR_WORKSPACE;
  uint8_t* const ws = static_cast<uint8_t*>(workspace);
  float* const o_parts = reinterpret_cast<float*>(ws);
  float* const lse_parts = reinterpret_cast<float*>(ws + lay.lse_off);
  part.o_part = o_parts;
  part.num_splits = plan.splits;
  part.kv_chunk = plan.chunk;
  s = run_fwd(q, k, v, nullptr, lse_parts, B, Hq, Hkv, Nq, Nkv, d, causal, scale, st, part);
  if (s != ATTN_OK) return s;
  // the merged result of the sub-ranges is the partial result of the whole range (fp32)
  return cuda_status(attn_sm100::launch_merge(o_parts, lse_parts, plan.splits,
                                              (long long)B * Hq * Nq, d, o_part, lse_part, st,
                                              true));
}

attn_status_t attn_fwd_splitkv(const void* q, const void* k, const void* v, void* o, float* lse,
                               int B, int Hq, int Hkv, int Nq, int Nkv, int d, int causal,
                               float scale, int num_splits, void* workspace,
                               size_t workspace_bytes, void* stream) {
  attn_status_t s = check_args(q, k, v, o, lse, B, Hq, Hkv, Nq, Nkv, d, causal, scale);
  if (s != ATTN_OK) return s;
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  const SplitPlan plan = plan_splits(B, Hq, Hkv, Nq, Nkv, d, num_splits);
  if (plan.splits == 1) return run_fwd(q, k, v, o, lse, B, Hq, Hkv, Nq, Nkv, d, causal, scale, st);
  if ((long long)B * plan.splits > 65535) return ATTN_ERR_UNSUPPORTED;
  const SplitLayout lay = splitkv_layout(plan.splits, B, Hq, Nq, d);
  if (!workspace || !aligned16(workspace) || workspace_bytes < lay.total) return ATTN_ERR_WORKSPACE;
  uint8_t* const ws = static_cast<uint8_t*>(workspace);
  float* const o_parts = reinterpret_cast<float*>(ws);
  float* const lse_parts = reinterpret_cast<float*>(ws + lay.lse_off);
  PartialArgs part;
  part.o_part = o_parts;
  part.num_splits = plan.splits;
  part.kv_chunk = plan.chunk;
  s = run_fwd(q, k, v, nullptr, lse_parts, B, Hq, Hkv, Nq, Nkv, d, causal, scale, st, part);
  if (s != ATTN_OK) return s;
  return cuda_status(attn_sm100::launch_merge(o_parts, lse_parts, plan.splits,
                                              (long long)B * Hq * Nq, d, o, lse, st));
}

attn_status_t attn_fwd_varlen(const void* q, const void* k, const void* v, void* o, float* lse,
                              const int* cu_seqlens_q, const int* cu_seqlens_k, int num_seqs,
                              int max_seqlen_q, int total_q, int total_k, int Hq, int Hkv, int d,
                              int causal, float scale, void* stream) {
  if (!cu_seqlens_q || !cu_seqlens_k) return ATTN_ERR_INVALID_ARG;
  if (num_seqs <= 0 || max_seqlen_q <= 0) return ATTN_ERR_INVALID_ARG;
  // the dense checks with B = 1 cover pointers, sizes, heads, scale, d and alignment
  attn_status_t s = check_args(q, k, v, o, lse, 1, Hq, Hkv, total_q, total_k, d, causal, scale,
                               true, true);
  if (s != ATTN_OK) return s;
  if (num_seqs > 65535) return ATTN_ERR_UNSUPPORTED;
  if ((reinterpret_cast<uintptr_t>(cu_seqlens_q) | reinterpret_cast<uintptr_t>(cu_seqlens_k)) & 3u)
    return ATTN_ERR_ALIGNMENT;
  return run_fwd_varlen(q, k, v, o, lse, cu_seqlens_q, cu_seqlens_k, num_seqs, max_seqlen_q,
                        total_q, total_k, Hq, Hkv, d, causal, scale, static_cast<cudaStream_t>(stream));
}

size_t attn_fwd_host_buffer_size(int B, int Hq, int Hkv, int Nq, int Nkv, int d) {
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || Nq <= 0 || Nkv <= 0 || d <= 0) return 0;
  return host_layout(B, Hq, Hkv, Nq, Nkv, d).total;
}

attn_status_t attn_fwd_host(const void* q_host, const void* k_host, const void* v_host,
                            void* o_host, float* lse_host, int B, int Hq, int Hkv, int Nq, int Nkv,
                            int d, int causal, float scale, void* dev_buf, size_t dev_buf_bytes,
                            void* stream) {
  attn_status_t s = check_args(q_host, k_host, v_host, o_host, lse_host, B, Hq, Hkv, Nq, Nkv, d,
                               causal, scale, true, true);
  if (s != ATTN_OK) return s;
  if (!dev_buf || !aligned16(dev_buf)) return ATTN_ERR_WORKSPACE;
  const HostLayout L = host_layout(B, Hq, Hkv, Nq, Nkv, d);
  if (dev_buf_bytes < L.total) return ATTN_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char* base = static_cast<char*>(dev_buf);
  HostPipe* P = host_pipe();
  if (!P || !device_status_ptr()) return ATTN_ERR_CUDA;
  int dev = 0;
  cudaGetDevice(&dev);
  // Pipeline over chunks of whole kv-head groups (flattened over batch and
  // heads, so each chunk is contiguous in every tensor): chunk c's inputs are
  // copied on P->in while chunk c-1 computes on `st` and chunk c-2's outputs
  // are copied back on P->out. Each chunk is attn_fwd on a sub-problem with
  // B = 1, Hq = its query heads, Hkv = its kv heads.
  const int G = Hq / Hkv;
  const long long groups = (long long)B * Hkv;
  const int n_chunks = (int)std::min<long long>(kHostChunks, groups);
  if ((groups + n_chunks - 1) / n_chunks * G > 65535) return ATTN_ERR_UNSUPPORTED;  // grid y of a chunk
  const size_t q_head = 2ull * Nq * d, kv_head = 2ull * Nkv * d, lse_head = 4ull * Nq;
  const char* qh = static_cast<const char*>(q_host);
  const char* kh = static_cast<const char*>(k_host);
  const char* vh = static_cast<const char*>(v_host);
  char* oh = static_cast<char*>(o_host);
  char* lh = reinterpret_cast<char*>(lse_host);
  auto fail = [&](cudaError_t e) { return e == cudaSuccess ? ATTN_OK : cuda_status(e); };
  std::unique_lock<std::mutex> lock(g_pipe_mutex[dev]);
  cudaError_t e = cudaEventRecord(P->start, st);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(P->in, P->start, 0);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(P->out, P->start, 0);
  if (e != cudaSuccess) return fail(e);
  for (int c = 0; c < n_chunks; ++c) {
    const long long g0 = groups * c / n_chunks, g1 = groups * (c + 1) / n_chunks;
    const long long h0 = g0 * G, nh = (g1 - g0) * G, nk = g1 - g0;
    e = cudaMemcpyAsync(base + L.q + h0 * q_head, qh + h0 * q_head, nh * q_head, cudaMemcpyHostToDevice, P->in);
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(base + L.k + g0 * kv_head, kh + g0 * kv_head, nk * kv_head, cudaMemcpyHostToDevice, P->in);
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(base + L.v + g0 * kv_head, vh + g0 * kv_head, nk * kv_head, cudaMemcpyHostToDevice, P->in);
    if (e == cudaSuccess) e = cudaEventRecord(P->loaded[c], P->in);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(st, P->loaded[c], 0);
    if (e != cudaSuccess) return fail(e);
    s = run_fwd(base + L.q + h0 * q_head, base + L.k + g0 * kv_head, base + L.v + g0 * kv_head,
                base + L.o + h0 * q_head, reinterpret_cast<float*>(base + L.lse + h0 * lse_head), 1,
                (int)nh, (int)nk, Nq, Nkv, d, causal, scale, st);
    if (s != ATTN_OK) return s;
    e = cudaEventRecord(P->computed[c], st);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(P->out, P->computed[c], 0);
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(oh + h0 * q_head, base + L.o + h0 * q_head, nh * q_head, cudaMemcpyDeviceToHost, P->out);
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(lh + h0 * lse_head, base + L.lse + h0 * lse_head, nh * lse_head,
                          cudaMemcpyDeviceToHost, P->out);
    if (e != cudaSuccess) return fail(e);
  }
  e = cudaEventRecord(P->done, P->out);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(st, P->done, 0);
  lock.unlock();
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  return fail(e);
}

size_t attn_fwd_q8_workspace_size(int B, int Hq, int Hkv, int Nq, int Nkv, int d) {
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || Nq <= 0 || Nkv <= 0 || d <= 0) return 0;
  size_t off[kQ8Regions + 1];
  q8_layout(B, Hq, Hkv, Nq, Nkv, d, off);
  return off[kQ8Regions];
}

attn_status_t attn_q8_workspace_offsets(int B, int Hq, int Hkv, int Nq, int Nkv, int d,
                                        size_t* offsets) {
  if (!offsets || B <= 0 || Hq <= 0 || Hkv <= 0 || Nq <= 0 || Nkv <= 0 || d <= 0)
    return ATTN_ERR_INVALID_ARG;
  size_t off[kQ8Regions + 1];
  q8_layout(B, Hq, Hkv, Nq, Nkv, d, off);
  for (int i = 0; i <= kQ8Regions; ++i) offsets[i] = off[i];
  return ATTN_OK;
}

attn_status_t attn_fwd_q8(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                          int Hq, int Hkv, int Nq, int Nkv, int d, int causal, float scale,
                          void* workspace, size_t workspace_bytes, void* stream) {
  attn_status_t s = check_args(q, k, v, o, lse, B, Hq, Hkv, Nq, Nkv, d, causal, scale, false);
  if (s != ATTN_OK) return s;
  return run_q8(q, k, v, o, lse, B, Hq, Hkv, Nq, Nkv, d, causal, scale, workspace,
                workspace_bytes, false, static_cast<cudaStream_t>(stream));
}

attn_status_t attn_q8_prepass(const void* q, const void* k, const void* v, int B, int Hq, int Hkv,
                              int Nq, int Nkv, int d, void* workspace, size_t workspace_bytes,
                              void* stream) {
  // o / lse are not touched by the prepass; reuse the common checks with q in their place
  attn_status_t s = check_args(q, k, v, q, q, B, Hq, Hkv, Nq, Nkv, d, 0, 1.0f, false);
  if (s != ATTN_OK) return s;
  return run_q8(q, k, v, nullptr, nullptr, B, Hq, Hkv, Nq, Nkv, d, 0, 1.0f, workspace,
                workspace_bytes, true, static_cast<cudaStream_t>(stream));
}

attn_status_t attn_fwd_fp8(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                           int Hq, int Hkv, int Nq, int Nkv, int d, int causal, float scale,
                           void* workspace, size_t workspace_bytes, void* stream) {
  attn_status_t s = check_args(q, k, v, o, lse, B, Hq, Hkv, Nq, Nkv, d, causal, scale, false);
  if (s != ATTN_OK) return s;
  return run_q8(q, k, v, o, lse, B, Hq, Hkv, Nq, Nkv, d, causal, scale, workspace,
                workspace_bytes, false, static_cast<cudaStream_t>(stream), true);
}

attn_status_t attn_fp8_prepass(const void* q, const void* k, const void* v, int B, int Hq, int Hkv,
                               int Nq, int Nkv, int d, void* workspace, size_t workspace_bytes,
                               void* stream) {
  attn_status_t s = check_args(q, k, v, q, q, B, Hq, Hkv, Nq, Nkv, d, 0, 1.0f, false);
  if (s != ATTN_OK) return s;
  return run_q8(q, k, v, nullptr, nullptr, B, Hq, Hkv, Nq, Nkv, d, 0, 1.0f, workspace,
                workspace_bytes, true, static_cast<cudaStream_t>(stream), true);
}

size_t attn_bwd_workspace_size(int B, int Hq, int Hkv, int Nq, int Nkv, int d) {
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || Nq <= 0 || Nkv <= 0 || d <= 0) return 0;
  return bwd_layout(B, Hq, Nq, d).total;
}

attn_status_t attn_bwd(const void* q, const void* k, const void* v, const void* o,
                       const float* lse, const void* dout, void* dq, void* dk, void* dv, int B,
                       int Hq, int Hkv, int Nq, int Nkv, int d, int causal, float scale,
                       void* workspace, size_t workspace_bytes, void* stream) {
  attn_status_t s = check_args(q, k, v, o, lse, B, Hq, Hkv, Nq, Nkv, d, causal, scale);
  if (s != ATTN_OK) return s;
  if (!dout || !dq || !dk || !dv) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(dout) || !aligned16(dq) || !aligned16(dk) || !aligned16(dv)) return ATTN_ERR_ALIGNMENT;
  if (!workspace || !aligned16(workspace) ||
      workspace_bytes < bwd_layout(B, Hq, Nq, d).total)
    return ATTN_ERR_WORKSPACE;
  return run_bwd(q, k, v, o, lse, dout, dq, dk, dv, nullptr, nullptr, B, Hq, Hkv, Nq, Nkv, Nq, Nkv, d,
                 causal, scale, workspace, static_cast<cudaStream_t>(stream));
}

attn_status_t attn_selftest_wait_timeout(int budget_us, void* stream) {
  if (budget_us < 1 || budget_us > 10000000) return ATTN_ERR_INVALID_ARG;
  int* status = device_status_ptr();
  if (!status) return ATTN_ERR_CUDA;
  selftest_wait_timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
      status, 1000ull * (unsigned long long)budget_us);
  return cuda_status(cudaGetLastError());
}

size_t attn_bwd_varlen_workspace_size(int num_seqs, int Hq, int max_seqlen_q, int d) {
  if (num_seqs <= 0 || Hq <= 0 || max_seqlen_q <= 0 || d <= 0) return 0;
  return bwd_layout(num_seqs, Hq, max_seqlen_q, d).total;
}

attn_status_t attn_bwd_varlen(const void* q, const void* k, const void* v, const void* o,
                              const float* lse, const void* dout, void* dq, void* dk, void* dv,
                              const int* cu_seqlens_q, const int* cu_seqlens_k, int num_seqs,
                              int max_seqlen_q, int max_seqlen_k, int total_q, int total_k, int Hq,
                              int Hkv, int d, int causal, float scale, void* workspace,
                              size_t workspace_bytes, void* stream) {
  if (!cu_seqlens_q || !cu_seqlens_k) return ATTN_ERR_INVALID_ARG;
  if (num_seqs <= 0 || max_seqlen_q <= 0 || max_seqlen_k <= 0) return ATTN_ERR_INVALID_ARG;
  // the dense checks with B = 1 cover pointers, sizes, heads, scale, d and alignment
  attn_status_t s = check_args(q, k, v, o, lse, 1, Hq, Hkv, total_q, total_k, d, causal, scale);
  if (s != ATTN_OK) return s;
  if (!dout || !dq || !dk || !dv) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(dout) || !aligned16(dq) || !aligned16(dk) || !aligned16(dv)) return ATTN_ERR_ALIGNMENT;
  if ((reinterpret_cast<uintptr_t>(cu_seqlens_q) | reinterpret_cast<uintptr_t>(cu_seqlens_k)) & 3u)
    return ATTN_ERR_ALIGNMENT;
  if (num_seqs > 65535) return ATTN_ERR_UNSUPPORTED;
  if (!workspace || !aligned16(workspace) ||
      workspace_bytes < bwd_layout(num_seqs, Hq, max_seqlen_q, d).total)
    return ATTN_ERR_WORKSPACE;
  return run_bwd(q, k, v, o, lse, dout, dq, dk, dv, cu_seqlens_q, cu_seqlens_k, num_seqs, Hq, Hkv,
                 total_q, total_k, max_seqlen_q, max_seqlen_k, d, causal, scale, workspace,
                 static_cast<cudaStream_t>(stream));
}

attn_status_t attn_get_status_ex(void* stream, int* where) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return ATTN_ERR_CUDA;
  int h[2] = {0, 0};
  if (cudaMemcpyFromSymbol(h, g_status, sizeof(h)) != cudaSuccess) return ATTN_ERR_CUDA;
  if (where) *where = h[1];
  if (h[0] != 0) {
    const int zero[2] = {0, 0};
    if (cudaMemcpyToSymbol(g_status, zero, sizeof(zero)) != cudaSuccess) return ATTN_ERR_CUDA;
  }
  return static_cast<attn_status_t>(h[0]);
}

attn_status_t attn_get_status(void* stream) { return attn_get_status_ex(stream, nullptr); }

attn_status_t attn_set_timeout_ms(int ms) {
  if (ms < 1) return ATTN_ERR_INVALID_ARG;
  g_timeout_ns.store((long long)ms * 1000000LL);
  return ATTN_OK;
}

const char* attn_status_string(attn_status_t s) {
  switch (s) {
    case ATTN_OK: return "ATTN_OK";
    case ATTN_ERR_INVALID_ARG: return "ATTN_ERR_INVALID_ARG";
    case ATTN_ERR_UNSUPPORTED: return "ATTN_ERR_UNSUPPORTED";
    case ATTN_ERR_ALIGNMENT: return "ATTN_ERR_ALIGNMENT";
    case ATTN_ERR_CUDA: return "ATTN_ERR_CUDA";
    case ATTN_ERR_TIMEOUT: return "ATTN_ERR_TIMEOUT";
    case ATTN_ERR_WORKSPACE: return "ATTN_ERR_WORKSPACE";
  }
  return "ATTN_ERR_UNKNOWN";
}

int attn_version(void) { return 100; }

int attn_last_cuda_error(const char** message) {
  if (message) *message = cudaGetErrorString(g_last_cuda_error);
  return static_cast<int>(g_last_cuda_error);
}

}  // extern "C"
