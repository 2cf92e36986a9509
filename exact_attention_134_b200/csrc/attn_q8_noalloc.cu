// attn_q8_noalloc.cu — the 8-bit forward with its scratch in a static device
// array, for callers that cannot allocate device memory.
//
// Who needs this: code that is handed only its input and output buffers and no
// allocator or workspace (a plugin or hook inside another framework's
// inference engine, for instance), and programs that must not call cudaMalloc
// once they are serving — cudaMalloc can synchronise the device, and it fails
// outright when another allocator has already reserved the GPU's memory.
//
// The scratch is a file-scope __device__ array of kAttnQ8StaticScratchBytes
// (32 MiB); every GPU that loads this library holds it until the process
// exits. Host code cannot pass the array's name to a kernel (on the host it is
// only a stand-in symbol, not a device address), so the first call on each
// device looks up the array's device address with cudaGetSymbolAddress, with
// that device current, and caches it. With CUDA's default lazy module loading
// that lookup is also what loads this file's module onto the device, and so
// what reserves the 32 MiB: make the first call on each device at start-up,
// before other allocators take the GPU's memory and before any stream capture.
#include <mutex>

#include "attn_internal.h"

namespace {

constexpr size_t kAttnQ8StaticScratchBytes = 32ull << 20;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_q8_scratch[kAttnQ8StaticScratchBytes];

std::mutex g_scratch_mutex;
void* g_scratch_ptr[kMaxDevices] = {nullptr};

// Device address of g_q8_scratch on the current device (looked up once per device).
cudaError_t scratch_for_current_device(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (!g_scratch_ptr[dev]) {
    void* ptr = nullptr;
    e = cudaGetSymbolAddress(&ptr, g_q8_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_ptr[dev] = ptr;
  }
  *out = g_scratch_ptr[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" {

size_t attn_fwd_q8_static_scratch_bytes(void) { return kAttnQ8StaticScratchBytes; }

attn_status_t attn_fwd_q8_noalloc(const void* q, const void* k, const void* v, void* o,
                                  float* lse, int B, int Hq, int Hkv, int Nq, int Nkv, int d,
                                  int causal, float scale, void* stream) {
  attn_status_t s =
      attn_sm100::validate_fwd_args(q, k, v, o, lse, B, Hq, Hkv, Nq, Nkv, d, causal, scale);
  if (s != ATTN_OK) return s;
  // problem too large for the static array: rejected before anything is queued
  if (attn_fwd_q8_workspace_size(B, Hq, Hkv, Nq, Nkv, d) > kAttnQ8StaticScratchBytes)
    return ATTN_ERR_WORKSPACE;
  void* scratch = nullptr;
  const cudaError_t e = scratch_for_current_device(&scratch);
  if (e != cudaSuccess) return attn_sm100::cuda_error_status(e);
  // Nothing in the scratch has to start at zero: every region the kernels read
  // is written earlier in the same call.
  return attn_sm100::q8_forward_with_workspace(q, k, v, o, lse, B, Hq, Hkv, Nq, Nkv, d, causal,
                                                scale, scratch, kAttnQ8StaticScratchBytes,
                                                static_cast<cudaStream_t>(stream));
}

}  // extern "C"
