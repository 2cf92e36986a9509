// attn_internal.h — declarations shared between the C-ABI layer and the
// kernel translation units (not part of the public ABI).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/attn.h"

namespace attn_sm100 {

// Kernel parameters of the bf16 forward (tensor maps are passed separately).
struct FwdParams {
  float* lse;                     // fp32 [B, Hq, Nq]
  int* status;                    // device status word: [0] code, [1] where
  int Nq, Nkv, Hq, Hkv;
  int causal;
  int num_row_blocks;             // ceil(Nq / rows per CTA)
  float scale_log2;               // scale * log2(e)
  unsigned long long timeout_ns;  // budget of every pipeline wait
};

cudaError_t launch_fwd_bf16(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                            const CUtensorMap& to, const FwdParams& p, int B, int Hq, int d,
                            cudaStream_t stream);
int fwd_rows_per_cta();

}  // namespace attn_sm100
