// Parameters of the decode-step proxy (decode_plan.cu).
#pragma once
#include "internal.h"

namespace cosa {

struct DecodePlanParams {
  int B, Hq, Hkv;
  int nkb, nkp, kpb;            // KV blocks, pooled keys per kv-head (Nkv/s), pooled keys per block (bk/s)
  int kp_stride;                // pooled-key rows per kv-head in kp
  int k, kmax;                  // blocks kept per row, row stride of order
  const uint16_t* q;            // [B, Hq, d] bf16: the query at position Nkv-1
  const uint16_t* kp;           // [B, Hkv, kp_stride, d] bf16 pooled keys
  int32_t* order;               // [B, Hq, kmax]
  int32_t* count;               // [B, Hq]
  int32_t* hrm_count;           // optional [B, Hq]
  float* block_score;           // optional [B, Hq, nKB]
  uint8_t* hrm_flags;           // optional [B, Hq, nKB]
};
size_t decode_plan_smem(int nkb, int k);
cudaError_t launch_decode_plan(const DecodePlanParams& p, cudaStream_t st);

}  // namespace cosa
