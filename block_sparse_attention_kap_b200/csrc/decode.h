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

// Parameters of the decode-step attention (decode_attend.cu).
struct DecodeAttendParams {
  int B, Hq, Hkv, Nkv, nkb, bk, paged, num_pages;
  int kmax;                     // row stride of order
  const uint16_t* q;            // [B, Hq, d] bf16: the query at position Nkv-1
  const uint16_t* k;            // [B, Hkv, Nkv, d] or pages [num_pages, Hkv, bk, d]
  const uint16_t* v;
  const int32_t* page_table;    // [B, nKB] when paged
  const int32_t* order;         // [B*Hq, kmax]
  const int32_t* count;         // [B*Hq]
  float T;                      // skip threshold, raw-logit units (-inf: never skip)
  float scale_log2, scale_ln;   // log2(e)/sqrt(d), 1/sqrt(d)
  uint16_t* out;                // [B*Hq, d] bf16
  float* lse;                   // optional [B*Hq]
  uint32_t* skip_bits;          // optional [B*Hq, skip_words]
  int skip_words;
  // workspace, carved by launch_decode_attend
  float* logits;                // [B*Hq, kmax, bk]
  float* mloc;                  // [B*Hq, kmax]
  float* partials;              // [B*Hq, max_producers, d + 1]
  uint32_t* counters;           // [B*Hq]
  int max_producers;
};
size_t decode_attend_workspace(int rows, int kmax, int bk);
size_t decode_attend_smem(int kmax, int bk);
cudaError_t launch_decode_attend(DecodeAttendParams p, uint8_t* workspace, cudaStream_t st);

}  // namespace cosa
