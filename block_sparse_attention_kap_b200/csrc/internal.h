// Internal launch interface between the host front end (cosa_api.cu) and
// the kernels.  Not part of the public C ABI.
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace cosa {

constexpr int kD = 128;          // head dimension the kernels implement
constexpr int kTileRows = 128;   // MMA M (query rows per tile) and pooled rows/keys per KAP tile

// ---------------------------------------------------------------- KAP pooling
struct PoolParams {
  const uint16_t* q;            // [B, Hq, Nq, d]
  const uint16_t* k;            // [B, Hkv, Nkv, d] or paged [P, Hkv, bk, d]
  const int32_t* page_table;    // [B, nKB] when paged
  uint16_t* qp;                 // [B, Hq, Nq/s, d]
  uint16_t* kp;                 // [B, Hkv, kp_stride, d]; rows kp_first .. Nkv/s-1 are written
  int B, Hq, Hkv, Nq, Nkv, s, bk, nkb, paged, num_pages;
  int kp_first;                 // first pooled key row to compute (rows below are already pooled)
  int kp_stride;                // pooled-key rows per kv-head in kp (>= Nkv/s)
  long long q_items;            // B*Hq*Nq/s pooled rows of Q
  long long k_items;            // B*Hkv*(Nkv/s - kp_first) pooled rows of K
};
cudaError_t launch_kap_pool(const PoolParams& p, cudaStream_t st);

// ---------------------------------------------------------------- KAP scoring
// Pooled key tiles a row tile of 128 pooled rows sees: tiles 0 .. nT-1.
__host__ __device__ inline int kap_row_tiles_seen(int R, int nqp, int nkp, int off_p) {
  const int rows_valid = min(kTileRows, nqp - R * kTileRows);
  const int cmax = off_p + R * kTileRows + rows_valid - 1;    // last pooled key any row sees
  return min(cmax / kTileRows + 1, (nkp + kTileRows - 1) / kTileRows);
}
// Split `split` of S covers key tiles [t0, t1) of the nT a row tile sees.
__host__ __device__ inline void kap_split_range(int nT, int S, int split, int& t0, int& t1) {
  const int per = (nT + S - 1) / S;
  t0 = min(nT, split * per);
  t1 = min(nT, t0 + per);
}

struct ScoreParams {
  int B, Hq, Hkv, G;
  int nqp, nkp;                 // pooled rows per head (Nq/s), pooled keys per kv-head (Nkv/s)
  int kp_stride;                // pooled-key rows per kv-head in the Kp buffer (>= nkp)
  int off_p;                    // (Nkv - Nq) / s
  int nkb;
  int kpb;                      // pooled keys per KV block (bk / s)
  int n_row_tiles;              // ceil(nqp / 128)
  int splits;                   // S: each row tile's key tiles are cut into S work items
  int rpq;                      // pooled rows per Q-block (bq / s): the Bs layout groups them
  float* bs;                    // [B*Hq, n_row_tiles, nKB, 128] max-pooled block scores
  float* part_max;              // [B*Hq, n_row_tiles, S, 2, 128] row max of each item and column half
  int32_t* part_arg;            // ... and the first block attaining it (-1: none)
  uint32_t* status;
};
cudaError_t launch_kap_score(const CUtensorMap& tm_qp, const CUtensorMap& tm_kp, const ScoreParams& p,
                             cudaStream_t st);

// ---------------------------------------------------------------- KAP rank + sort
struct SortParams {
  int B, Hq, nqb, nkb, Nq, Nkv, bq, bk;
  int rpq;                      // pooled rows per Q-block (bq / s)
  int nqp, n_row_tiles, splits; // as in ScoreParams
  int bp;                       // budget in basis points
  int kmax;
  const float* bs;              // from kap_score
  const float* part_max;
  const int32_t* part_arg;
  int32_t* order;               // [B, Hq, nQB, kmax]
  int32_t* count;               // [B, Hq, nQB]
  int32_t* hrm_count;           // optional [B, Hq, nQB]
  float* block_score;           // optional [B, Hq, nQB, nKB]: -inf written for invisible blocks
  uint8_t* hrm_flags;           // optional [B, Hq, nQB, nKB]: 0 written for invisible blocks
};
cudaError_t launch_kap_sort(const SortParams& p, cudaStream_t st);
cudaError_t launch_dense_order(int rows, int nqb, int nkb, int Nq, int Nkv, int bq, int bk, int kmax,
                               int32_t* order, int32_t* count, cudaStream_t st);

// ---------------------------------------------------------------- OSK
struct OskParams {
  int B, Hq, Hkv, G, Nq, Nkv, bq, nqb, nkb, paged, num_pages;
  const int32_t* page_table;    // [B, nKB] when paged
  const int32_t* order;         // [B, Hq, nQB, kmax]
  const int32_t* count;         // [B, Hq, nQB]
  int kmax;
  float T;                      // skip threshold, raw-logit units (-inf: never skip)
  float scale_log2;             // log2(e) / sqrt(d)
  float scale_ln;               // 1 / sqrt(d)
  uint16_t* out;                // [B, Hq, Nq, d] bf16
  float* lse;                   // optional [B, Hq, Nq]
  uint32_t* skip_bits;          // optional [B, Hq, nQB, skip_words]
  int skip_words;
  uint32_t* status;
  int kv_tail;                  // keys in the last KV block when it is ragged (Nkv % bk), else 0
  uint64_t wait_limit_ns;       // limit of every pipeline wait (1 s; shorter only in the test hook)
  int stall_test;               // 0; 1 only in the wait-timeout test hook
};
cudaError_t launch_osk(const CUtensorMap& tm_q, const CUtensorMap& tm_k, const CUtensorMap& tm_v,
                       const OskParams& p, int bk, cudaStream_t st);
// The same with one order per (b, kv-head, Q-block) shared by the G query
// heads (order [B, Hkv, nQB, kmax], count [B, Hkv, nQB]); G even.
cudaError_t launch_osk_group(const CUtensorMap& tm_q, const CUtensorMap& tm_k, const CUtensorMap& tm_v,
                             const OskParams& p, int bk, cudaStream_t st);

}  // namespace cosa
