// Parameters of the block-union kernels (block_union.cu).
#pragma once
#include "internal.h"

namespace cosa {

// ---------------------------------------------------------------- block union
struct UnionParams {
  int B, Hq, Hkv, nqb, nkb, Nq, Nkv, bq, bk;
  const int32_t* order;         // [B, Hq, nQB, kmax] per-head selection (M_KAP)
  const int32_t* count;         // [B, Hq, nQB]
  int kmax;
  int32_t* table;               // [B, Hkv, nKB] union table, ascending, padded -1
  int32_t* table_len;           // [B, Hkv]
  int32_t* union_order;         // optional [B, Hq, nQB, union_kmax]: causally visible table prefix
  int32_t* union_count;         // [B, Hq, nQB] (with union_order)
  int union_kmax;
};
cudaError_t launch_block_union(const UnionParams& p, cudaStream_t st);

}  // namespace cosa
