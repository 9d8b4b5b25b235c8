// block_union: the selection stage of CompactAttention ("CompactAttention:
// Accelerating Chunked Prefill with Block-Union KV Selection", method,
// selection stage): a per-head block-sparse selection -- here M_KAP, the
// (head, Q-block) -> KV-block lists of kap_sort -- becomes one KV block table
// per (batch, kv-head group) by a union over the Q-blocks of the chunk and
// over the query heads that share the kv-head.  Every block any Q-block or
// head of the group selected stays selected, and no other block enters.
//
// union_table_kernel: one CTA per (b, kv-head).  The selected block indices
// of the G heads x nQB Q-blocks are OR-ed into a shared-memory bitmap (one
// bit per KV block), which is compacted in ascending block order with a
// block-wide scan of the words' popcounts.
// union_expand_kernel: one warp per (b, h, Q-block) writes the table entries
// that Q-block can see causally (a prefix: the table ascends) as an
// attention order, so cosa_attend executes the union.
#include "block_union.h"

namespace cosa {

namespace {

constexpr int kUnionThreads = 512;

__device__ __forceinline__ int visible_blocks(int I, int Nq, int Nkv, int bq, int bk, int nkb) {
  const int last_tok = min((I + 1) * bq, Nq) - 1;
  return min(nkb, (Nkv - Nq + last_tok) / bk + 1);
}

__global__ void __launch_bounds__(kUnionThreads) union_table_kernel(UnionParams p) {
  extern __shared__ uint32_t bm[];                     // nkb bits, then per-warp partial sums
  const int words = (p.nkb + 31) >> 5;
  int* warp_sum = reinterpret_cast<int*>(bm + words);
  const int bg = blockIdx.x;
  const int b = bg / p.Hkv, g = bg - b * p.Hkv;
  const int G = p.Hq / p.Hkv;
  for (int w = threadIdx.x; w < words; w += blockDim.x) bm[w] = 0u;
  __syncthreads();

  // OR every selected block of the group's G heads x nQB Q-blocks into the bitmap
  const long long per_head = (long long)p.nqb * p.kmax;
  const long long entries = (long long)G * per_head;
  const int32_t* ord = p.order + ((long long)b * p.Hq + (long long)g * G) * per_head;
  const int32_t* cnt = p.count + ((long long)b * p.Hq + (long long)g * G) * p.nqb;
  for (long long e = threadIdx.x; e < entries; e += blockDim.x) {
    const int row = (int)(e / p.kmax), t = (int)(e - (long long)row * p.kmax);
    const int c = min(max(cnt[row], 0), p.kmax);
    if (t < c) {
      const int j = ord[e];
      if (j >= 0 && j < p.nkb) atomicOr(&bm[j >> 5], 1u << (j & 31));
    }
  }
  __syncthreads();

  // compaction: thread t owns words [t*wpt, (t+1)*wpt); exclusive scan of their popcounts
  const int wpt = (words + blockDim.x - 1) / blockDim.x;
  const int w0 = threadIdx.x * wpt, w1 = min(words, w0 + wpt);
  int mine = 0;
  for (int w = w0; w < w1; ++w) mine += __popc(bm[w]);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = mine;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) warp_sum[warp] = incl;
  __syncthreads();
  int before = 0, total = 0;
  const int nwarps = blockDim.x >> 5;
  for (int w = 0; w < nwarps; ++w) {
    const int s = warp_sum[w];
    before += w < warp ? s : 0;
    total += s;
  }
  int pos = before + incl - mine;
  int32_t* tab = p.table + (long long)bg * p.nkb;
  for (int w = w0; w < w1; ++w) {
    uint32_t bits = bm[w];
    while (bits) {
      const int k = __ffs(bits) - 1;
      bits &= bits - 1;
      tab[pos++] = (w << 5) + k;
    }
  }
  for (int k = total + threadIdx.x; k < p.nkb; k += blockDim.x) tab[k] = -1;
  if (threadIdx.x == 0) p.table_len[bg] = total;
}

__global__ void __launch_bounds__(256) union_expand_kernel(UnionParams p, int rows) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x * (blockDim.x >> 5) + warp;
  if (row >= rows) return;
  const int I = row % p.nqb;
  const int h = (row / p.nqb) % p.Hq, b = row / (p.nqb * p.Hq);
  const int bg = b * p.Hkv + h / (p.Hq / p.Hkv);
  const int len = p.table_len[bg];
  const int32_t* tab = p.table + (long long)bg * p.nkb;
  const int lim = visible_blocks(I, p.Nq, p.Nkv, p.bq, p.bk, p.nkb);   // blocks 0 .. lim-1 are visible
  // the table ascends, so the visible entries are a prefix: count them
  int n = 0;
  for (int base = 0; base < len; base += 32) {
    const int k = base + lane;
    const bool vis = k < len && tab[k] < lim;
    n += __popc(__ballot_sync(0xffffffffu, vis));
  }
  int32_t* dst = p.union_order + (long long)row * p.union_kmax;
  for (int k = lane; k < p.union_kmax; k += 32) dst[k] = k < n ? tab[k] : -1;
  if (lane == 0) p.union_count[row] = n;
}

}  // namespace

cudaError_t launch_block_union(const UnionParams& p, cudaStream_t st) {
  const int groups = p.B * p.Hkv;
  if (groups == 0) return cudaSuccess;
  const int words = (p.nkb + 31) / 32;
  const size_t smem = (size_t)words * 4 + (kUnionThreads / 32) * sizeof(int);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(union_table_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  union_table_kernel<<<groups, kUnionThreads, smem, st>>>(p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess || !p.union_order) return e;
  const int rows = p.B * p.Hq * p.nqb;
  if (rows == 0) return cudaSuccess;
  union_expand_kernel<<<(rows + 7) / 8, 256, 0, st>>>(p, rows);
  return cudaGetLastError();
}

}  // namespace cosa
