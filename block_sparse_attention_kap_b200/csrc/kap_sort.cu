// kap_sort: flag-grouped sorting of the Kernel-Aware Proxy (CoSA technical
// summary Sec. 2.2): per (head, Q-block), the causally visible KV blocks are
// ordered HRM blocks first, then by estimated score, ties by block index,
// and the first k_I = max(1, ceil(n_I * budget)) form the computation-order
// mask M_KAP.  One CTA per (b, h, Q-block): a shared-memory bitonic sort of
// packed 64-bit keys (ranking key in the high word, inverted block index in
// the low word, so keys are unique and ties resolve to the smaller index).
#include "internal.h"

namespace cosa {

namespace {

constexpr int kSortThreads = 256;

__device__ __forceinline__ uint32_t orderable(float f) {
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ int causal_blocks(int I, int Nq, int Nkv, int bq, int bk, int nkb) {
  const int last_tok = min((I + 1) * bq, Nq) - 1;
  return min(nkb, (Nkv - Nq + last_tok) / bk + 1);
}

__global__ void __launch_bounds__(kSortThreads) kap_sort_kernel(SortParams p, int pmax) {
  extern __shared__ uint64_t keys[];
  __shared__ int hrm_total;
  const int row = blockIdx.x;
  const int I = row % p.nqb;
  const int n = causal_blocks(I, p.Nq, p.Nkv, p.bq, p.bk, p.nkb);
  int k = (int)(((long long)n * p.bp + 9999) / 10000);
  k = max(1, min(k, n));
  int P = 1;
  while (P < n) P <<= 1;
  if (P > pmax) P = pmax;   // cannot happen: pmax >= nkb >= n
  if (threadIdx.x == 0) hrm_total = 0;
  const float* rk = p.rank + (size_t)row * p.nkb;
  int my_hrm = 0;
  for (int i = threadIdx.x; i < P; i += kSortThreads) {
    uint64_t key = 0;
    if (i < n) {
      const float r = rk[i];
      my_hrm += (r == 1.0f);
      key = ((uint64_t)orderable(r) << 32) | (uint64_t)(0xffffffffu - (uint32_t)i);
    }
    keys[i] = key;
  }
  __syncthreads();
  if (my_hrm) atomicAdd(&hrm_total, my_hrm);
  // bitonic network, descending
  for (int kk = 2; kk <= P; kk <<= 1) {
    for (int j = kk >> 1; j > 0; j >>= 1) {
      for (int i = threadIdx.x; i < P; i += kSortThreads) {
        const int ixj = i ^ j;
        if (ixj > i) {
          const uint64_t a = keys[i], b = keys[ixj];
          const bool desc = (i & kk) == 0;
          if (desc ? (a < b) : (a > b)) {
            keys[i] = b;
            keys[ixj] = a;
          }
        }
      }
      __syncthreads();
    }
  }
  int32_t* ord = p.order + (size_t)row * p.kmax;
  for (int t = threadIdx.x; t < p.kmax; t += kSortThreads)
    ord[t] = t < k ? (int32_t)(0xffffffffu - (uint32_t)(keys[t] & 0xffffffffu)) : -1;
  if (threadIdx.x == 0) {
    p.count[row] = k;
    if (p.hrm_count) p.hrm_count[row] = hrm_total;
  }
  // blocks no query of this Q-block can see: -inf score, no flag
  if (p.block_score)
    for (int j = n + threadIdx.x; j < p.nkb; j += kSortThreads) p.block_score[(size_t)row * p.nkb + j] = -INFINITY;
  if (p.hrm_flags)
    for (int j = n + threadIdx.x; j < p.nkb; j += kSortThreads) p.hrm_flags[(size_t)row * p.nkb + j] = 0;
}

__global__ void dense_order_kernel(int rows, int nqb, int nkb, int Nq, int Nkv, int bq, int bk, int kmax,
                                   int32_t* order, int32_t* count) {
  const int row = blockIdx.x;
  const int n = causal_blocks(row % nqb, Nq, Nkv, bq, bk, nkb);
  for (int t = threadIdx.x; t < kmax; t += blockDim.x) order[(size_t)row * kmax + t] = t < n ? t : -1;
  if (threadIdx.x == 0) count[row] = n;
}

}  // namespace

cudaError_t launch_kap_sort(const SortParams& p, cudaStream_t st) {
  const int rows = p.B * p.Hq * p.nqb;
  if (rows == 0) return cudaSuccess;
  int pmax = 1;
  while (pmax < p.nkb) pmax <<= 1;
  const size_t smem = (size_t)pmax * sizeof(uint64_t);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(kap_sort_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  kap_sort_kernel<<<rows, kSortThreads, smem, st>>>(p, pmax);
  return cudaGetLastError();
}

cudaError_t launch_dense_order(int rows, int nqb, int nkb, int Nq, int Nkv, int bq, int bk, int kmax,
                               int32_t* order, int32_t* count, cudaStream_t st) {
  if (rows == 0) return cudaSuccess;
  dense_order_kernel<<<rows, 256, 0, st>>>(rows, nqb, nkb, Nq, Nkv, bq, bk, kmax, order, count);
  return cudaGetLastError();
}

}  // namespace cosa
