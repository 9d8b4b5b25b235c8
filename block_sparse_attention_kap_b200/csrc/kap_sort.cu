// kap_sort: the ranking and flag-grouped sorting of the Kernel-Aware Proxy
// (CoSA technical summary Sec. 2.2) as a kernel of its own: one warp per
// (b, h, Q-block), several per CTA, synchronised only with __syncwarp; the
// work of each warp is rank_qblock (kap_rank.cuh).  It runs after kap_score,
// whose block scores Bs and partial row maxima it reads.
#include "kap_rank.cuh"

namespace cosa {

namespace {

constexpr int kMaxWarps = 8;

template <int RPQ>
__global__ void __launch_bounds__(32 * kMaxWarps) kap_sort_kernel(SortParams p, int pk, int rows) {
  extern __shared__ __align__(16) uint8_t dyn[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x * (blockDim.x >> 5) + warp;
  if (row >= rows) return;                       // whole warps only; no block-wide barrier below
  rank_qblock<RPQ>(p, row, pk, dyn + (size_t)warp * select_smem(p.nkb, pk), lane);
}

__global__ void dense_order_kernel(int rows, int nqb, int nkb, int Nq, int Nkv, int bq, int bk, int kmax,
                                   int32_t* order, int32_t* count) {
  const int row = blockIdx.x;
  const int n = kap_causal_blocks(row % nqb, Nq, Nkv, bq, bk, nkb);
  for (int t = threadIdx.x; t < kmax; t += blockDim.x) order[(size_t)row * kmax + t] = t < n ? t : -1;
  if (threadIdx.x == 0) count[row] = n;
}

}  // namespace

cudaError_t launch_kap_sort(const SortParams& p, cudaStream_t st) {
  const int rows = p.B * p.Hq * p.nqb;
  if (rows == 0) return cudaSuccess;
  int pk = 1;
  while (pk < p.kmax) pk <<= 1;
  const size_t per_warp = select_smem(p.nkb, pk);
  int warps = (int)((96 * 1024) / per_warp);
  warps = warps < 1 ? 1 : (warps > kMaxWarps ? kMaxWarps : warps);
  const size_t smem = per_warp * warps;
  if (smem > 227 * 1024) return cudaErrorInvalidValue;
  const unsigned grid = (unsigned)((rows + warps - 1) / warps);
#define COSA_LAUNCH_SORT(R)                                                                           \
  case R: {                                                                                           \
    cudaError_t e = cudaFuncSetAttribute(kap_sort_kernel<R>, cudaFuncAttributeMaxDynamicSharedMemorySize, \
                                         (int)smem);                                                  \
    if (e != cudaSuccess) return e;                                                                   \
    kap_sort_kernel<R><<<grid, 32 * warps, smem, st>>>(p, pk, rows);                                  \
    break;                                                                                            \
  }
  switch (p.rpq) {
    COSA_LAUNCH_SORT(2)
    COSA_LAUNCH_SORT(4)
    COSA_LAUNCH_SORT(8)
    COSA_LAUNCH_SORT(16)
    COSA_LAUNCH_SORT(32)
    default:
      return cudaErrorInvalidValue;
  }
#undef COSA_LAUNCH_SORT
  return cudaGetLastError();
}

cudaError_t launch_dense_order(int rows, int nqb, int nkb, int Nq, int Nkv, int bq, int bk, int kmax,
                               int32_t* order, int32_t* count, cudaStream_t st) {
  if (rows == 0) return cudaSuccess;
  dense_order_kernel<<<rows, 256, 0, st>>>(rows, nqb, nkb, Nq, Nkv, bq, bk, kmax, order, count);
  return cudaGetLastError();
}

}  // namespace cosa
