// kap_sort: flag-grouped sorting of the Kernel-Aware Proxy (CoSA technical
// summary Sec. 2.2): per (head, Q-block), the causally visible KV blocks are
// ordered HRM blocks first, then by estimated score, ties by block index,
// and the first k_I = max(1, ceil(n_I * budget)) form the computation-order
// mask M_KAP.
//
// One CTA per (b, h, Q-block).  Each block's ranking key (+1 for HRM blocks,
// else its score <= 0, written by kap_score) is mapped to an order-preserving
// 32-bit integer.  A 4-pass, 8-bit radix select finds the k-th largest value
// T; the blocks above T plus the lowest-indexed blocks equal to T (an ordered
// block scan) are compacted, and only those k keys -- packed with the
// inverted block index so ties resolve to the smaller index -- are sorted by
// a shared-memory bitonic network.  At a 10% budget this sorts a tenth of
// the keys a full sort would.
#include "internal.h"

namespace cosa {

namespace {

constexpr int kSortThreads = 256;
constexpr int kWarps = kSortThreads / 32;

__device__ __forceinline__ uint32_t orderable(float f) {
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ int causal_blocks(int I, int Nq, int Nkv, int bq, int bk, int nkb) {
  const int last_tok = min((I + 1) * bq, Nq) - 1;
  return min(nkb, (Nkv - Nq + last_tok) / bk + 1);
}

// Exclusive block-wide prefix sum of v (all threads); returns the total too.
__device__ __forceinline__ int block_exclusive_scan(int v, int* warp_tot, int& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_tot[warp] = x;
  __syncthreads();
  int base = 0;
  total = 0;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) {
    const int t = warp_tot[w];
    if (w < warp) base += t;
    total += t;
  }
  __syncthreads();
  return base + x - v;
}

__global__ void __launch_bounds__(kSortThreads) kap_sort_kernel(SortParams p, int pmax) {
  extern __shared__ uint64_t dyn[];
  uint64_t* sel = dyn;                                          // [pmax] selected keys
  uint32_t* hi = reinterpret_cast<uint32_t*>(dyn + pmax);        // [pmax] orderable ranking keys
  __shared__ int hist[256];
  __shared__ int warp_tot[kWarps];
  __shared__ uint32_t s_prefix;
  __shared__ int s_remaining, s_hrm;

  const int tid = threadIdx.x;
  const int row = blockIdx.x;
  const int I = row % p.nqb;
  const int n = causal_blocks(I, p.Nq, p.Nkv, p.bq, p.bk, p.nkb);
  int k = (int)(((long long)n * p.bp + 9999) / 10000);
  k = max(1, min(k, n));
  const float* rk = p.rank + (size_t)row * p.nkb;
  const uint32_t hrm_key = orderable(1.0f);

  if (tid == 0) s_hrm = 0;
  int my_hrm = 0;
  for (int i = tid; i < n; i += kSortThreads) {
    const uint32_t h = orderable(rk[i]);
    hi[i] = h;
    my_hrm += (h == hrm_key);
  }
  __syncthreads();
  if (my_hrm) atomicAdd(&s_hrm, my_hrm);

  // ---------------------------------------------------------------- radix select of the k-th largest
  uint32_t T = 0;            // threshold value
  int need = k;              // how many of the elements equal to T are taken
  if (k < n) {
    uint32_t prefix = 0, mask = 0;
    int remaining = k;
    for (int shift = 24; shift >= 0; shift -= 8) {
      for (int b = tid; b < 256; b += kSortThreads) hist[b] = 0;
      __syncthreads();
      for (int i = tid; i < n; i += kSortThreads) {
        const uint32_t h = hi[i];
        if ((h & mask) == prefix) atomicAdd(&hist[(h >> shift) & 255u], 1);
      }
      __syncthreads();
      if (tid < 32) {
        // lane l owns digits 255-8l .. 248-8l (descending); suffix counts from the top digit
        int c[8], s = 0;
#pragma unroll
        for (int q = 0; q < 8; ++q) { c[q] = hist[255 - 8 * tid - q]; s += c[q]; }
        int incl = s;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int y = __shfl_up_sync(0xffffffffu, incl, o);
          if (tid >= o) incl += y;
        }
        const int excl = incl - s;
        // the lane whose range contains the remaining-th largest element
        if (excl < remaining && remaining <= incl) {
          int acc = excl;
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            if (acc + c[q] >= remaining) {
              s_prefix = prefix | ((uint32_t)(255 - 8 * tid - q) << shift);
              s_remaining = remaining - acc;
              break;
            }
            acc += c[q];
          }
        }
      }
      __syncthreads();
      prefix = s_prefix;
      remaining = s_remaining;
      mask |= 255u << shift;
      __syncthreads();
    }
    T = prefix;
    need = remaining;
  }

  // ---------------------------------------------------------------- compaction (ordered for ties)
  const int chunk = (n + kSortThreads - 1) / kSortThreads;
  const int lo = min(n, tid * chunk), up = min(n, lo + chunk);
  int gt = 0, eq = 0;
  if (k < n)
    for (int i = lo; i < up; ++i) { gt += hi[i] > T; eq += hi[i] == T; }
  int total_gt, total_eq;
  const int gt_base = block_exclusive_scan(gt, warp_tot, total_gt);
  const int eq_base = block_exclusive_scan(eq, warp_tot, total_eq);
  if (k < n) {
    int g = gt_base, e = eq_base;
    for (int i = lo; i < up; ++i) {
      const uint32_t h = hi[i];
      const uint64_t key = ((uint64_t)h << 32) | (uint64_t)(0xffffffffu - (uint32_t)i);
      if (h > T) sel[g++] = key;
      else if (h == T) {
        if (e < need) sel[total_gt + e] = key;
        ++e;
      }
    }
  } else {
    for (int i = lo; i < up; ++i)
      sel[i] = ((uint64_t)hi[i] << 32) | (uint64_t)(0xffffffffu - (uint32_t)i);
  }
  int P = 1;
  while (P < k) P <<= 1;
  for (int i = k + tid; i < P; i += kSortThreads) sel[i] = 0;
  __syncthreads();

  // ---------------------------------------------------------------- bitonic sort of the k keys, descending
  for (int kk = 2; kk <= P; kk <<= 1) {
    for (int j = kk >> 1; j > 0; j >>= 1) {
      for (int i = tid; i < P; i += kSortThreads) {
        const int ixj = i ^ j;
        if (ixj > i) {
          const uint64_t a = sel[i], b = sel[ixj];
          const bool desc = (i & kk) == 0;
          if (desc ? (a < b) : (a > b)) {
            sel[i] = b;
            sel[ixj] = a;
          }
        }
      }
      __syncthreads();
    }
  }
  int32_t* ord = p.order + (size_t)row * p.kmax;
  for (int t = tid; t < p.kmax; t += kSortThreads)
    ord[t] = t < k ? (int32_t)(0xffffffffu - (uint32_t)(sel[t] & 0xffffffffu)) : -1;
  if (tid == 0) {
    p.count[row] = k;
    if (p.hrm_count) p.hrm_count[row] = s_hrm;
  }
  // blocks no query of this Q-block can see: -inf score, no flag
  if (p.block_score)
    for (int j = n + tid; j < p.nkb; j += kSortThreads) p.block_score[(size_t)row * p.nkb + j] = -INFINITY;
  if (p.hrm_flags)
    for (int j = n + tid; j < p.nkb; j += kSortThreads) p.hrm_flags[(size_t)row * p.nkb + j] = 0;
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
  const size_t smem = (size_t)pmax * (sizeof(uint64_t) + sizeof(uint32_t));
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
