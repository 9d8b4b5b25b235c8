// Warp-level selection of the k largest ranking keys and their sort, shared
// by the prefill (kap_sort) and decode (decode_plan) proxies: the
// flag-grouped order of the CoSA technical summary, Sec. 2.2, once every
// block carries one order-preserving 32-bit key (HRM blocks above all
// others, then the score), ties resolved to the smaller block index.
//
// A 4-pass, 8-bit radix select (warp-private shared-memory histogram) finds
// the k-th largest key T; the keys above T plus the lowest-indexed keys equal
// to T are compacted in index order with warp ballots, and only those k --
// packed with the inverted index so ties resolve to the smaller index -- are
// sorted by a bitonic network in shared memory.  One warp, __syncwarp only.
#pragma once
#include "internal.h"

namespace cosa {

__device__ __forceinline__ uint32_t orderable(float f) {
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__host__ __device__ __forceinline__ size_t align16(size_t x) { return (x + 15) & ~size_t(15); }

// Per-warp shared memory: a 256-bin histogram, n keys, P >= k selected keys.
__host__ __device__ __forceinline__ size_t select_smem(int n, int pk) {
  return 1024 + align16((size_t)n * 4) + (size_t)pk * 8;
}

// hi[0..n): keys (read only); hist: 256 ints; sel: pow2(k) 64-bit slots.
// Writes ord[0..kmax): the k selected indices in order, then -1.
__device__ __forceinline__ void warp_select_sort(const uint32_t* hi, int n, int k, int* hist, uint64_t* sel,
                                                 int32_t* ord, int kmax, int lane) {
  const unsigned full = 0xffffffffu;
  const unsigned lt_mask = (1u << lane) - 1u;
  // ------------------------------------------------------------ radix select of the k-th largest
  uint32_t T = 0;
  int need = k;
  if (k < n) {
    uint32_t prefix = 0, mask = 0;
    int remaining = k;
    for (int shift = 24; shift >= 0; shift -= 8) {
      for (int b = lane; b < 256; b += 32) hist[b] = 0;
      __syncwarp();
      for (int i = lane; i < n; i += 32) {
        const uint32_t h = hi[i];
        if ((h & mask) == prefix) atomicAdd(&hist[(h >> shift) & 255u], 1);
      }
      __syncwarp();
      // lane l owns digits 255-8l .. 248-8l (descending); counts from the top digit
      int c[8], tot = 0;
#pragma unroll
      for (int q = 0; q < 8; ++q) { c[q] = hist[255 - 8 * lane - q]; tot += c[q]; }
      int incl = tot;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(full, incl, o);
        if (lane >= o) incl += y;
      }
      const int excl = incl - tot;
      const bool here = excl < remaining && remaining <= incl;
      uint32_t digit = 0;
      int rem_here = 0;
      if (here) {
        int acc = excl;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          if (acc + c[q] >= remaining) { digit = 255 - 8 * lane - q; rem_here = remaining - acc; break; }
          acc += c[q];
        }
      }
      const int src = __ffs(__ballot_sync(full, here)) - 1;
      digit = __shfl_sync(full, digit, src);
      remaining = __shfl_sync(full, rem_here, src);
      prefix |= digit << shift;
      mask |= 255u << shift;
      __syncwarp();
    }
    T = prefix;
    need = remaining;
  }

  // ------------------------------------------------------------ compaction in index order
  const int total_gt = k - need;
  int g = 0, e = 0;
  for (int base = 0; base < n; base += 32) {
    const int i = base + lane;
    const uint32_t h = i < n ? hi[i] : 0u;
    const uint64_t key = ((uint64_t)h << 32) | (uint64_t)(0xffffffffu - (uint32_t)i);
    if (k == n) {
      if (i < n) sel[i] = key;
      continue;
    }
    const bool gt = i < n && h > T, eq = i < n && h == T;
    const unsigned bg = __ballot_sync(full, gt), be = __ballot_sync(full, eq);
    if (gt) sel[g + __popc(bg & lt_mask)] = key;
    if (eq) {
      const int r = e + __popc(be & lt_mask);
      if (r < need) sel[total_gt + r] = key;
    }
    g += __popc(bg);
    e += __popc(be);
  }
  int P = 1;
  while (P < k) P <<= 1;
  for (int i = k + lane; i < P; i += 32) sel[i] = 0;
  __syncwarp();

  // ------------------------------------------------------------ bitonic sort of the k keys, descending
  for (int kk = 2; kk <= P; kk <<= 1) {
    for (int j = kk >> 1; j > 0; j >>= 1) {
      for (int i = lane; i < P; i += 32) {
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
      __syncwarp();
    }
  }
  for (int t = lane; t < kmax; t += 32)
    ord[t] = t < k ? (int32_t)(0xffffffffu - (uint32_t)(sel[t] & 0xffffffffu)) : -1;
}

}  // namespace cosa
