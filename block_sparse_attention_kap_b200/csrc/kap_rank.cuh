// The ranking and flag-grouped sorting of the Kernel-Aware Proxy for one
// (b, h, Q-block) (CoSA technical summary Sec. 2.2, "Block Ranking", "HRM
// Flag Generation" and the sort), run by one warp: from the max-pooled block
// scores Bs of the Q-block's pooled rows (kap_score),
//   rowmax[r]  = max_j Bs[r, j]; HRM block of r = first j attaining it
//   score[j]   = max over the Q-block's rows r of (Bs[r, j] - rowmax[r])
// (MaxNorm, then the aggregate), and the causally visible blocks are ordered
// HRM blocks first, then by score, ties by block index; the first
// k_I = max(1, ceil(n_I * budget)) form the computation-order mask M_KAP.
// Every value is fp32 and every decision is taken on fp32 values.  The row
// maxima come from kap_score's per-item partial maxima (ties resolved to the
// smaller block index).  Each block's ranking key (+1 for HRM blocks, else
// its score <= 0) is mapped to an order-preserving 32-bit integer, and
// warp_select_sort (kap_select.cuh) emits the order.  Used by kap_sort, one
// warp per (b, h, Q-block); Bs and the partial maxima come from the
// preceding kap_score launch and are read through the read-only path.
#pragma once
#include "kap_select.cuh"

namespace cosa {

__device__ __forceinline__ int kap_causal_blocks(int I, int Nq, int Nkv, int bq, int bk, int nkb) {
  const int last_tok = min((I + 1) * bq, Nq) - 1;
  return min(nkb, (Nkv - Nq + last_tok) / bk + 1);
}

// row = (b * Hq + h) * nQB + I; mine: this warp's select_smem(nkb, pk) bytes
// of shared memory (16-byte aligned).
template <int RPQ>
__device__ __forceinline__ void rank_qblock(const SortParams& p, int row, int pk, uint8_t* mine, int lane) {
  int* hist = reinterpret_cast<int*>(mine);
  uint32_t* hi = reinterpret_cast<uint32_t*>(mine + 1024);
  uint64_t* sel = reinterpret_cast<uint64_t*>(mine + 1024 + align16((size_t)p.nkb * 4));
  const unsigned full = 0xffffffffu;
  const int I = row % p.nqb;
  const int hb = row / p.nqb;                    // b * Hq + h
  const int n = kap_causal_blocks(I, p.Nq, p.Nkv, p.bq, p.bk, p.nkb);
  int k = (int)(((long long)n * p.bp + 9999) / 10000);
  k = max(1, min(k, n));

  // ------------------------------------------------------------ row maxima of the Q-block's pooled rows
  const int r_abs0 = I * RPQ;                    // first pooled row (a Q-block never straddles row tiles)
  const int R = r_abs0 / kTileRows, row0 = r_abs0 % kTileRows;
  float my_max = -INFINITY;
  int my_arg = -1;
  if (lane < RPQ) {
    const size_t base = ((size_t)hb * p.n_row_tiles + R) * p.splits * 2 * kTileRows + row0 + lane;
    for (int q = 0; q < 2 * p.splits; ++q) {
      const float m = __ldg(p.part_max + base + (size_t)q * kTileRows);
      const int a = __ldg(p.part_arg + base + (size_t)q * kTileRows);
      if (m > my_max || (m == my_max && a >= 0 && (my_arg < 0 || a < my_arg))) { my_max = m; my_arg = a; }
    }
  }
  float rmax[RPQ];
  int rarg[RPQ];
#pragma unroll
  for (int i = 0; i < RPQ; ++i) {
    rmax[i] = __shfl_sync(full, my_max, i);
    rarg[i] = __shfl_sync(full, my_arg, i);
  }

  // ------------------------------------------------------------ MaxNorm, aggregate, HRM -> ranking keys
  const float* bs = p.bs + ((size_t)hb * p.n_row_tiles + R) * p.nkb * kTileRows + (size_t)(row0 / RPQ) * p.nkb * RPQ;
  const size_t out_row = (size_t)row * p.nkb;
  const uint32_t hrm_key = orderable(1.0f);
  int hrm = 0;
  for (int j = lane; j < n; j += 32) {
    float v[RPQ];
    const float* src = bs + (size_t)j * RPQ;
    if constexpr (RPQ % 4 == 0) {
#pragma unroll
      for (int i = 0; i < RPQ; i += 4) {
        const float4 f = __ldg(reinterpret_cast<const float4*>(src + i));
        v[i] = f.x; v[i + 1] = f.y; v[i + 2] = f.z; v[i + 3] = f.w;
      }
    } else {
#pragma unroll
      for (int i = 0; i < RPQ; ++i) v[i] = __ldg(src + i);
    }
    float z = -INFINITY;
    bool flag = false;
#pragma unroll
    for (int i = 0; i < RPQ; ++i) {
      if (v[i] != -INFINITY) z = fmaxf(z, __fsub_rn(v[i], rmax[i]));
      flag |= rarg[i] == j;
    }
    const uint32_t h = flag ? hrm_key : orderable(z);
    hi[j] = h;
    hrm += flag;
    if (p.block_score) p.block_score[out_row + j] = z;
    if (p.hrm_flags) p.hrm_flags[out_row + j] = (uint8_t)flag;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) hrm += __shfl_xor_sync(full, hrm, o);
  __syncwarp();

  warp_select_sort(hi, n, k, hist, sel, p.order + (size_t)row * p.kmax, p.kmax, lane);
  if (lane == 0) {
    p.count[row] = k;
    if (p.hrm_count) p.hrm_count[row] = hrm;
  }
  // blocks no query of this Q-block can see: -inf score, no flag
  if (p.block_score)
    for (int j = n + lane; j < p.nkb; j += 32) p.block_score[(size_t)row * p.nkb + j] = -INFINITY;
  if (p.hrm_flags)
    for (int j = n + lane; j < p.nkb; j += 32) p.hrm_flags[(size_t)row * p.nkb + j] = 0;
}

}  // namespace cosa
