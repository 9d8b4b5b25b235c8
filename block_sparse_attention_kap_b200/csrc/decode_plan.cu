// decode_plan: the Kernel-Aware Proxy for one decode step (CoSA technical
// summary Sec. 2.2 applied to a single query row; the pages leave decoding
// to future work, Sec. 4).  Each head's query -- one token at position
// Nkv-1, not pooled -- is scored against the pooled keys of its kv-head
// (the chunk cache that cosa_plan_chunk maintains; every pooled key is
// visible to the last position):
//   S[c]     = q . Kp[c]                       (fp32 sums of bf16 products)
//   Bs[j]    = max over the pooled keys c of block j    (MaxPool)
//   z[j]     = Bs[j] - max_j Bs[j]             (MaxNorm)
//   HRM      = the first block holding the maximum
// and the blocks are ordered HRM first, then by z, ties by block index, the
// first k = max(1, ceil(nKB * budget)) kept (warp_select_sort).
//
// One cluster of kCluster CTAs (8 warps each) per (b, h): CTA r of the
// cluster scores the r-th contiguous share of the blocks -- warp w its
// blocks w, w+8, ...: eight lanes per pooled key (16 bf16 dimensions each,
// two 16-byte loads), four keys per step, a three-step shuffle sum, a
// running max per block -- and stores each block score straight into the
// shared memory of CTA 0 of the cluster (distributed shared memory).  After
// a cluster barrier CTA 0 alone holds every block score: a CTA-wide arg-max,
// the keys, and one warp's select-and-sort follow.  Splitting the scoring
// over the cluster puts eight times as many warps on the pooled-key reads,
// which are latency-bound at one CTA per head.
#include "kap_select.cuh"
#include "decode.h"

namespace cosa {

namespace {

constexpr int kWarps = 8;
constexpr int kCluster = 8;                   // CTAs per (b, h)

// Store v at the same shared-memory offset as `local` in CTA `rank` of the cluster.
__device__ __forceinline__ void st_cluster_f32(const float* local, uint32_t rank, float v) {
  uint32_t remote;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote)
               : "r"(static_cast<uint32_t>(__cvta_generic_to_shared(local))), "r"(rank));
  asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(remote), "f"(v) : "memory");
}
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

__global__ void __cluster_dims__(kCluster, 1, 1) __launch_bounds__(32 * kWarps) decode_plan_kernel(DecodePlanParams p) {
  extern __shared__ __align__(16) uint8_t dyn[];
  float* bs = reinterpret_cast<float*>(dyn);                               // [nkb] block scores, then keys
  int* hist = reinterpret_cast<int*>(dyn + align16((size_t)p.nkb * 4));
  uint64_t* sel = reinterpret_cast<uint64_t*>(dyn + align16((size_t)p.nkb * 4) + 1024);
  __shared__ float red_m[kWarps];
  __shared__ int red_j[kWarps];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int hb = blockIdx.x / kCluster;                                   // b * Hq + h
  const uint32_t rank = cluster_rank();
  const int per = (p.nkb + kCluster - 1) / kCluster;                       // this CTA's blocks: [j0, j1)
  const int j0 = min(p.nkb, (int)rank * per), j1 = min(p.nkb, j0 + per);
  const int b = hb / p.Hq, h = hb - b * p.Hq;
  const int g = h / (p.Hq / p.Hkv);
  const int grp = lane >> 3, part = lane & 7;                              // key within the step, 16-dim slice

  // this lane's 16 query dimensions
  const uint4* qv = reinterpret_cast<const uint4*>(p.q + (size_t)hb * kD + part * 16);
  const uint4 q0 = qv[0], q1 = qv[1];
  float qf[16];
  {
    const uint32_t w[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) { qf[2 * i] = bf16_lo(w[i]); qf[2 * i + 1] = bf16_hi(w[i]); }
  }
  const uint16_t* kp = p.kp + ((size_t)b * p.Hkv + g) * (size_t)p.kp_stride * kD;
  cluster_sync();                     // every CTA of the cluster runs before any remote store
  for (int j = j0 + warp; j < j1; j += kWarps) {
    float m = -INFINITY;
    const int c0 = j * p.kpb, c1 = min(c0 + p.kpb, p.nkp);
    const int steps = (c1 - c0 + 3) / 4;                                // every lane runs every step
    for (int st = 0; st < steps; ++st) {
      const int c = c0 + 4 * st + grp;
      float acc = 0.0f;
      if (c < c1) {
        const uint4* kr = reinterpret_cast<const uint4*>(kp + (size_t)c * kD + part * 16);
        const uint4 k0 = __ldg(kr), k1 = __ldg(kr + 1);
        const uint32_t w[8] = {k0.x, k0.y, k0.z, k0.w, k1.x, k1.y, k1.z, k1.w};
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          acc = fmaf(qf[2 * i], bf16_lo(w[i]), acc);
          acc = fmaf(qf[2 * i + 1], bf16_hi(w[i]), acc);
        }
      }
#pragma unroll
      for (int o = 1; o < 8; o <<= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
      if (c < c1) m = fmaxf(m, acc);
    }
#pragma unroll
    for (int o = 8; o < 32; o <<= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (lane == 0) st_cluster_f32(bs + j, 0u, m);                          // into CTA 0's block scores
  }
  cluster_sync();                                                          // every score is in CTA 0
  if (rank != 0) return;

  // CTA-wide maximum and the first block attaining it
  float m = -INFINITY;
  int jm = 0x7fffffff;
  for (int j = threadIdx.x; j < p.nkb; j += blockDim.x)
    if (bs[j] > m) { m = bs[j]; jm = j; }                                  // ascending j: first wins
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float mo = __shfl_xor_sync(0xffffffffu, m, o);
    const int jo = __shfl_xor_sync(0xffffffffu, jm, o);
    if (mo > m || (mo == m && jo < jm)) { m = mo; jm = jo; }
  }
  if (lane == 0) { red_m[warp] = m; red_j[warp] = jm; }
  __syncthreads();
  float rowmax = red_m[0];
  int jstar = red_j[0];
  for (int w = 1; w < kWarps; ++w)
    if (red_m[w] > rowmax || (red_m[w] == rowmax && red_j[w] < jstar)) { rowmax = red_m[w]; jstar = red_j[w]; }

  // MaxNorm + HRM -> order-preserving ranking keys (in place)
  const size_t out_row = (size_t)hb * p.nkb;
  uint32_t* hi = reinterpret_cast<uint32_t*>(bs);
  for (int j = threadIdx.x; j < p.nkb; j += blockDim.x) {
    const float v = bs[j];
    const float z = v != -INFINITY ? __fsub_rn(v, rowmax) : -INFINITY;
    const bool flag = j == jstar;
    if (p.block_score) p.block_score[out_row + j] = z;
    if (p.hrm_flags) p.hrm_flags[out_row + j] = (uint8_t)flag;
    hi[j] = orderable(flag ? 1.0f : z);
  }
  __syncthreads();
  if (warp == 0) {
    warp_select_sort(hi, p.nkb, p.k, hist, sel, p.order + (size_t)hb * p.kmax, p.kmax, lane);
    if (lane == 0) {
      p.count[hb] = p.k;
      if (p.hrm_count) p.hrm_count[hb] = jstar < p.nkb ? 1 : 0;
    }
  }
}

}  // namespace

size_t decode_plan_smem(int nkb, int k) {
  int pk = 1;
  while (pk < k) pk <<= 1;
  return align16((size_t)nkb * 4) + 1024 + (size_t)pk * 8;
}

cudaError_t launch_decode_plan(const DecodePlanParams& p, cudaStream_t st) {
  const int rows = p.B * p.Hq;
  if (rows == 0) return cudaSuccess;
  const size_t smem = decode_plan_smem(p.nkb, p.k);
  if (smem > 227 * 1024) return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(decode_plan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  decode_plan_kernel<<<rows * kCluster, 32 * kWarps, smem, st>>>(p);
  return cudaGetLastError();
}

}  // namespace cosa
