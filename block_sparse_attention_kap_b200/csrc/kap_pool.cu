// kap_pool: the downsampling step of the Kernel-Aware Proxy ("downsamples
// queries and keys", CoSA technical summary Sec. 2.2).  Pooled row r is the
// mean of tokens s*r .. s*r+s-1: an fp32 sum in token order, times 1/s,
// rounded to bf16 (nearest-even).  One HBM-bound pass over Q and K (the
// paged K cache is read in place through the page table) that writes the
// pooled tensors in the logical [B, H, N/s, d] layout.
#include <cuda_bf16.h>
#include "internal.h"

namespace cosa {

namespace {

__device__ __forceinline__ uint4 ld_stream(const uint16_t* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ void add_bf16x2(float& a, float& b, uint32_t w) {
  a = __fadd_rn(a, __uint_as_float(w << 16));
  b = __fadd_rn(b, __uint_as_float(w & 0xffff0000u));
}

template <int S>
__device__ __forceinline__ void pool_rows(const uint16_t* src, int s_rt, float (&acc)[8]) {
  if constexpr (S > 0) {
    uint4 v[S];
#pragma unroll
    for (int t = 0; t < S; ++t) v[t] = ld_stream(src + (size_t)t * kD);
#pragma unroll
    for (int t = 0; t < S; ++t) {
      add_bf16x2(acc[0], acc[1], v[t].x);
      add_bf16x2(acc[2], acc[3], v[t].y);
      add_bf16x2(acc[4], acc[5], v[t].z);
      add_bf16x2(acc[6], acc[7], v[t].w);
    }
  } else {
    for (int t = 0; t < s_rt; ++t) {
      uint4 v = ld_stream(src + (size_t)t * kD);
      add_bf16x2(acc[0], acc[1], v.x);
      add_bf16x2(acc[2], acc[3], v.y);
      add_bf16x2(acc[4], acc[5], v.z);
      add_bf16x2(acc[6], acc[7], v.w);
    }
  }
}

// 16 threads per pooled row, 8 bf16 columns (16 bytes) per thread.
template <int S>
__global__ void __launch_bounds__(256) kap_pool_kernel(PoolParams p) {
  const long long tid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long item = tid >> 4;
  const int part = (int)(tid & 15);
  if (item >= p.q_items + p.k_items) return;
  const int s = S > 0 ? S : p.s;
  const uint16_t* src;
  uint16_t* dst;
  if (item < p.q_items) {
    src = p.q + item * s * kD;   // pooled row item of head (b,h) starts at token item*s of the flat Q
    dst = p.qp + item * kD;
  } else {
    // K rows kp_first .. Nkv/s-1 of each (b, kv-head); rows below kp_first
    // were pooled by an earlier call (chunked prefill) and are not touched
    const int n_new = p.Nkv / s - p.kp_first;
    const long long it = item - p.q_items;
    const long long bg = it / n_new;
    const int c = p.kp_first + (int)(it - bg * n_new);
    dst = p.kp + (bg * p.kp_stride + c) * kD;
    if (!p.paged) {
      src = p.k + (bg * p.Nkv + (long long)c * s) * kD;
    } else {
      const int b = (int)(bg / p.Hkv), g = (int)(bg - (long long)b * p.Hkv);
      const int tok = c * s, j = tok / p.bk, w = tok - j * p.bk;
      int page = p.page_table[(size_t)b * p.nkb + j];
      page = page < 0 ? 0 : (page >= p.num_pages ? p.num_pages - 1 : page);   // never read outside the pool
      src = p.k + (((long long)page * p.Hkv + g) * p.bk + w) * kD;
    }
  }
  src += part * 8;
  dst += part * 8;
  float acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.0f;
  pool_rows<S>(src, s, acc);
  const float inv = 1.0f / (float)s;   // a power of two: exact
  uint32_t o[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    __nv_bfloat162 two = __halves2bfloat162(__float2bfloat16_rn(__fmul_rn(acc[2 * e], inv)),
                                            __float2bfloat16_rn(__fmul_rn(acc[2 * e + 1], inv)));
    o[e] = *reinterpret_cast<uint32_t*>(&two);
  }
  *reinterpret_cast<uint4*>(dst) = make_uint4(o[0], o[1], o[2], o[3]);
}

}  // namespace

cudaError_t launch_kap_pool(const PoolParams& p, cudaStream_t st) {
  const long long threads = (p.q_items + p.k_items) * 16;
  if (threads == 0) return cudaSuccess;
  const unsigned blocks = (unsigned)((threads + 255) / 256);
  if (p.s == 16) kap_pool_kernel<16><<<blocks, 256, 0, st>>>(p);
  else if (p.s == 8) kap_pool_kernel<8><<<blocks, 256, 0, st>>>(p);
  else kap_pool_kernel<0><<<blocks, 256, 0, st>>>(p);
  return cudaGetLastError();
}

}  // namespace cosa
