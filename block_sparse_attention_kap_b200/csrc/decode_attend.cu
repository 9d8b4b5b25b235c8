// decode_attend: the Ordered-Skipping Kernel for one decode step (a single
// query row per head), with the semantics of CoSA's OSK (technical summary
// Sec. 2.3) on that row: visit order[0..count-1]; skip a visit when
// fp32(m_loc - m_run) < T (the tile-wide vote of a one-row tile is the
// row's own test), else fold the block into the online softmax.  The pages
// leave decoding to future work (Sec. 4); this is the plainest single-row
// reading, the same one cosa_attend computes on Nq = 1.
//
// A decode step reads each visited K tile once and each computed V tile once
// and does ~2 flops per byte: it is bound by memory, not by the tensor
// cores, so it runs on the CUDA cores and is parallel over the visits rather
// than a chain of visits:
//  * the running max a visit is tested against equals the maximum of m_loc
//    over ALL earlier visits: with T <= 0 a skipped visit has
//    fp32(m_loc - m_run) < 0, i.e. m_loc < m_run, so it never raises m_run.
//    The decisions are therefore a prefix-max scan over the visits' m_loc;
//  * the softmax of the computed visits is taken against their common
//    maximum M (the last prefix max), so the computed visits' partial sums
//    need no rescaling and can be formed independently.
// decode_qk_kernel: one CTA per (row, 8 consecutive visits): the logits of
// each visited block (fp32, raw q.k) and its m_loc, into the workspace.
// decode_pv_kernel: one CTA per (row, 8 consecutive computed visits): the
// scan (redone by every CTA of the row, it is short), the skip bits, then
// P = exp((s - M)/sqrt(d)) and P.V of its visits, and a partial (sum P, P.V)
// per CTA; the last CTA of the row (a counter) adds the partials in a fixed
// order and writes out = O / l and lse.
#include <cuda_bf16.h>
#include "decode.h"

namespace cosa {

namespace {

constexpr int kThreads = 256;
constexpr int kQkVisits = 8;              // decode_qk: visits per CTA
constexpr int kVisitsPerCta = 8;          // decode_pv: computed visits per CTA
constexpr int kWarps = kThreads / 32;

__device__ __forceinline__ size_t kv_base(const DecodeAttendParams& p, int b, int g, int j, int bk) {
  if (!p.paged) return (((size_t)b * p.Hkv + g) * p.Nkv + (size_t)j * bk) * kD;
  int page = p.page_table[(size_t)b * p.nkb + j];
  page = page < 0 ? 0 : (page >= p.num_pages ? p.num_pages - 1 : page);   // never read outside the pool
  return (((size_t)page * p.Hkv + g) * bk) * kD;
}

__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// TPK threads per key, 128 / TPK dimensions each.
template <int BK>
__global__ void __launch_bounds__(kThreads) decode_qk_kernel(const DecodeAttendParams p) {
  constexpr int TPK = kThreads / BK;                  // 2 (BK = 128) or 4 (BK = 64)
  constexpr int DPT = kD / TPK;                       // dimensions per thread: 64 or 32
  constexpr int NV = DPT / 8;                         // 16-byte loads per thread
  __shared__ float wmax[kWarps];
  const int row = blockIdx.y;
  const int b = row / p.Hq, h = row % p.Hq, g = h / (p.Hq / p.Hkv);
  if (blockIdx.x == 0 && threadIdx.x == 0) p.counters[row] = 0u;     // for decode_pv's last-CTA count
  int n = p.count[row];
  n = n < 0 ? 0 : (n > p.kmax ? p.kmax : n);
  const int t0 = blockIdx.x * kQkVisits;
  if (t0 >= n) return;
  const int tid = threadIdx.x, key = tid / TPK, part = tid % TPK;
  // this thread's slice of the query, fp32
  float qv[DPT];
  {
    const uint4* qs = reinterpret_cast<const uint4*>(p.q + (size_t)row * kD + part * DPT);
#pragma unroll
    for (int i = 0; i < NV; ++i) {
      const uint4 w = qs[i];
      qv[8 * i + 0] = bf16lo(w.x); qv[8 * i + 1] = bf16hi(w.x);
      qv[8 * i + 2] = bf16lo(w.y); qv[8 * i + 3] = bf16hi(w.y);
      qv[8 * i + 4] = bf16lo(w.z); qv[8 * i + 5] = bf16hi(w.z);
      qv[8 * i + 6] = bf16lo(w.w); qv[8 * i + 7] = bf16hi(w.w);
    }
  }
  const int32_t* ord = p.order + (size_t)row * p.kmax;
  const int t1 = min(n, t0 + kQkVisits);
  for (int t = t0; t < t1; ++t) {
    const int j = ord[t];
    const bool valid = j >= 0 && j < p.nkb && j * BK + key < p.Nkv;   // keys past the cache are not read
    float acc = 0.0f;
    if (valid) {
      const uint4* kr = reinterpret_cast<const uint4*>(p.k + kv_base(p, b, g, j, BK) + (size_t)key * kD + part * DPT);
      uint4 w[NV];
#pragma unroll
      for (int i = 0; i < NV; ++i) w[i] = __ldg(kr + i);
#pragma unroll
      for (int i = 0; i < NV; ++i) {
        acc = fmaf(qv[8 * i + 0], bf16lo(w[i].x), acc); acc = fmaf(qv[8 * i + 1], bf16hi(w[i].x), acc);
        acc = fmaf(qv[8 * i + 2], bf16lo(w[i].y), acc); acc = fmaf(qv[8 * i + 3], bf16hi(w[i].y), acc);
        acc = fmaf(qv[8 * i + 4], bf16lo(w[i].z), acc); acc = fmaf(qv[8 * i + 5], bf16hi(w[i].z), acc);
        acc = fmaf(qv[8 * i + 6], bf16lo(w[i].w), acc); acc = fmaf(qv[8 * i + 7], bf16hi(w[i].w), acc);
      }
    }
    // the key's logit: the TPK partial sums (consecutive lanes), added in a fixed order
#pragma unroll
    for (int o = 1; o < TPK; o <<= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    const float s = valid ? acc : -INFINITY;
    if (part == 0) p.logits[((size_t)row * p.kmax + t) * BK + key] = s;
    float m = s;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if ((tid & 31) == 0) wmax[tid >> 5] = m;
    __syncthreads();
    if (tid == 0) {
      float mm = wmax[0];
#pragma unroll
      for (int w = 1; w < kWarps; ++w) mm = fmaxf(mm, wmax[w]);
      p.mloc[(size_t)row * p.kmax + t] = mm;          // -inf for an entry that is not a block
    }
    __syncthreads();
  }
}

// Dynamic shared memory of decode_pv: the computed-visit list and skip bitmap
// of the row, then per warp the P values of one visit, then the partials.
__host__ __device__ inline size_t pv_smem(int kmax, int bk) {
  return (size_t)kmax * 4 + (size_t)((kmax + 31) / 32) * 4 + (size_t)kWarps * bk * 4 + (size_t)kWarps * (kD + 1) * 4 +
         64;
}

template <int BK>
__global__ void __launch_bounds__(kThreads) decode_pv_kernel(const DecodeAttendParams p) {
  extern __shared__ __align__(16) uint8_t dyn[];
  __shared__ float s_M;
  __shared__ int s_nc, s_last;
  const int row = blockIdx.y;
  const int b = row / p.Hq, h = row % p.Hq, g = h / (p.Hq / p.Hkv);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  int n = p.count[row];
  n = n < 0 ? 0 : (n > p.kmax ? p.kmax : n);
  int* comp = reinterpret_cast<int*>(dyn);                                  // computed visits, in visit order
  uint32_t* skipw = reinterpret_cast<uint32_t*>(dyn + (size_t)p.kmax * 4);  // skip bit of every visit
  float* pbuf = reinterpret_cast<float*>(dyn + (size_t)p.kmax * 4 + (size_t)((p.kmax + 31) / 32) * 4);
  float* part = pbuf + kWarps * BK;                                          // [kWarps][d + 1]
  const int words = (n + 31) / 32;
  const float* mloc = p.mloc + (size_t)row * p.kmax;

  // ---------------------------------------------------------------- decisions (warp 0)
  if (warp == 0) {
    for (int w = lane; w < words; w += 32) skipw[w] = 0u;
    __syncwarp();
    const int seg = (n + 31) / 32;
    const int s0 = min(n, lane * seg), s1 = min(n, s0 + seg);
    float smax = -INFINITY;
    for (int t = s0; t < s1; ++t) smax = fmaxf(smax, __ldcg(mloc + t));
    // exclusive prefix max over the lanes' segments
    float incl = smax;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const float y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl = fmaxf(incl, y);
    }
    float pmax = __shfl_up_sync(0xffffffffu, incl, 1);
    if (lane == 0) pmax = -INFINITY;
    // each lane's decisions and computed count
    int nc = 0;
    for (int t = s0; t < s1; ++t) {
      const float ml = __ldcg(mloc + t);
      const bool skip = ml == -INFINITY || (pmax != -INFINITY && __fsub_rn(ml, pmax) < p.T);
      if (skip) atomicOr(&skipw[t >> 5], 1u << (t & 31));
      nc += !skip;
      pmax = fmaxf(pmax, ml);
    }
    int before = nc;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, before, o);
      if (lane >= o) before += y;
    }
    const int total = __shfl_sync(0xffffffffu, before, 31);
    before -= nc;
    __syncwarp();
    for (int t = s0; t < s1; ++t)
      if (!((skipw[t >> 5] >> (t & 31)) & 1u)) comp[before++] = t;
    if (lane == 31) {
      s_M = incl;                        // the maximum of every visit's m_loc
      s_nc = total;
    }
  }
  __syncthreads();
  const int nc = s_nc;
  const float M = s_M;
  const int producers = (nc + kVisitsPerCta - 1) / kVisitsPerCta;
  if (blockIdx.x == 0 && p.skip_bits) {
    uint32_t* sb = p.skip_bits + (size_t)row * p.skip_words;
    for (int w = tid; w < p.skip_words; w += kThreads) sb[w] = w < words ? skipw[w] : 0u;
  }
  uint16_t* orow = p.out + (size_t)row * kD;
  if (nc == 0) {                         // no block with a key: the row is 0, lse -inf
    if (blockIdx.x == 0) {
      if (tid < kD / 2) reinterpret_cast<uint32_t*>(orow)[tid] = 0u;
      if (tid == 0 && p.lse) p.lse[row] = -INFINITY;
    }
    return;
  }
  if ((int)blockIdx.x >= producers) return;

  // ---------------------------------------------------------------- P.V of this CTA's computed visits
  // P of visit v (the CTA's v-th computed visit) by warp v, into pbuf[v];
  // then warp w takes keys [w*BK/8, (w+1)*BK/8) of every visit, so a visit's
  // V tile is read by all eight warps at once
  constexpr int KPW = BK / kWarps;        // keys per warp: 16 or 8
  const int c0 = blockIdx.x * kVisitsPerCta;
  const int nv = min(kVisitsPerCta, nc - c0);
  __shared__ int s_j[kVisitsPerCta], s_nvalid[kVisitsPerCta];
  float l = 0.0f;
  if (warp < nv) {
    const int t = comp[c0 + warp];
    const int j = p.order[(size_t)row * p.kmax + t];   // a computed visit names a block
    const int nvalid = min(BK, p.Nkv - j * BK);
    const float* sv = p.logits + ((size_t)row * p.kmax + t) * BK;
    float* pw = pbuf + warp * BK;
#pragma unroll
    for (int i = 0; i < BK / 32; ++i) {
      const int kk = lane + 32 * i;
      const float x = kk < nvalid ? __ldcg(sv + kk) : -INFINITY;
      const float pr = exp2f((x - M) * p.scale_log2);
      pw[kk] = pr;
      l += pr;
    }
    if (lane == 0) { s_j[warp] = j; s_nvalid[warp] = nvalid; }
  }
  __syncthreads();
  float o[4] = {0.0f, 0.0f, 0.0f, 0.0f};  // dimensions 4*lane .. 4*lane+3, keys of this warp
#pragma unroll 2
  for (int v = 0; v < nv; ++v) {
    const int j = s_j[v], nvalid = s_nvalid[v];
    const float* pw = pbuf + v * BK;
    const uint2* vr = reinterpret_cast<const uint2*>(p.v + kv_base(p, b, g, j, BK)) + lane;
    uint2 w[KPW];
    // keys past the end of the cache are not read (their rows may hold anything)
#pragma unroll
    for (int u = 0; u < KPW; ++u) {
      const int kk = warp * KPW + u;
      w[u] = kk < nvalid ? __ldg(vr + (size_t)kk * (kD / 4)) : make_uint2(0u, 0u);
    }
#pragma unroll
    for (int u = 0; u < KPW; ++u) {
      const float pr = pw[warp * KPW + u];   // 0 past the end
      o[0] = fmaf(pr, bf16lo(w[u].x), o[0]); o[1] = fmaf(pr, bf16hi(w[u].x), o[1]);
      o[2] = fmaf(pr, bf16lo(w[u].y), o[2]); o[3] = fmaf(pr, bf16hi(w[u].y), o[3]);
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) l += __shfl_xor_sync(0xffffffffu, l, off);
  float* pr_w = part + warp * (kD + 1);
#pragma unroll
  for (int i = 0; i < 4; ++i) pr_w[4 * lane + i] = o[i];
  if (lane == 0) pr_w[kD] = l;
  __syncthreads();
  // this CTA's partial: the warps added in a fixed order
  float* gpart = p.partials + ((size_t)row * p.max_producers + blockIdx.x) * (kD + 1);
  if (tid <= kD) {
    float acc = 0.0f;
    for (int w = 0; w < kWarps; ++w) acc += part[w * (kD + 1) + tid];
    gpart[tid] = acc;
  }
  // the last producer of the row adds the partials in producer order
  __threadfence();
  __syncthreads();
  if (tid == 0) s_last = (atomicAdd(p.counters + row, 1u) + 1u == (uint32_t)producers);
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  __shared__ float fin[kD + 1];
  if (tid <= kD) {
    float acc = 0.0f;
    for (int x = 0; x < producers; ++x) acc += __ldcg(p.partials + ((size_t)row * p.max_producers + x) * (kD + 1) + tid);
    fin[tid] = acc;
  }
  __syncthreads();
  const float lsum = fin[kD];
  const float inv = 1.0f / lsum;
  if (tid < kD / 2) {
    __nv_bfloat162 two = __floats2bfloat162_rn(fin[2 * tid] * inv, fin[2 * tid + 1] * inv);
    reinterpret_cast<__nv_bfloat162*>(orow)[tid] = two;
  }
  if (tid == 0 && p.lse) p.lse[row] = M * p.scale_ln + logf(lsum);
}

template <int BK>
cudaError_t launch_bk(const DecodeAttendParams& p, cudaStream_t st) {
  const int rows = p.B * p.Hq;
  dim3 grid((unsigned)((p.kmax + kQkVisits - 1) / kQkVisits), (unsigned)rows);
  decode_qk_kernel<BK><<<grid, kThreads, 0, st>>>(p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const size_t smem = pv_smem(p.kmax, BK);
  if (smem > 48 * 1024) {
    e = cudaFuncSetAttribute(decode_pv_kernel<BK>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  grid.x = (unsigned)p.max_producers;
  decode_pv_kernel<BK><<<grid, kThreads, smem, st>>>(p);
  return cudaGetLastError();
}

}  // namespace

size_t decode_attend_workspace(int rows, int kmax, int bk) {
  const size_t producers = (size_t)(kmax + kVisitsPerCta - 1) / kVisitsPerCta;
  size_t off = 0;
  off += (size_t)rows * kmax * bk * 4;                  // logits
  off = (off + 255) & ~size_t(255);
  off += (size_t)rows * kmax * 4;                       // m_loc
  off = (off + 255) & ~size_t(255);
  off += (size_t)rows * producers * (kD + 1) * 4;       // partials
  off = (off + 255) & ~size_t(255);
  off += (size_t)rows * 4;                              // counters
  return (off + 255) & ~size_t(255);
}

size_t decode_attend_smem(int kmax, int bk) { return pv_smem(kmax, bk); }

cudaError_t launch_decode_attend(DecodeAttendParams p, uint8_t* ws, cudaStream_t st) {
  const int rows = p.B * p.Hq;
  if (rows == 0) return cudaSuccess;
  p.max_producers = (p.kmax + kVisitsPerCta - 1) / kVisitsPerCta;
  size_t off = 0;
  p.logits = reinterpret_cast<float*>(ws + off);
  off += (size_t)rows * p.kmax * p.bk * 4;
  off = (off + 255) & ~size_t(255);
  p.mloc = reinterpret_cast<float*>(ws + off);
  off += (size_t)rows * p.kmax * 4;
  off = (off + 255) & ~size_t(255);
  p.partials = reinterpret_cast<float*>(ws + off);
  off += (size_t)rows * p.max_producers * (kD + 1) * 4;
  off = (off + 255) & ~size_t(255);
  p.counters = reinterpret_cast<uint32_t*>(ws + off);
  if (p.bk == 128) return launch_bk<128>(p, st);
  if (p.bk == 64) return launch_bk<64>(p, st);
  return cudaErrorInvalidValue;
}

}  // namespace cosa
