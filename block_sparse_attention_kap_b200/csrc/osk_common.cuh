// Pieces shared by the two forms of the Ordered-Skipping Kernel (CoSA
// technical summary Sec. 2.3): osk_attention (one query head per CTA, its own
// visit order) and osk_group (two query heads of one GQA group per CTA, one
// shared visit order, each K/V tile loaded once for both).
//
// softmax_stream() is the per-visit work of the 256 softmax threads of one
// query head's 128-row Q tile: the row maxima of S = Q K^T, the tile-wide
// skip vote (m_loc = -inf, or m_run finite and fp32(m_loc - m_run) < T on
// every row: the bucket effect of Sec. 1), and on computed blocks the
// online-softmax update with P = exp(S - m) written back over S in TMEM as
// bf16, then the epilogue O / l.  Two threads per row: TMEM lane = row
// (warp % 4 picks the lane quarter), warp / 4 within the group picks the
// 64-column half.  fp32 subtraction is monotone, so the vote needs no
// exchange between the halves; they trade maxima only on computed blocks.
#pragma once
#include <cuda_bf16.h>
#include "internal.h"
#include "sm100.cuh"

namespace cosa {
namespace osk {

constexpr int kRowThreads = 256;                 // softmax threads of one Q tile
constexpr uint32_t kDecisionSkip = 1, kDecisionCompute = 2;
constexpr int kOrderCap = 1024;                  // order entries staged in shared memory

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Named barrier `id` over the kRowThreads threads of one Q tile, with an AND
// reduction of v.
__device__ __forceinline__ bool all_rows(bool v, uint32_t id) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred pi, po;\n\t"
      "setp.ne.u32 pi, %1, 0;\n\t"
      "bar.red.and.pred po, %2, 256, pi;\n\t"
      "selp.u32 %0, 1, 0, po;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)v), "r"(id)
      : "memory");
  return r != 0;
}

__device__ __forceinline__ float max3f(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}
__device__ __forceinline__ uint64_t pk2(float a, float b) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ void up2(uint64_t r, float& a, float& b) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(r));
}
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t add2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 t = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&t);
}

// First row of KV block j of kv-head g in the 2D [rows, 128] view of K / V
// (through the page table for a paged cache).
template <int BK>
__device__ __forceinline__ int kv_row(const OskParams& p, int b, int g, int j) {
  const int jc = j < 0 ? 0 : (j >= p.nkb ? p.nkb - 1 : j);
  if (!p.paged) return (b * p.Hkv + g) * p.Nkv + jc * BK;
  const int page = p.page_table[(size_t)b * p.nkb + jc];
  return (page * p.Hkv + g) * BK;   // out-of-pool pages land outside the tensor map: zero fill
}

// Zero the V rows [valid, 16 * ceil(valid / 16)) of a K/V slot (two
// 64-column chunks of `chunk` bytes, 128-byte rows): the rows of a ragged
// last block past the end of the cache that share a 16-key MMA step with
// real keys.  Their P is 0, but 0 * NaN is NaN inside the MMA, and those rows
// hold another head's keys, zero fill or whatever a page's tail holds.  The
// swizzle permutes 16-byte units within a row, so whole rows are zeroed.
// Returns the number of 16-key steps that hold real keys.
__device__ __forceinline__ int clear_v_tail(uint8_t* slot, uint32_t chunk, int valid) {
  const int ksteps = (valid + 15) >> 4;
  if (valid < 16 * ksteps) {
    const uint4 z = make_uint4(0u, 0u, 0u, 0u);
    for (int c = 0; c < 2; ++c)
      for (int r = valid; r < 16 * ksteps; ++r) {
        uint4* dst = reinterpret_cast<uint4*>(slot + c * chunk + r * 128);
#pragma unroll
        for (int u = 0; u < 8; ++u) dst[u] = z;
      }
    fence_proxy_async_smem();                   // visible to the tensor core's reads
  }
  return ksteps;
}

// Shared-memory exchange area of one Q tile's softmax threads.
struct RowShared {
  float mx[2][128];             // half-row maxima, traded on computed blocks
  float lx[2][128];             // half-row sums, traded once at the end
};

// The hand-offs between one Q tile's softmax threads and the issuing thread.
struct StreamSync {
  uint64_t* s_full;             // S of the current visit is in TMEM
  uint64_t* decided;            // the tile-wide decision is in *decision
  uint64_t* p_ready;            // P is in TMEM (or S was read, on a skipped visit)
  uint64_t* o_final;            // every MMA has completed
  uint32_t* decision;
  uint32_t vote_bar, xchg_bar;  // named barrier ids of this Q tile
};

// One Q tile's softmax threads over the whole visit list, then the epilogue.
// tid: 0..255 within the tile's threads; h: query head; row: index of
// (b, h, I) in skip_bits; order_at(t): block of visit t.
template <int BK, typename OrderAt>
__device__ __forceinline__ void softmax_stream(const OskParams& p, int tid, int b, int h, int I, size_t row, int n,
                                               const OrderAt& order_at, uint32_t tS, uint32_t tO,
                                               const StreamSync& ss, RowShared* xs, volatile uint32_t* abort) {
  const int warp = tid >> 5;
  const int quarter = warp & 3, half = warp >> 2;
  const int r = 32 * quarter + (tid & 31);
  const int rows_valid = min(p.bq, p.Nq - I * p.bq);
  const bool row_ok = r < rows_valid;
  const int qpos = (p.Nkv - p.Nq) + I * p.bq + r;
  const float sl2 = p.scale_log2;
  const float tau = 8.0f / sl2;          // refresh the exponent reference past a 2^8 growth
  const uint32_t lane_base = (uint32_t)(32 * quarter) << 16;
  constexpr int HC = BK / 2;              // S columns of this half: [c_base, c_base + HC)
  const int c_base = half * HC;
  float m_run = -INFINITY, m_scale = -INFINITY, l = 0.0f;   // l: this half's share of the row sum
  bool any_pv = false;
  uint32_t skip_word = 0;
  uint32_t* skip_out = p.skip_bits ? p.skip_bits + row * p.skip_words : nullptr;
  for (int t = 0; t < n; ++t) {
    const int j = order_at(t);
    const bool j_ok = j >= 0 && j < p.nkb;
    // after a failure every thread still runs the same barriers, without waiting
    const bool got = wait_or_abort(ss.s_full, t & 1, abort, p.status, DEV_TIMEOUT_MMA, p.wait_limit_ns);
    tc_fence_after();
    const int lim = min(qpos - j * BK, p.Nkv - 1 - j * BK);   // last visible column
    // pass 1: max over this half's visible columns (one 64-column TMEM load
    // at BK=128, 4 independent partial maxima)
    float mp[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) mp[i] = -INFINITY;
    if constexpr (HC == 64) {
      uint32_t v[64];
      tmem_ld_x64(tS + lane_base + c_base, v);
      if (lim >= c_base + 63) {
#pragma unroll
        for (int i = 0; i < 32; ++i) mp[i & 3] = max3f(mp[i & 3], __uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
      } else {
#pragma unroll
        for (int i = 0; i < 64; ++i) mp[i & 3] = fmaxf(mp[i & 3], c_base + i <= lim ? __uint_as_float(v[i]) : -INFINITY);
      }
    } else {
#pragma unroll 1
      for (int c0 = c_base; c0 < c_base + HC; c0 += 32) {
        uint32_t v[32];
        tmem_ld_x32(tS + lane_base + c0, v);
        if (lim >= c0 + 31) {
#pragma unroll
          for (int i = 0; i < 32; ++i) mp[i & 3] = fmaxf(mp[i & 3], __uint_as_float(v[i]));
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) mp[i & 3] = fmaxf(mp[i & 3], c0 + i <= lim ? __uint_as_float(v[i]) : -INFINITY);
        }
      }
    }
    const float m_half = fmaxf(fmaxf(mp[0], mp[1]), fmaxf(mp[2], mp[3]));
    const bool vote = !got || !row_ok || !j_ok || m_half == -INFINITY ||
                      (m_run != -INFINITY && __fsub_rn(m_half, m_run) < p.T);
    tc_fence_before();                  // S reads are ordered before the hand-off below
    const bool skip = all_rows(vote, ss.vote_bar);
    if (tid == 0) {
      *ss.decision = skip ? kDecisionSkip : kDecisionCompute;
      mbar_arrive(ss.decided);
      if (skip) skip_word |= 1u << (t & 31);
    }
    if (!skip) {
      xs->mx[half][r] = m_half;
      named_barrier(ss.xchg_bar, kRowThreads);
      const float m_loc = fmaxf(xs->mx[0][r], xs->mx[1][r]);
      m_run = fmaxf(m_run, m_loc);
      float alpha = 1.0f;
      if (m_loc != -INFINITY && (m_scale == -INFINITY || m_loc > m_scale + tau)) {
        alpha = (m_scale == -INFINITY) ? 0.0f : ex2((m_scale - m_loc) * sl2);
        m_scale = m_loc;
      }
      l *= alpha;
      // pass 2: P = exp2((S - m_scale) * log2(e)/sqrt(d)) over this half's
      // columns, re-read 32 at a time and written back as bf16 pairs into
      // TMEM columns [c_base, c_base + HC/2): inside this half's own S range
      // and behind its reads, so the other half's S is never overwritten
      const float msl = (m_scale == -INFINITY) ? 0.0f : m_scale * sl2;
      uint64_t ls2[2] = {0ull, 0ull};           // packed partial row sums
      const uint64_t sl2x2 = pk2(sl2, sl2), nmsl2 = pk2(-msl, -msl);
#pragma unroll 1
      for (int c0 = c_base; c0 < c_base + HC; c0 += 32) {
        uint32_t v[32];
        tmem_ld_x32(tS + lane_base + c0, v);
        if (lim < c0 + 31) {
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (c0 + i > lim) v[i] = __float_as_uint(-INFINITY);
        }
        uint32_t w[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          float x0, x1;
          up2(fma2(pk2(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1])), sl2x2, nmsl2), x0, x1);
          const float p0 = ex2(x0), p1 = ex2(x1);
          ls2[i & 1] = add2(ls2[i & 1], pk2(p0, p1));
          w[i] = pack_bf16(p0, p1);
        }
        tmem_st_x16_nowait(tS + lane_base + c_base + (c0 - c_base) / 2, w);
      }
      tmem_wait_st();                           // every P store of this half is in TMEM
      {
        float a0, a1, b0, b1;
        up2(ls2[0], a0, a1);
        up2(ls2[1], b0, b1);
        l += (a0 + b0) + (a1 + b1);
      }
      // rescale this half of O when the exponent reference moved
      if (any_pv && __any_sync(0xffffffffu, alpha != 1.0f)) {
#pragma unroll 1
        for (int c0 = 0; c0 < 64; c0 += 32) {
          uint32_t o[32];
          tmem_ld_x32(tO + lane_base + 64 * half + c0, o);
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
          tmem_st_x32(tO + lane_base + 64 * half + c0, o);
        }
      }
      any_pv = true;
    }
    tc_fence_before();
    mbar_arrive(ss.p_ready);
    if (tid == 0 && skip_out && ((t & 31) == 31 || t == n - 1)) {
      skip_out[t >> 5] = skip_word;
      skip_word = 0;
    }
  }
  if (tid == 0 && skip_out)
    for (int w = (n + 31) >> 5; w < p.skip_words; ++w) skip_out[w] = 0;
  // ------------------------------------------------------------ epilogue
  bool have_o = any_pv;
  if (n > 0) {
    if (!wait_or_abort(ss.o_final, 0, abort, p.status, DEV_TIMEOUT_MMA, p.wait_limit_ns)) have_o = false;
    tc_fence_after();
  }
  xs->lx[half][r] = l;
  named_barrier(ss.xchg_bar, kRowThreads);
  const float l_row = xs->lx[0][r] + xs->lx[1][r];
  const float inv_l = l_row > 0.0f ? 1.0f / l_row : 0.0f;
  uint16_t* orow = p.out + (((size_t)(b * p.Hq + h)) * p.Nq + (size_t)I * p.bq + r) * kD + 64 * half;
#pragma unroll 1
  for (int c0 = 0; c0 < 64; c0 += 32) {
    uint32_t o[32];
    if (have_o) {
      tmem_ld_x32(tO + lane_base + 64 * half + c0, o);
    } else {
#pragma unroll
      for (int i = 0; i < 32; ++i) o[i] = 0u;
    }
    uint32_t w[16];
#pragma unroll
    for (int i = 0; i < 16; ++i)
      w[i] = pack_bf16(__uint_as_float(o[2 * i]) * inv_l, __uint_as_float(o[2 * i + 1]) * inv_l);
    if (row_ok) {
      uint4* dst = reinterpret_cast<uint4*>(orow + c0);
#pragma unroll
      for (int i = 0; i < 4; ++i) dst[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
    }
  }
  if (row_ok && half == 0 && p.lse)
    p.lse[((size_t)(b * p.Hq + h)) * p.Nq + (size_t)I * p.bq + r] =
        l_row > 0.0f ? m_scale * p.scale_ln + logf(l_row) : -INFINITY;
}

}  // namespace osk
}  // namespace cosa
