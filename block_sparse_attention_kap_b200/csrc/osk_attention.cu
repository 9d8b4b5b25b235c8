// osk_attention: the Ordered-Skipping Kernel of CoSA (technical summary
// Sec. 2.3), consuming the computation-order mask M_KAP.
//
// One CTA per (batch, query head, Q-block).  It visits only the KV blocks
// order[0..count-1], in that order ("mask-skipped" blocks are never touched:
// their tiles are simply never addressed, paged caches are read in place
// through the page table).  Per visited block:
//   S = Q K^T          tcgen05 MMA, bf16 x bf16 -> fp32 accumulator in TMEM
//   m_loc[r]           row max over causally visible keys
//   skip vote          m_loc = -inf, or m_run finite and m_loc - m_run < T
//   block skipped      iff all rows vote skip (tile-wide: the "bucket
//                      effect" of Sec. 1); a skipped block costs QK only
//   otherwise          online-softmax update (Sec. 2.1), P = exp(...) in
//                      bf16 written back into TMEM over S, O += P V with P
//                      read from TMEM and V from shared memory.
// m_run is the exact running row max over the computed blocks (it drives
// the skip test); the exponent reference m_scale is refreshed only when the
// max grows by more than 2^8 in probability terms, so O in TMEM is rarely
// rescaled.  The result O / l is written as bf16.
//
// Roles: warp 8 (one elected thread) issues every TMA load and MMA; warps
// 0-7 run the softmax, two threads per query row (TMEM lane = row, warp%4
// picks the lane quarter, warp/4 the column half).  The skip vote needs no
// exchange between the halves: fp32 subtraction is monotone, so
// fp32(m_loc - m_run) < T holds iff it holds for both half maxima; the
// halves trade maxima only on computed blocks.  TMEM: S/P at columns
// [0, BK), O at [128, 256); 256 columns and ~104 KB of shared memory per
// CTA, so two CTAs share an SM and one CTA's softmax overlaps the other's
// tensor-core work.
// Each CTA is one dependency chain per visit -- QK, the max and the vote,
// the exponentials, PV, the next QK (S and P share TMEM columns) -- and no
// single pipe is saturated: the chain's latency sets the pace, and the
// second CTA on the SM fills part of it.  Pass 1 takes maxima three at a
// time and pass 2 forms the exponent arguments and row sums with packed
// f32x2 arithmetic and stores P without waiting per store, to shorten the
// softmax's share of the chain.
#include "osk_common.cuh"

namespace cosa {

namespace {

using namespace osk;

constexpr int kSoftmaxThreads = kRowThreads;               // 8 warps, two threads per row
constexpr int kThreads = kSoftmaxThreads + 32;
constexpr int kCtrl = kSoftmaxThreads;                     // the control thread (warp 8, lane 0)
constexpr uint32_t kQBytes = 128 * 256;

struct __align__(8) OskSmem {
  uint64_t q_full, full[2], s_full, decided, p_ready, o_final;
  uint64_t never;               // nothing ever arrives here (the wait-timeout test hook waits on it)
  uint32_t decision;
  uint32_t tmem_base;
  uint32_t abort;               // set once any wait of this CTA gave up
  int32_t order[kOrderCap];     // this CTA's visit order (first kOrderCap entries)
  RowShared xs;
};

template <int BK>
struct OskCfg {
  static constexpr uint32_t kKVBytes = BK * 256;           // BK rows x 128 bf16
  static constexpr uint32_t kChunk = BK * 128;             // one 64-column chunk
  // tiles, the control block, and up to 1023 bytes lost aligning the base to 1 KB
  static constexpr int kSmem = kQBytes + 2 * kKVBytes + (int)sizeof(OskSmem) + 1024;
  static_assert(2 * (kSmem + 1024) <= 228 * 1024, "two CTAs must share an SM");
};

// Two CTAs per SM: 18 warps, so one SM sub-partition holds 5 warps and the
// kernel must fit in 16K / 5 / 32 = 102 registers per thread.
template <int BK>
__global__ void __launch_bounds__(kThreads, 2)
osk_attention_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, const OskParams p) {
  using Cfg = OskCfg<BK>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = base;
  uint8_t* sK = base + kQBytes;
  uint8_t* sV = sK + Cfg::kKVBytes;
  OskSmem* sm = reinterpret_cast<OskSmem*>(sV + Cfg::kKVBytes);
  volatile uint32_t* abort = &sm->abort;

  const int failed = p.status ? (int)*reinterpret_cast<volatile uint32_t*>(p.status) : 0;
  if (__syncthreads_or(failed)) return;

  const int tid = threadIdx.x, warp = tid >> 5;
  // One kv-head (and batch) at a time, heaviest (last) Q-blocks first, the G
  // query heads of the kv-head adjacent: the CTAs resident together then
  // serve a few dozen consecutive Q-blocks of one kv-head, whose selections
  // share most K/V tiles, so the tiles they read stay in L2 (4% faster than
  // all kv-heads of a few Q-blocks at a time at 128K, budget 10%)
  int x = blockIdx.x;
  const int hg = x % p.G; x /= p.G;
  const int I = p.nqb - 1 - x % p.nqb; x /= p.nqb;
  const int g = x % p.Hkv; x /= p.Hkv;
  const int b = x;
  const int h = g * p.G + hg;
  const size_t row = ((size_t)(b * p.Hq + h)) * p.nqb + I;
  const int32_t* ord = p.order + row * p.kmax;
  int n = p.count[row];
  n = n < 0 ? 0 : (n > p.kmax ? p.kmax : n);

  for (int t = tid; t < n && t < kOrderCap; t += kThreads) sm->order[t] = ord[t];
  auto order_at = [&](int t) -> int { return t < kOrderCap ? sm->order[t] : ord[t]; };
  if (warp == kCtrl / 32) {
    tmem_alloc(&sm->tmem_base, 256);
    tmem_relinquish();
  }
  if (tid == kCtrl) {
    mbar_init(&sm->q_full, 1);
    mbar_init(&sm->full[0], 1);
    mbar_init(&sm->full[1], 1);
    mbar_init(&sm->s_full, 1);
    mbar_init(&sm->decided, 1);
    mbar_init(&sm->p_ready, kSoftmaxThreads);
    mbar_init(&sm->o_final, 1);
    mbar_init(&sm->never, 1);
    sm->abort = 0;
    fence_mbar_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm->tmem_base;
  const uint32_t tS = tmem, tO = tmem + 128;

  if (tid == kCtrl) {
    // ------------------------------------------------------------ control thread
    if (n > 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      const int q_y = (b * p.Hq + h) * p.Nq + I * p.bq;
      const uint32_t id_qk = idesc_bf16(128, BK, false, false);
      const uint32_t id_pv = idesc_bf16(128, 128, false, true);
      const uint32_t q_addr = smem_u32(sQ), k_addr = smem_u32(sK), v_addr = smem_u32(sV);
      // Two 32 KB buffers ("slots") for K and V tiles.  K of the next visit is
      // always in flight in the free slot, so a skipped block never waits for
      // its successor's K; V of a visit is fetched only once the tile-wide vote
      // says the block is computed, into the slot its K has just vacated,
      // while the softmax warps are still exponentiating.
      auto slot = [&](int sl) { return sl ? sV : sK; };
      auto slot_addr = [&](int sl) { return sl ? v_addr : k_addr; };
      uint32_t fph = 0u;     // bit sl: parity of the next completion to wait for on slot sl
      uint32_t busy = 0u;    // bit sl: a load into slot sl was issued and not yet seen complete
      // K/V tiles are read again soon by the other heads of the group and by
      // neighbouring Q-blocks: keep them in L2; each Q tile is read once
      const uint64_t pol_kv = l2_evict_last(), pol_q = l2_evict_first();
      auto load = [&](int sl, const CUtensorMap* tm, int j) {
        const int y = kv_row<BK>(p, b, g, j);
        busy |= 1u << sl;
        mbar_arrive_expect_tx(&sm->full[sl], Cfg::kKVBytes);
        tma_load_2d_hint(slot(sl), tm, &sm->full[sl], 0, y, pol_kv);
        tma_load_2d_hint(slot(sl) + Cfg::kChunk, tm, &sm->full[sl], 64, y, pol_kv);
      };
      auto wait_slot = [&](int sl) {
        const bool r = wait_or_abort(&sm->full[sl], (fph >> sl) & 1u, abort, p.status, DEV_TIMEOUT_TMA, p.wait_limit_ns);
        if (r) {
          fph ^= 1u << sl;
          busy &= ~(1u << sl);
        }
        return r;
      };
      auto issue_qk = [&](int sl) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ss(tS, desc_sw128(q_addr + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024),
                 desc_sw128(slot_addr(sl) + (kk >> 2) * Cfg::kChunk + (kk & 3) * 32, 16, 1024), id_qk, kk > 0);
        tc_commit(&sm->s_full);
      };
      mbar_arrive_expect_tx(&sm->q_full, kQBytes);
      tma_load_2d_hint(sQ, &tm_q, &sm->q_full, 0, q_y, pol_q);
      tma_load_2d_hint(sQ + 16384, &tm_q, &sm->q_full, 64, q_y, pol_q);
      load(0, &tm_k, order_at(0));
      if (n > 1) load(1, &tm_k, order_at(1));
      bool any_pv = false;
      const bool q_seen = wait_or_abort(&sm->q_full, 0, abort, p.status, DEV_TIMEOUT_TMA, p.wait_limit_ns);
      bool ok = q_seen && wait_slot(0);
      // failure-detection test hook: a wait that cannot complete, so the
      // bounded wait gives up and every thread takes the abort path
      if (ok && p.stall_test) ok = wait_or_abort(&sm->never, 0, abort, p.status, DEV_TIMEOUT_PIPE, p.wait_limit_ns);
      if (ok) { tc_fence_after(); issue_qk(0); }
      int ks = 0;            // slot holding K of visit t
      int pend_k = -1;       // K load deferred until the PV reading its slot has completed
      for (int t = 0; ok && t < n; ++t) {
        const uint32_t ph = t & 1;
        const int ns = ks ^ 1;
        if (!wait_or_abort(&sm->s_full, ph, abort, p.status, DEV_TIMEOUT_MMA, p.wait_limit_ns)) break;
        // QK_t and every earlier MMA are complete
        if (pend_k >= 0) { load(ns, &tm_k, order_at(pend_k)); pend_k = -1; }
        if (!wait_or_abort(&sm->decided, ph, abort, p.status, DEV_TIMEOUT_PIPE, p.wait_limit_ns)) break;
        const uint32_t dec = *reinterpret_cast<volatile uint32_t*>(&sm->decision);
        if (dec == kDecisionCompute) {
          const int jv = order_at(t);
          load(ks, &tm_v, jv);
          if (!wait_or_abort(&sm->p_ready, ph, abort, p.status, DEV_TIMEOUT_PIPE, p.wait_limit_ns)) break;
          if (!wait_slot(ks)) break;
          // a ragged last block: no MMA step past the end of the cache, and the
          // non-key rows of the last step zeroed (see clear_v_tail)
          int ksteps = BK / 16;
          if (p.kv_tail && jv == p.nkb - 1) ksteps = clear_v_tail(slot(ks), Cfg::kChunk, p.kv_tail);
          tc_fence_after();
          // P of keys [16kk, 16kk+16): each column half packs its P at the
          // start of its own S range (TMEM columns half*BK/2 + ...)
          auto pv_step = [&](int kk) {
            mma_ts(tO, tS + (kk / (BK / 32)) * (BK / 2) + (kk % (BK / 32)) * 8,
                   desc_sw128(slot_addr(ks) + kk * 2048, Cfg::kChunk, 1024), id_pv, (any_pv || kk > 0) ? 1u : 0u);
          };
          if (ksteps == BK / 16) {
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk) pv_step(kk);
          } else {
            for (int kk = 0; kk < ksteps; ++kk) pv_step(kk);
          }
          any_pv = true;
          if (t + 2 < n) pend_k = t + 2;
        }
        // a skipped block's S was fully read before the vote: the next QK may
        // overwrite it at once (p_ready of this visit completes before the
        // next vote, so its phase parity stays in step); its slot then takes
        // K of visit t + 2, issued after that QK so the QK is not delayed
        if (t + 1 < n) {
          if (!wait_slot(ns)) break;
          tc_fence_after();
          issue_qk(ns);
        }
        if (dec != kDecisionCompute && t + 2 < n) load(ks, &tm_k, order_at(t + 2));
        ks = ns;

      }
      // o_final completes once every MMA issued above has; TMEM is released after it
      tc_commit(&sm->o_final);
      mbar_wait(&sm->o_final, 0);
      // no copy may still be writing shared memory when the CTA exits: after a
      // failed wait, wait again (bounded) for the loads not yet seen complete
      // (a slot holds at most one outstanding load; none on the normal path)
      if (!q_seen) mbar_wait(&sm->q_full, 0);
      for (int sl = 0; sl < 2; ++sl)
        if (busy & (1u << sl)) mbar_wait(&sm->full[sl], (fph >> sl) & 1u);
    }
  } else if (warp < kSoftmaxThreads / 32) {
    const StreamSync ss{&sm->s_full, &sm->decided, &sm->p_ready, &sm->o_final, &sm->decision, 1u, 2u};
    softmax_stream<BK>(p, tid, b, h, I, row, n, order_at, tS, tO, ss, &sm->xs, abort);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kCtrl / 32) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

template <int BK>
cudaError_t launch_bk(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const OskParams& p,
                      cudaStream_t st) {
  const unsigned grid = (unsigned)(p.B * p.Hq * p.nqb);
  if (grid == 0) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(osk_attention_kernel<BK>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       OskCfg<BK>::kSmem);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(osk_attention_kernel<BK>, cudaFuncAttributePreferredSharedMemoryCarveout,
                           cudaSharedmemCarveoutMaxShared);
  if (e != cudaSuccess) return e;
  osk_attention_kernel<BK><<<grid, kThreads, OskCfg<BK>::kSmem, st>>>(tq, tk, tv, p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_osk(const CUtensorMap& tm_q, const CUtensorMap& tm_k, const CUtensorMap& tm_v,
                       const OskParams& p, int bk, cudaStream_t st) {
  if (bk == 128) return launch_bk<128>(tm_q, tm_k, tm_v, p, st);
  if (bk == 64) return launch_bk<64>(tm_q, tm_k, tm_v, p, st);
  return cudaErrorInvalidValue;
}

}  // namespace cosa
