// osk_group: the Ordered-Skipping Kernel (CoSA technical summary Sec. 2.3)
// for a visit order shared by the query heads of a GQA group, the execution
// form CompactAttention ("Accelerating Chunked Prefill with Block-Union KV
// Selection", method, execution stage) gives its per-group block tables, and
// the form of the dense path (every causal block, in natural order).
//
// One CTA per (batch, kv-head, Q-block, pair of query heads of the group).
// The two heads' 128-row Q tiles sit side by side in shared memory and TMEM
// (S0, S1, O0, O1: all 512 columns, one CTA per SM); every K and V tile of the
// shared order is loaded once for both.  The arithmetic per head is exactly
// osk_attention's: each head keeps its own running maxima and votes on its
// own tile (a block one head skips may be computed by the other), so the
// result of each head equals cosa_attend's on the same order.
//
// Roles: warp 16 (one thread) issues every TMA load and MMA; warps 0-7 run
// head 0's softmax and warps 8-15 head 1's (softmax_stream, osk_common.cuh).
// The issue order per visit t is QK0(t+1) right after PV0(t) and QK1(t+1)
// right after PV1(t), so one head's softmax runs while the tensor cores work
// on the other head's tiles (ping-pong), and the tensor pipe sees both heads'
// MMAs back to back.  Two K/V slots: K of the next visit is always in
// flight; V of a visit is loaded into the slot its K vacated once both QKs
// have completed and either head has voted to compute.
#include "osk_common.cuh"

namespace cosa {

namespace {

using namespace osk;

constexpr int kHeads = 2;                                    // query heads per CTA
constexpr int kThreads = kHeads * kRowThreads + 32;
constexpr int kCtrl = kHeads * kRowThreads;                  // the control thread (warp 16, lane 0)
constexpr uint32_t kQBytes = 128 * 256;

struct __align__(8) GroupSmem {
  uint64_t q_full, full[2], s_full[kHeads], decided[kHeads], p_ready[kHeads], o_final;
  uint32_t decision[kHeads];
  uint32_t tmem_base;
  uint32_t abort;               // set once any wait of this CTA gave up
  int32_t order[kOrderCap];     // the shared visit order (first kOrderCap entries)
  RowShared xs[kHeads];
};

template <int BK>
struct GroupCfg {
  static constexpr uint32_t kKVBytes = BK * 256;             // BK rows x 128 bf16
  static constexpr uint32_t kChunk = BK * 128;               // one 64-column chunk
  // two Q tiles, two K/V slots, the control block, up to 1023 bytes of alignment
  static constexpr int kSmem = kHeads * kQBytes + 2 * kKVBytes + (int)sizeof(GroupSmem) + 1024;
  static_assert(kSmem <= 227 * 1024, "shared memory of one CTA");
};

template <int BK>
__global__ void __launch_bounds__(kThreads, 1)
osk_group_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                 const __grid_constant__ CUtensorMap tm_v, const OskParams p) {
  using Cfg = GroupCfg<BK>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = base;                                        // head 0, then head 1
  uint8_t* sK = base + kHeads * kQBytes;
  uint8_t* sV = sK + Cfg::kKVBytes;
  GroupSmem* sm = reinterpret_cast<GroupSmem*>(sV + Cfg::kKVBytes);
  volatile uint32_t* abort = &sm->abort;

  const int failed = p.status ? (int)*reinterpret_cast<volatile uint32_t*>(p.status) : 0;
  if (__syncthreads_or(failed)) return;

  const int tid = threadIdx.x, warp = tid >> 5;
  // one kv-head (and batch) at a time, heaviest (last) Q-blocks first, the
  // head pairs of the kv-head adjacent (as in osk_attention: the K/V tiles of
  // the resident CTAs stay in L2)
  const int pairs = p.G / kHeads;
  int x = blockIdx.x;
  const int pr = x % pairs; x /= pairs;
  const int I = p.nqb - 1 - x % p.nqb; x /= p.nqb;
  const int g = x % p.Hkv; x /= p.Hkv;
  const int b = x;
  const int h0 = g * p.G + kHeads * pr;
  const size_t orow = ((size_t)(b * p.Hkv + g)) * p.nqb + I;  // the group's order row
  const int32_t* ord = p.order + orow * p.kmax;
  int n = p.count[orow];
  n = n < 0 ? 0 : (n > p.kmax ? p.kmax : n);

  for (int t = tid; t < n && t < kOrderCap; t += kThreads) sm->order[t] = ord[t];
  auto order_at = [&](int t) -> int { return t < kOrderCap ? sm->order[t] : ord[t]; };
  if (warp == kCtrl / 32) {
    tmem_alloc(&sm->tmem_base, 512);
    tmem_relinquish();
  }
  if (tid == kCtrl) {
    mbar_init(&sm->q_full, 1);
    mbar_init(&sm->full[0], 1);
    mbar_init(&sm->full[1], 1);
    for (int hh = 0; hh < kHeads; ++hh) {
      mbar_init(&sm->s_full[hh], 1);
      mbar_init(&sm->decided[hh], 1);
      mbar_init(&sm->p_ready[hh], kRowThreads);
    }
    mbar_init(&sm->o_final, 1);
    sm->abort = 0;
    fence_mbar_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm->tmem_base;
  // TMEM columns: S of head hh at 128*hh, O of head hh at 256 + 128*hh
  auto tS = [&](int hh) { return tmem + 128u * hh; };
  auto tO = [&](int hh) { return tmem + 256u + 128u * hh; };

  if (tid == kCtrl) {
    // ------------------------------------------------------------ control thread
    if (n > 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      const uint32_t id_qk = idesc_bf16(128, BK, false, false);
      const uint32_t id_pv = idesc_bf16(128, 128, false, true);
      const uint32_t q_addr = smem_u32(sQ), k_addr = smem_u32(sK), v_addr = smem_u32(sV);
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
        const bool r = wait_or_abort(&sm->full[sl], (fph >> sl) & 1u, abort, p.status, DEV_TIMEOUT_TMA,
                                     p.wait_limit_ns);
        if (r) {
          fph ^= 1u << sl;
          busy &= ~(1u << sl);
        }
        return r;
      };
      auto issue_qk = [&](int hh, int sl) {
        const uint32_t qa = q_addr + hh * kQBytes;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ss(tS(hh), desc_sw128(qa + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024),
                 desc_sw128(slot_addr(sl) + (kk >> 2) * Cfg::kChunk + (kk & 3) * 32, 16, 1024), id_qk, kk > 0);
        tc_commit(&sm->s_full[hh]);
      };
      mbar_arrive_expect_tx(&sm->q_full, kHeads * kQBytes);
      for (int hh = 0; hh < kHeads; ++hh) {
        const int q_y = (b * p.Hq + h0 + hh) * p.Nq + I * p.bq;
        tma_load_2d_hint(sQ + hh * kQBytes, &tm_q, &sm->q_full, 0, q_y, pol_q);
        tma_load_2d_hint(sQ + hh * kQBytes + 16384, &tm_q, &sm->q_full, 64, q_y, pol_q);
      }
      load(0, &tm_k, order_at(0));
      if (n > 1) load(1, &tm_k, order_at(1));
      bool any_pv[kHeads] = {false, false};
      const bool q_seen = wait_or_abort(&sm->q_full, 0, abort, p.status, DEV_TIMEOUT_TMA, p.wait_limit_ns);
      bool ok = q_seen && wait_slot(0);
      if (ok) {
        tc_fence_after();
        issue_qk(0, 0);
        issue_qk(1, 0);
      }
      int ks = 0;            // slot holding K of visit t
      int pend_k = -1;       // K load deferred until the PVs reading its slot have completed
      for (int t = 0; ok && t < n; ++t) {
        const uint32_t ph = t & 1;
        const int ns = ks ^ 1;
        // QK1(t) and every earlier MMA (QK0(t) included) are complete: the K
        // slot of visit t is free, and so is the slot the PVs of the last
        // computed visit read
        if (!wait_or_abort(&sm->s_full[1], ph, abort, p.status, DEV_TIMEOUT_MMA, p.wait_limit_ns)) break;
        if (pend_k >= 0) { load(ns, &tm_k, order_at(pend_k)); pend_k = -1; }
        uint32_t dec[kHeads];
        bool v_loaded = false;
        const int jv = order_at(t);
        bool got = true;
#pragma unroll
        for (int hh = 0; hh < kHeads; ++hh) {
          if (!got) break;
          got = wait_or_abort(&sm->decided[hh], ph, abort, p.status, DEV_TIMEOUT_PIPE, p.wait_limit_ns);
          dec[hh] = *reinterpret_cast<volatile uint32_t*>(&sm->decision[hh]);
          if (got && dec[hh] == kDecisionCompute && !v_loaded) {
            load(ks, &tm_v, jv);
            v_loaded = true;
          }
        }
        if (!got) break;
        bool v_seen = false;
        int ksteps = BK / 16;
        bool next_ready = false;
#pragma unroll
        for (int hh = 0; hh < kHeads; ++hh) {
          if (dec[hh] == kDecisionCompute) {
            if (!wait_or_abort(&sm->p_ready[hh], ph, abort, p.status, DEV_TIMEOUT_PIPE, p.wait_limit_ns)) { ok = false; break; }
            if (!v_seen) {
              if (!wait_slot(ks)) { ok = false; break; }
              // a ragged last block: no MMA step past the end of the cache,
              // and the non-key rows of the last step zeroed (clear_v_tail)
              if (p.kv_tail && jv == p.nkb - 1) ksteps = clear_v_tail(slot(ks), Cfg::kChunk, p.kv_tail);
              v_seen = true;
            }
            tc_fence_after();
            // P of keys [16kk, 16kk+16): each column half of the head's S
            // range holds its P at the start of that half
            auto pv_step = [&](int kk) {
              mma_ts(tO(hh), tS(hh) + (kk / (BK / 32)) * (BK / 2) + (kk % (BK / 32)) * 8,
                     desc_sw128(slot_addr(ks) + kk * 2048, Cfg::kChunk, 1024), id_pv,
                     (any_pv[hh] || kk > 0) ? 1u : 0u);
            };
            if (ksteps == BK / 16) {
#pragma unroll
              for (int kk = 0; kk < BK / 16; ++kk) pv_step(kk);
            } else {
              for (int kk = 0; kk < ksteps; ++kk) pv_step(kk);
            }
            any_pv[hh] = true;
          }
          // this head's S (or P, read by the PV just issued, which runs
          // first) may now be overwritten by its QK of the next visit; a
          // skipped visit's S was read before the vote
          if (t + 1 < n) {
            if (!next_ready) {
              if (!wait_slot(ns)) { ok = false; break; }
              next_ready = true;
            }
            tc_fence_after();
            issue_qk(hh, ns);
          }
        }
        if (!ok) break;
        if (v_loaded) {
          if (t + 2 < n) pend_k = t + 2;
        } else if (t + 2 < n) {
          load(ks, &tm_k, order_at(t + 2));
        }
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
  } else if (warp < kCtrl / 32) {
    const int hh = warp / 8;                                  // warps 0-7: head 0, 8-15: head 1
    const int h = h0 + hh;
    const size_t row = ((size_t)(b * p.Hq + h)) * p.nqb + I;  // this head's skip-bit row
    const StreamSync ss{&sm->s_full[hh], &sm->decided[hh], &sm->p_ready[hh], &sm->o_final, &sm->decision[hh],
                        1u + hh, 3u + hh};
    softmax_stream<BK>(p, tid - kRowThreads * hh, b, h, I, row, n, order_at, tS(hh), tO(hh), ss, &sm->xs[hh],
                       abort);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kCtrl / 32) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <int BK>
cudaError_t launch_group_bk(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                            const OskParams& p, cudaStream_t st) {
  const unsigned grid = (unsigned)(p.B * p.Hkv * (p.G / kHeads) * p.nqb);
  if (grid == 0) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(osk_group_kernel<BK>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       GroupCfg<BK>::kSmem);
  if (e != cudaSuccess) return e;
  osk_group_kernel<BK><<<grid, kThreads, GroupCfg<BK>::kSmem, st>>>(tq, tk, tv, p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_osk_group(const CUtensorMap& tm_q, const CUtensorMap& tm_k, const CUtensorMap& tm_v,
                             const OskParams& p, int bk, cudaStream_t st) {
  if (p.G % kHeads != 0) return cudaErrorInvalidValue;
  if (bk == 128) return launch_group_bk<128>(tm_q, tm_k, tm_v, p, st);
  if (bk == 64) return launch_group_bk<64>(tm_q, tm_k, tm_v, p, st);
  return cudaErrorInvalidValue;
}

}  // namespace cosa
