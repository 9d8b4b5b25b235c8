// kap_score: the block-scoring step of the Kernel-Aware Proxy (CoSA
// technical summary Sec. 2.2, "Block Ranking"): pooled scores and MaxPool
// over the keys of each KV block.
//
// A work item is one run of key tiles (128 pooled keys each) of one row tile
// (128 pooled query rows) of one head; the key tiles a row tile sees are cut
// into S items so that short and long rows, and chunks of few queries after
// a long cache, all spread over the GPU.  Per item, one CTA streams its key
// tiles through a TMA ring and contracts them on the tensor cores (tcgen05,
// bf16 x bf16 -> fp32 in TMEM, two TMEM accumulators so the next tile's MMA
// overlaps this tile's epilogue):
//   S[r, c]   = Qp[r] . Kp[c]                    (raw pooled scores)
//   Bs[r, j]  = max over visible c in block j     (MaxPool over keys)
// It stores Bs and, per pooled row and column half, the largest Bs of the
// item and the first block attaining it.  MaxNorm, the HRM flags and the
// Q-block aggregate need every item of the row and run in kap_sort.
// Every value is fp32; nothing is rounded after the contraction.
//
// Roles: warp 8 (one thread) issues the MMAs, warp 9 (one thread) the TMA
// loads, refilling a stage as soon as the MMAs of its tile have completed, so
// the MMA issue never waits for a refill; warps 0-7 are the epilogue, two per
// TMEM lane quarter (row = 32*(warp%4) + lane), each taking one 64-column
// half of every tile.
#include <cuda_bf16.h>
#include "internal.h"
#include "sm100.cuh"

namespace cosa {

namespace {

constexpr int kEpiWarps = 8;
constexpr int kThreads = 32 * (kEpiWarps + 2);
constexpr int kCtrl = 32 * kEpiWarps;            // the MMA-issuing thread
constexpr int kProd = 32 * (kEpiWarps + 1);      // the TMA-issuing thread
constexpr uint32_t kTileBytes = 128 * 256;       // 128 rows x 128 bf16

struct __align__(8) ScoreSmem {
  uint64_t q_full;
  uint64_t k_full[2];
  uint64_t s_full[2];
  uint64_t s_free[2];
  uint64_t drained;
  uint32_t tmem_base;
  uint32_t abort;
};

// tiles, the control block, and up to 1023 bytes lost aligning the base to 1 KB
constexpr int kSmemBytes = 3 * kTileBytes + (int)sizeof(ScoreSmem) + 1024;
static_assert(2 * (kSmemBytes + 1024) <= 228 * 1024, "two CTAs must share an SM");

// K-major SW128 descriptor of k-step kk (16 bf16) of a 128-row tile stored
// as two 64-column chunks of 16 KB.
__device__ __forceinline__ uint64_t tile_desc(uint32_t base, int kk) {
  return desc_sw128(base + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024);
}

template <int KPB>
__global__ void __launch_bounds__(kThreads, 2)
kap_score_kernel(const __grid_constant__ CUtensorMap tm_qp, const __grid_constant__ CUtensorMap tm_kp,
                 const ScoreParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = base;
  uint8_t* sK = base + kTileBytes;               // two stages
  ScoreSmem* sm = reinterpret_cast<ScoreSmem*>(base + 3 * kTileBytes);
  volatile uint32_t* abort = &sm->abort;

  // a CTA launched after another one reported a device error does no work
  const int failed = p.status ? (int)*reinterpret_cast<volatile uint32_t*>(p.status) : 0;
  if (__syncthreads_or(failed)) return;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int heads = p.Hq * p.B;
  const int hb = blockIdx.x % heads;
  const int item = blockIdx.x / heads;                         // heaviest row tiles first
  const int R = p.n_row_tiles - 1 - item / p.splits;
  const int split = item % p.splits;
  const int h = hb % p.Hq, b = hb / p.Hq, g = h / p.G;
  const int r_first = R * kTileRows;
  const int rows_valid = min(kTileRows, p.nqp - r_first);
  const int nT = kap_row_tiles_seen(R, p.nqp, p.nkp, p.off_p);
  int t0, t1;
  kap_split_range(nT, p.splits, split, t0, t1);
  const int U = t1 - t0;                                       // key tiles of this item (may be 0)
  constexpr int BPT = kTileRows / KPB;                         // KV blocks per key tile
  constexpr int BPH = BPT / 2;                                 // per 64-column half

  if (warp == kEpiWarps) {
    tmem_alloc(&sm->tmem_base, 256);
    tmem_relinquish();
  }
  if (tid == kCtrl) {
    mbar_init(&sm->q_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sm->k_full[i], 1);
      mbar_init(&sm->s_full[i], 1);
      mbar_init(&sm->s_free[i], 32 * kEpiWarps);
    }
    mbar_init(&sm->drained, 1);
    sm->abort = 0;
    fence_mbar_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm->tmem_base;

  if (tid == kProd) {
    // ------------------------------------------------ producer: TMA loads
    tma_prefetch_desc(&tm_qp);
    tma_prefetch_desc(&tm_kp);
    const int qp_y = (b * p.Hq + h) * p.nqp + r_first;
    const int kp_y0 = (b * p.Hkv + g) * p.kp_stride;
    if (U > 0) {
      mbar_arrive_expect_tx(&sm->q_full, kTileBytes);
      tma_load_2d(sQ, &tm_qp, &sm->q_full, 0, qp_y);
      tma_load_2d(sQ + 16384, &tm_qp, &sm->q_full, 64, qp_y);
    }
    int loads[2] = {0, 0};   // key-tile loads issued on each stage
    auto load = [&](int st, int u) {
      uint8_t* dst = sK + st * kTileBytes;
      const int y = kp_y0 + (t0 + u) * kTileRows;
      ++loads[st];
      mbar_arrive_expect_tx(&sm->k_full[st], kTileBytes);
      tma_load_2d(dst, &tm_kp, &sm->k_full[st], 0, y);
      tma_load_2d(dst + 16384, &tm_kp, &sm->k_full[st], 64, y);
    };
    for (int u = 0; u < 2 && u < U; ++u) load(u, u);
    // refill a stage with tile u + 2 once the MMAs of tile u have completed
    for (int u = 0; u + 2 < U; ++u) {
      if (!wait_or_abort(&sm->s_full[u & 1], (u >> 1) & 1, abort, p.status, DEV_TIMEOUT_MMA)) break;
      load(u & 1, u + 2);
    }
    // no copy may still be writing shared memory when the CTA exits: wait
    // (bounded) for the last load of each stage and for Q; on the normal path
    // the issuing thread has seen them all complete already
    if (U > 0) mbar_wait(&sm->q_full, 0);
    for (int st = 0; st < 2; ++st)
      if (loads[st] > 0) mbar_wait(&sm->k_full[st], (uint32_t)(loads[st] - 1) & 1u);
  } else if (tid == kCtrl) {
    // ------------------------------------------------ MMA issue
    const bool q_seen = U > 0 && wait_or_abort(&sm->q_full, 0, abort, p.status, DEV_TIMEOUT_TMA);
    bool ok = q_seen;
    const uint32_t idesc = idesc_bf16(128, 128, false, false);
    const uint32_t q_addr = smem_u32(sQ);
    for (int u = 0; ok && u < U; ++u) {
      const int st = u & 1;
      const uint32_t ph = (u >> 1) & 1;
      if (!wait_or_abort(&sm->k_full[st], ph, abort, p.status, DEV_TIMEOUT_TMA)) break;
      if (u >= 2 && !wait_or_abort(&sm->s_free[st], ((u >> 1) - 1) & 1, abort, p.status, DEV_TIMEOUT_PIPE)) break;
      tc_fence_after();
      const uint32_t k_addr = smem_u32(sK + st * kTileBytes);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        mma_ss(tmem + st * 128, tile_desc(q_addr, kk), tile_desc(k_addr, kk), idesc, kk > 0);
      tc_commit(&sm->s_full[st]);
    }
    // every MMA this thread issued has completed before TMEM is released
    tc_commit(&sm->drained);
    mbar_wait(&sm->drained, 0);
  } else if (warp < kEpiWarps) {
    // ------------------------------------------------ epilogue: one pooled row, one column half
    const int quarter = warp & 3, half = warp >> 2;
    const int row = 32 * quarter + lane;
    const int r = r_first + row;
    const bool row_ok = row < rows_valid;
    const int climit = p.off_p + r;
    float rowmax = -INFINITY;
    int argj = -1;
    // this row's Bs: per (head, row tile) [Q-block][nKB][rows of the Q-block],
    // so kap_sort reads each Q-block's scores contiguously
    float* bs_row = p.bs + ((size_t)hb * p.n_row_tiles + R) * p.nkb * kTileRows + (size_t)(row / p.rpq) * p.nkb * p.rpq + row % p.rpq;
    for (int u = 0; u < U; ++u) {
      const int st = u & 1;
      const int T = t0 + u;
      const bool got = wait_or_abort(&sm->s_full[st], (u >> 1) & 1, abort, p.status, DEV_TIMEOUT_MMA);
      tc_fence_after();
      float bsv[BPH];
#pragma unroll
      for (int jh = 0; jh < BPH; ++jh) bsv[jh] = -INFINITY;
      const int c_lo = T * kTileRows + 64 * half;              // first pooled key of this half
      // a half every column of which this row sees needs no per-column test
      const bool full = got && row_ok && c_lo + 63 <= climit && c_lo + 64 <= p.nkp;
      {
        uint32_t v[64];
        tmem_ld_x64(tmem_addr(tmem, 32 * quarter, st * 128 + 64 * half), v);
        // the accumulator stage is in registers: hand it back to the MMA at once
        tc_fence_before();
        mbar_arrive(&sm->s_free[st]);
        if (full) {
#pragma unroll
          for (int i = 0; i < 64; i += 2) {
            float m3;
            asm("max.f32 %0, %1, %2, %3;" : "=f"(m3) : "f"(bsv[i / KPB]), "f"(__uint_as_float(v[i])), "f"(__uint_as_float(v[i + 1])));
            bsv[i / KPB] = m3;
          }
        } else {
#pragma unroll
          for (int i = 0; i < 64; ++i) {
            const int c = c_lo + i;
            const bool vis = got && row_ok && c <= climit && c < p.nkp;
            bsv[i / KPB] = fmaxf(bsv[i / KPB], vis ? __uint_as_float(v[i]) : -INFINITY);
          }
        }
      }

      const int j0 = T * BPT + half * BPH;                     // first block of this half
#pragma unroll
      for (int jh = 0; jh < BPH; ++jh)
        if (j0 + jh < p.nkb) bs_row[(size_t)(j0 + jh) * p.rpq] = bsv[jh];
#pragma unroll
      for (int jh = 0; jh < BPH; ++jh)
        if (bsv[jh] > rowmax) { rowmax = bsv[jh]; argj = j0 + jh; }
    }
    // this item's row maximum for this column half (-inf / -1 when it saw nothing)
    const size_t pi = ((((size_t)hb * p.n_row_tiles + R) * p.splits + split) * 2 + half) * kTileRows + row;
    p.part_max[pi] = rowmax;
    p.part_arg[pi] = argj;
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kEpiWarps) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

}  // namespace

cudaError_t launch_kap_score(const CUtensorMap& tm_qp, const CUtensorMap& tm_kp, const ScoreParams& p,
                             cudaStream_t st) {
  const unsigned grid = (unsigned)(p.n_row_tiles * p.splits * p.Hq * p.B);
  if (grid == 0) return cudaSuccess;
#define COSA_LAUNCH_SCORE(K)                                                                          \
  case K: {                                                                                           \
    cudaError_t e = cudaFuncSetAttribute(kap_score_kernel<K>, cudaFuncAttributeMaxDynamicSharedMemorySize, \
                                         kSmemBytes);                                                 \
    if (e != cudaSuccess) return e;                                                                   \
    e = cudaFuncSetAttribute(kap_score_kernel<K>, cudaFuncAttributePreferredSharedMemoryCarveout,     \
                             cudaSharedmemCarveoutMaxShared);                                         \
    if (e != cudaSuccess) return e;                                                                   \
    kap_score_kernel<K><<<grid, kThreads, kSmemBytes, st>>>(tm_qp, tm_kp, p);                         \
    break;                                                                                            \
  }
  switch (p.kpb) {
    COSA_LAUNCH_SCORE(4)
    COSA_LAUNCH_SCORE(8)
    COSA_LAUNCH_SCORE(16)
    COSA_LAUNCH_SCORE(32)
    default:
      return cudaErrorInvalidValue;
  }
#undef COSA_LAUNCH_SCORE
  return cudaGetLastError();
}

}  // namespace cosa
