// Host front end of the C ABI declared in include/cosa.h: argument
// validation, workspace carving, TMA tensor-map encoding and kernel launch.
// No device memory is allocated here; every launch goes to the caller's
// stream.
#include <cudaTypedefs.h>
#include <cmath>
#include <algorithm>
#include <cstring>
#include <mutex>
#include <vector>

#include "cosa.h"
#include "internal.h"
#include "block_union.h"
#include "decode.h"

using namespace cosa;

namespace {

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

bool encoder() {
  std::call_once(g_encode_once, [] {
    cudaDriverEntryPointQueryResult q;
    void* fn = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  return g_encode != nullptr;
}

// [rows, 128] bf16 row-major viewed as a 2D tensor; box = 64 columns x
// box_rows rows, 128-byte swizzle (the layout the MMA descriptors expect).
cosa_status make_map(CUtensorMap* m, const void* ptr, long long rows, int box_rows) {
  if (!encoder()) return COSA_ECUDA;
  cuuint64_t dims[2] = {(cuuint64_t)kD, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)kD * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  cuuint32_t es[2] = {1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, es,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? COSA_OK : COSA_ECUDA;
}

int cdiv(int a, int b) { return (a + b - 1) / b; }
size_t align256(size_t x) { return (x + 255) & ~size_t(255); }
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }
bool pow2(int x) { return x > 0 && (x & (x - 1)) == 0; }

// Shape checks shared by every entry point.
cosa_status check_shape(const cosa_shape* s) {
  if (!s) return COSA_EINVAL;
  if (s->B < 0 || s->Hq < 1 || s->Hkv < 1 || s->Nq < 0 || s->Nkv < 0) return COSA_EINVAL;
  if (s->Hq % s->Hkv || s->Nkv < s->Nq) return COSA_ESHAPE;
  if (s->d != kD) return COSA_EUNSUPPORTED;
  if ((s->bq != 64 && s->bq != 128) || (s->bk != 64 && s->bk != 128)) return COSA_EUNSUPPORTED;
  if (s->paged && s->num_pages < 1) return COSA_EINVAL;
  // TMA coordinates are 32-bit
  const long long lim = 1ll << 31;
  if ((long long)s->B * s->Hq * (s->Nq + 128) >= lim || (long long)s->B * s->Hkv * (s->Nkv + 128) >= lim)
    return COSA_EUNSUPPORTED;
  if (s->paged && (long long)s->num_pages * s->Hkv * s->bk >= lim) return COSA_EUNSUPPORTED;
  return COSA_OK;
}

// Additional checks of the proxy (pooling stride).
cosa_status check_plan_shape(const cosa_shape* s) {
  cosa_status st = check_shape(s);
  if (st != COSA_OK) return st;
  const int str = s->stride;
  if (!pow2(str) || s->bq % str || s->bk % str) return COSA_EUNSUPPORTED;
  const int kpb = s->bk / str, rpq = s->bq / str;
  if (kpb < 4 || kpb > 32 || rpq > 32) return COSA_EUNSUPPORTED;
  if (s->Nq % str || s->Nkv % str) return COSA_ESHAPE;
  if (cdiv(s->Nkv, s->bk) > 16384) return COSA_EUNSUPPORTED;   // sort keys must fit shared memory
  return COSA_OK;
}

int n_qblocks(const cosa_shape* s) { return cdiv(s->Nq, s->bq); }
int n_kblocks(const cosa_shape* s) { return cdiv(s->Nkv, s->bk); }

int causal_blocks(const cosa_shape* s, int I) {
  const int last = std::min((I + 1) * s->bq, s->Nq) - 1;
  return std::min(n_kblocks(s), (s->Nkv - s->Nq + last) / s->bk + 1);
}

int budget_bp(double budget) { return (int)std::lround(budget * 10000.0); }

int budget_k(int n, int bp) {
  long long k = ((long long)n * bp + 9999) / 10000;
  if (k < 1) k = 1;
  if (k > n) k = n;
  return (int)k;
}

// Work items per row tile of kap_score (S): half of what it takes to fill
// the GPU with four CTAs per slot (two slots per SM) and to keep every item
// under an eighth of a slot's share of all key tiles, and at least eight key
// tiles per item where rows are long enough.  Halving the count of the full
// rule measured 3-6% faster on the 128K and 32K layers and the 4096-query
// chunk (one B200, same-box A/B): a CTA's set-up costs more than the tail
// the extra items save.
int score_splits(const cosa_shape* s) {
  const int nqp = s->Nq / s->stride, nkp = s->Nkv / s->stride, off_p = (s->Nkv - s->Nq) / s->stride;
  const int nrt = cdiv(nqp, kTileRows);
  if (nrt == 0 || s->B == 0) return 1;
  long long tiles = 0;
  int nt_max = 0;
  for (int R = 0; R < nrt; ++R) {
    const int nt = kap_row_tiles_seen(R, nqp, nkp, off_p);
    tiles += nt;
    nt_max = std::max(nt_max, nt);
  }
  const long long heads = (long long)s->B * s->Hq, slots = 2ll * 148;
  tiles *= heads;
  const long long s_fill = (4 * slots + heads * nrt - 1) / (heads * nrt);
  const long long s_tail = (8ll * nt_max * slots + tiles - 1) / std::max(1ll, tiles);
  const long long s_cap = std::max(1, nt_max / 4);
  return (int)std::max(1ll, std::min(std::max(s_fill, s_tail), s_cap) / 2);
}

struct Workspace {
  size_t qp, kp, bs, pmax, parg, total;
  int splits;
};

Workspace carve(const cosa_shape* s) {
  Workspace w;
  const long long rows_q = std::max<long long>((long long)s->B * s->Hq * (s->Nq / s->stride), 0) + 128;
  const long long rows_k = std::max<long long>((long long)s->B * s->Hkv * (s->Nkv / s->stride), 0) + 128;
  const size_t row_tiles = (size_t)cdiv(s->Nq / s->stride, kTileRows);
  const size_t heads = (size_t)s->B * s->Hq;
  w.splits = score_splits(s);
  w.qp = 0;
  w.kp = align256(w.qp + (size_t)rows_q * kD * 2);
  w.bs = align256(w.kp + (size_t)rows_k * kD * 2);
  w.pmax = align256(w.bs + heads * row_tiles * n_kblocks(s) * kTileRows * sizeof(float));
  w.parg = align256(w.pmax + heads * row_tiles * w.splits * 2 * kTileRows * sizeof(float));
  w.total = align256(w.parg + heads * row_tiles * w.splits * 2 * kTileRows * sizeof(int32_t));
  return w;
}

cosa_status launch_status(cudaError_t e) { return e == cudaSuccess ? COSA_OK : COSA_ECUDA; }

// Shared body of cosa_plan and cosa_plan_chunk.  Pooled keys live in `kp`
// ([B, Hkv, kp_stride, d]); rows kp_first .. Nkv/s-1 are pooled from k here,
// rows below kp_first are read as they are.
cosa_status plan_impl(const cosa_shape* shape, const void* q, const void* k, const int32_t* page_table,
                      uint16_t* kp, long long kp_map_rows, int kp_stride, int kp_first, double budget,
                      int kmax, int32_t* order, int32_t* count, int32_t* hrm_count, float* block_score,
                      uint8_t* hrm_flags, uint8_t* ws, uint32_t* dev_status, cudaStream_t stream) {
  cosa_status st;
  const cosa_shape& s = *shape;
  const Workspace w = carve(&s);
  uint16_t* qp = reinterpret_cast<uint16_t*>(ws + w.qp);
  float* bs = reinterpret_cast<float*>(ws + w.bs);
  float* pmax = reinterpret_cast<float*>(ws + w.pmax);
  int32_t* parg = reinterpret_cast<int32_t*>(ws + w.parg);
  const int str = s.stride;

  PoolParams pp;
  pp.q = static_cast<const uint16_t*>(q);
  pp.k = static_cast<const uint16_t*>(k);
  pp.page_table = page_table;
  pp.qp = qp;
  pp.kp = kp;
  pp.B = s.B; pp.Hq = s.Hq; pp.Hkv = s.Hkv; pp.Nq = s.Nq; pp.Nkv = s.Nkv; pp.s = str; pp.bk = s.bk;
  pp.nkb = n_kblocks(&s); pp.paged = s.paged; pp.num_pages = s.num_pages;
  pp.kp_first = kp_first; pp.kp_stride = kp_stride;
  pp.q_items = (long long)s.B * s.Hq * (s.Nq / str);
  pp.k_items = (long long)s.B * s.Hkv * (s.Nkv / str - kp_first);
  if ((st = launch_status(launch_kap_pool(pp, stream))) != COSA_OK) return st;

  CUtensorMap tm_qp, tm_kp;
  if ((st = make_map(&tm_qp, qp, pp.q_items + 128, 128)) != COSA_OK) return st;
  if ((st = make_map(&tm_kp, kp, kp_map_rows, 128)) != COSA_OK) return st;
  ScoreParams sp;
  sp.B = s.B; sp.Hq = s.Hq; sp.Hkv = s.Hkv; sp.G = s.Hq / s.Hkv;
  sp.nqp = s.Nq / str; sp.nkp = s.Nkv / str; sp.kp_stride = kp_stride; sp.off_p = (s.Nkv - s.Nq) / str;
  sp.nkb = n_kblocks(&s);
  sp.kpb = s.bk / str;
  sp.n_row_tiles = cdiv(sp.nqp, kTileRows);
  sp.splits = w.splits;
  sp.rpq = s.bq / str;
  sp.bs = bs; sp.part_max = pmax; sp.part_arg = parg; sp.status = dev_status;
  if ((st = launch_status(launch_kap_score(tm_qp, tm_kp, sp, stream))) != COSA_OK) return st;

  SortParams so;
  so.B = s.B; so.Hq = s.Hq; so.nqb = n_qblocks(&s); so.nkb = sp.nkb; so.Nq = s.Nq; so.Nkv = s.Nkv;
  so.bq = s.bq; so.bk = s.bk; so.rpq = s.bq / str;
  so.nqp = sp.nqp; so.n_row_tiles = sp.n_row_tiles; so.splits = sp.splits;
  so.bp = budget_bp(budget); so.kmax = kmax;
  so.bs = bs; so.part_max = pmax; so.part_arg = parg;
  so.order = order; so.count = count; so.hrm_count = hrm_count;
  so.block_score = block_score; so.hrm_flags = hrm_flags;
  return launch_status(launch_kap_sort(so, stream));
}

// Checks common to cosa_plan and cosa_plan_chunk.  *done is set when there
// is nothing to launch (no Q-blocks).
cosa_status check_plan_args(const cosa_shape* shape, const void* q, const void* k,
                            const int32_t* page_table, double budget, int kmax, const int32_t* order,
                            const int32_t* count, const void* workspace, size_t ws_bytes, bool* done) {
  *done = false;
  cosa_status st = check_plan_shape(shape);
  if (st != COSA_OK) return st;
  if (!(budget > 0.0) || budget > 1.0) return COSA_EINVAL;
  const cosa_shape& s = *shape;
  if ((long long)s.B * s.Hq * n_qblocks(&s) == 0) {
    *done = true;
    return COSA_OK;
  }
  if (!q || !k || !order || !count || (s.paged && !page_table)) return COSA_EINVAL;
  if (!aligned16(q) || !aligned16(k)) return COSA_EALIGN;
  if (kmax < cosa_kmax(&s, budget)) return COSA_EINVAL;
  if (!workspace || ws_bytes < carve(&s).total) return COSA_EWORKSPACE;
  if (reinterpret_cast<uintptr_t>(workspace) & 255) return COSA_EALIGN;
  return COSA_OK;
}

}  // namespace

extern "C" {

int cosa_num_qblocks(const cosa_shape* shape) { return check_shape(shape) == COSA_OK ? n_qblocks(shape) : -1; }
int cosa_num_kblocks(const cosa_shape* shape) { return check_shape(shape) == COSA_OK ? n_kblocks(shape) : -1; }

int cosa_kmax(const cosa_shape* shape, double budget) {
  if (check_plan_shape(shape) != COSA_OK || !(budget > 0.0) || budget > 1.0) return -1;
  if (shape->Nq == 0) return 0;
  return budget_k(causal_blocks(shape, n_qblocks(shape) - 1), budget_bp(budget));
}

size_t cosa_plan_workspace_bytes(const cosa_shape* shape) {
  if (check_plan_shape(shape) != COSA_OK) return 0;
  return carve(shape).total;
}

float cosa_skip_threshold(double eps, int d) {
  if (!(eps > 0.0)) return -INFINITY;
  return (float)(std::log(eps) * std::sqrt((double)d));
}

cosa_status cosa_plan(const cosa_shape* shape, const void* q, const void* k, const int32_t* page_table,
                      double budget, int kmax, int32_t* order, int32_t* count, int32_t* hrm_count,
                      float* block_score, uint8_t* hrm_flags, void* workspace, size_t ws_bytes,
                      uint32_t* dev_status, cudaStream_t stream) {
  bool done;
  cosa_status st = check_plan_args(shape, q, k, page_table, budget, kmax, order, count, workspace, ws_bytes, &done);
  if (st != COSA_OK || done) return st;
  const cosa_shape& s = *shape;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const Workspace w = carve(&s);
  const int nkp = s.Nkv / s.stride;
  return plan_impl(&s, q, k, page_table, reinterpret_cast<uint16_t*>(ws + w.kp),
                   (long long)s.B * s.Hkv * nkp + 128, nkp, 0, budget, kmax, order, count, hrm_count,
                   block_score, hrm_flags, ws, dev_status, stream);
}

cosa_status cosa_plan_chunk(const cosa_shape* shape, const void* q, const void* k, const int32_t* page_table,
                            void* kp_cache, int kp_capacity, int kp_valid, double budget, int kmax,
                            int32_t* order, int32_t* count, int32_t* hrm_count, float* block_score,
                            uint8_t* hrm_flags, void* workspace, size_t ws_bytes, uint32_t* dev_status,
                            cudaStream_t stream) {
  bool done;
  cosa_status st = check_plan_args(shape, q, k, page_table, budget, kmax, order, count, workspace, ws_bytes, &done);
  if (st != COSA_OK || done) return st;
  const cosa_shape& s = *shape;
  const int nkp = s.Nkv / s.stride;
  if (!kp_cache) return COSA_EINVAL;
  if (!aligned16(kp_cache)) return COSA_EALIGN;
  if (kp_capacity < nkp || kp_valid < 0 || kp_valid > nkp) return COSA_EINVAL;
  if ((long long)s.B * s.Hkv * kp_capacity >= (1ll << 31)) return COSA_EUNSUPPORTED;
  return plan_impl(&s, q, k, page_table, static_cast<uint16_t*>(kp_cache), (long long)s.B * s.Hkv * kp_capacity,
                   kp_capacity, kp_valid, budget, kmax, order, count, hrm_count, block_score, hrm_flags,
                   static_cast<uint8_t*>(workspace), dev_status, stream);
}

cosa_status cosa_check_order(const cosa_shape* shape, const int32_t* order_host, const int32_t* count_host,
                             int kmax, int64_t* first_bad) {
  if (first_bad) *first_bad = 0;
  cosa_status st = check_shape(shape);
  if (st != COSA_OK) return st;
  if (kmax < 1) return COSA_ESHAPE;
  const int nqb = n_qblocks(shape), nkb = n_kblocks(shape);
  const long long rows = (long long)shape->B * shape->Hq * nqb;
  if (rows == 0) return COSA_OK;
  if (!order_host || !count_host) return COSA_EINVAL;
  std::vector<uint64_t> seen((size_t)(nkb + 63) / 64);
  for (long long row = 0; row < rows; ++row) {
    const int n = count_host[row];
    if (n < 0 || n > kmax) {
      if (first_bad) *first_bad = -1 - row;
      return COSA_EINVAL;
    }
    const int n_vis = causal_blocks(shape, (int)(row % nqb));
    std::fill(seen.begin(), seen.end(), 0ull);
    const int32_t* ord = order_host + row * kmax;
    for (int t = 0; t < n; ++t) {
      const int j = ord[t];
      const bool bad = j < 0 || j >= n_vis || ((seen[(size_t)j >> 6] >> (j & 63)) & 1ull);
      if (bad) {
        if (first_bad) *first_bad = row * kmax + t;
        return COSA_EINVAL;
      }
      seen[(size_t)j >> 6] |= 1ull << (j & 63);
    }
  }
  return COSA_OK;
}

cosa_status cosa_dense_order(const cosa_shape* shape, int kmax, int32_t* order, int32_t* count,
                             cudaStream_t stream) {
  cosa_status st = check_shape(shape);
  if (st != COSA_OK) return st;
  const int rows = shape->B * shape->Hq * n_qblocks(shape);
  if (rows == 0) return COSA_OK;
  if (!order || !count) return COSA_EINVAL;
  if (kmax < causal_blocks(shape, n_qblocks(shape) - 1)) return COSA_EINVAL;
  return launch_status(launch_dense_order(rows, n_qblocks(shape), n_kblocks(shape), shape->Nq, shape->Nkv,
                                          shape->bq, shape->bk, kmax, order, count, stream));
}

cosa_status cosa_decode_plan(const cosa_shape* shape, const void* q, const void* k, const int32_t* page_table,
                             void* kp_cache, int kp_capacity, int kp_valid, double budget, int kmax,
                             int32_t* order, int32_t* count, int32_t* hrm_count, float* block_score,
                             uint8_t* hrm_flags, cudaStream_t stream) {
  cosa_status st = check_shape(shape);
  if (st != COSA_OK) return st;
  const cosa_shape& s = *shape;
  if (s.Nq != 1) return COSA_ESHAPE;
  const int str = s.stride;
  if (!pow2(str) || s.bk % str || s.bk / str > 32 || s.Nkv % str) return COSA_EUNSUPPORTED;
  if (!(budget > 0.0) || budget > 1.0) return COSA_EINVAL;
  const int nkb = n_kblocks(&s), nkp = s.Nkv / str;
  if (nkb > 16384) return COSA_EUNSUPPORTED;
  if ((long long)s.B * s.Hq == 0 || s.Nkv == 0) return COSA_OK;
  if (!q || !k || !kp_cache || !order || !count || (s.paged && !page_table)) return COSA_EINVAL;
  if (!aligned16(q) || !aligned16(k) || !aligned16(kp_cache)) return COSA_EALIGN;
  if (kp_capacity < nkp || kp_valid < 0 || kp_valid > nkp) return COSA_EINVAL;
  if ((long long)s.B * s.Hkv * kp_capacity >= (1ll << 31)) return COSA_EUNSUPPORTED;
  const int kk = budget_k(nkb, budget_bp(budget));
  if (kmax < kk) return COSA_EINVAL;
  if (decode_plan_smem(nkb, kk) > 227 * 1024) return COSA_EUNSUPPORTED;
  // pool the keys no earlier call pooled into the cache
  PoolParams pp;
  pp.q = nullptr; pp.qp = nullptr;
  pp.k = static_cast<const uint16_t*>(k);
  pp.page_table = page_table;
  pp.kp = static_cast<uint16_t*>(kp_cache);
  pp.B = s.B; pp.Hq = s.Hq; pp.Hkv = s.Hkv; pp.Nq = s.Nq; pp.Nkv = s.Nkv; pp.s = str; pp.bk = s.bk;
  pp.nkb = nkb; pp.paged = s.paged; pp.num_pages = s.num_pages;
  pp.kp_first = kp_valid; pp.kp_stride = kp_capacity;
  pp.q_items = 0;
  pp.k_items = (long long)s.B * s.Hkv * (nkp - kp_valid);
  if ((st = launch_status(launch_kap_pool(pp, stream))) != COSA_OK) return st;
  DecodePlanParams dp;
  dp.B = s.B; dp.Hq = s.Hq; dp.Hkv = s.Hkv;
  dp.nkb = nkb; dp.nkp = nkp; dp.kpb = s.bk / str; dp.kp_stride = kp_capacity;
  dp.k = kk; dp.kmax = kmax;
  dp.q = static_cast<const uint16_t*>(q);
  dp.kp = static_cast<const uint16_t*>(kp_cache);
  dp.order = order; dp.count = count; dp.hrm_count = hrm_count;
  dp.block_score = block_score; dp.hrm_flags = hrm_flags;
  return launch_status(launch_decode_plan(dp, stream));
}

size_t cosa_decode_attend_workspace_bytes(const cosa_shape* shape, int kmax) {
  if (check_shape(shape) != COSA_OK || shape->Nq != 1 || kmax < 1) return 0;
  return decode_attend_workspace(shape->B * shape->Hq, kmax, shape->bk);
}

cosa_status cosa_decode_attend(const cosa_shape* shape, const void* q, const void* k, const void* v,
                               const int32_t* page_table, const int32_t* order, const int32_t* count, int kmax,
                               double skip_eps, void* out, float* lse, uint32_t* skip_bits, void* workspace,
                               size_t ws_bytes, cudaStream_t stream) {
  cosa_status st = check_shape(shape);
  if (st != COSA_OK) return st;
  const cosa_shape& s = *shape;
  if (s.Nq != 1) return COSA_ESHAPE;
  if (!(skip_eps >= 0.0) || skip_eps >= 1.0) return COSA_EINVAL;
  const int rows = s.B * s.Hq;
  if (rows == 0) return COSA_OK;
  if (!q || !k || !v || !out || !order || !count || (s.paged && !page_table)) return COSA_EINVAL;
  if (kmax < 1) return COSA_EINVAL;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return COSA_EALIGN;
  if (decode_attend_smem(kmax, s.bk) > 227 * 1024) return COSA_EUNSUPPORTED;
  if (!workspace || ws_bytes < decode_attend_workspace(rows, kmax, s.bk)) return COSA_EWORKSPACE;
  if (reinterpret_cast<uintptr_t>(workspace) & 255) return COSA_EALIGN;
  DecodeAttendParams p;
  p.B = s.B; p.Hq = s.Hq; p.Hkv = s.Hkv; p.Nkv = s.Nkv; p.nkb = n_kblocks(&s); p.bk = s.bk;
  p.paged = s.paged; p.num_pages = s.num_pages; p.kmax = kmax;
  p.q = static_cast<const uint16_t*>(q);
  p.k = static_cast<const uint16_t*>(k);
  p.v = static_cast<const uint16_t*>(v);
  p.page_table = page_table; p.order = order; p.count = count;
  p.T = cosa_skip_threshold(skip_eps, s.d);
  p.scale_ln = (float)(1.0 / std::sqrt((double)s.d));
  p.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)s.d));
  p.out = static_cast<uint16_t*>(out); p.lse = lse; p.skip_bits = skip_bits; p.skip_words = cdiv(kmax, 32);
  return launch_status(launch_decode_attend(p, static_cast<uint8_t*>(workspace), stream));
}

cosa_status cosa_block_union(const cosa_shape* shape, const int32_t* order, const int32_t* count, int kmax,
                             int32_t* table, int32_t* table_len, int32_t* union_order, int32_t* union_count,
                             int union_kmax, cudaStream_t stream) {
  cosa_status st = check_shape(shape);
  if (st != COSA_OK) return st;
  const cosa_shape& s = *shape;
  if ((long long)s.B * s.Hkv == 0) return COSA_OK;
  if (!table || !table_len || kmax < 0) return COSA_EINVAL;
  const int nqb = n_qblocks(&s);
  if (nqb > 0 && kmax > 0 && (!order || !count)) return COSA_EINVAL;
  if (union_order || union_count) {
    if (!union_order || !union_count) return COSA_EINVAL;
    if (nqb > 0 && union_kmax < causal_blocks(&s, nqb - 1)) return COSA_EINVAL;
  }
  UnionParams p;
  p.B = s.B; p.Hq = s.Hq; p.Hkv = s.Hkv; p.nqb = nqb; p.nkb = n_kblocks(&s);
  p.Nq = s.Nq; p.Nkv = s.Nkv; p.bq = s.bq; p.bk = s.bk;
  p.order = order; p.count = count; p.kmax = (nqb > 0) ? kmax : 0;
  p.table = table; p.table_len = table_len;
  p.union_order = union_order; p.union_count = union_count; p.union_kmax = union_kmax;
  return launch_status(launch_block_union(p, stream));
}

}  // extern "C"

namespace {

cosa_status attend_impl(const cosa_shape* shape, const void* q, const void* k, const void* v,
                        const int32_t* page_table, const int32_t* order, const int32_t* count, int kmax,
                        double skip_eps, void* out, float* lse, uint32_t* skip_bits, uint32_t* dev_status,
                        uint64_t wait_limit_ns, int stall_test, bool group, cudaStream_t stream) {
  cosa_status st = check_shape(shape);
  if (st != COSA_OK) return st;
  if (!(skip_eps >= 0.0) || skip_eps >= 1.0) return COSA_EINVAL;
  const cosa_shape& s = *shape;
  const long long rows = (long long)s.B * s.Hq * n_qblocks(&s);
  if (rows == 0) return COSA_OK;
  if (!q || !k || !v || !out || !order || !count || (s.paged && !page_table)) return COSA_EINVAL;
  if (kmax < 1) return COSA_EINVAL;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return COSA_EALIGN;
  CUtensorMap tm_q, tm_k, tm_v;
  const long long kv_rows = s.paged ? (long long)s.num_pages * s.Hkv * s.bk : (long long)s.B * s.Hkv * s.Nkv;
  if ((st = make_map(&tm_q, q, (long long)s.B * s.Hq * s.Nq, 128)) != COSA_OK) return st;
  if ((st = make_map(&tm_k, k, kv_rows, s.bk)) != COSA_OK) return st;
  if ((st = make_map(&tm_v, v, kv_rows, s.bk)) != COSA_OK) return st;
  OskParams p;
  p.B = s.B; p.Hq = s.Hq; p.Hkv = s.Hkv; p.G = s.Hq / s.Hkv; p.Nq = s.Nq; p.Nkv = s.Nkv; p.bq = s.bq;
  p.nqb = n_qblocks(&s); p.nkb = n_kblocks(&s); p.paged = s.paged; p.num_pages = s.num_pages;
  p.page_table = page_table; p.order = order; p.count = count; p.kmax = kmax;
  p.T = cosa_skip_threshold(skip_eps, s.d);
  p.scale_ln = (float)(1.0 / std::sqrt((double)s.d));
  p.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)s.d));
  p.out = static_cast<uint16_t*>(out); p.lse = lse; p.skip_bits = skip_bits; p.skip_words = cdiv(kmax, 32);
  p.status = dev_status;
  p.kv_tail = s.Nkv % s.bk;
  p.wait_limit_ns = wait_limit_ns;
  p.stall_test = stall_test;
  if (group) return launch_status(launch_osk_group(tm_q, tm_k, tm_v, p, s.bk, stream));
  return launch_status(launch_osk(tm_q, tm_k, tm_v, p, s.bk, stream));
}

}  // namespace

extern "C" {

cosa_status cosa_attend(const cosa_shape* shape, const void* q, const void* k, const void* v,
                        const int32_t* page_table, const int32_t* order, const int32_t* count, int kmax,
                        double skip_eps, void* out, float* lse, uint32_t* skip_bits, uint32_t* dev_status,
                        cudaStream_t stream) {
  return attend_impl(shape, q, k, v, page_table, order, count, kmax, skip_eps, out, lse, skip_bits, dev_status,
                     1000000000ull, 0, false, stream);
}

cosa_status cosa_attend_group(const cosa_shape* shape, const void* q, const void* k, const void* v,
                              const int32_t* page_table, const int32_t* order, const int32_t* count, int kmax,
                              double skip_eps, void* out, float* lse, uint32_t* skip_bits, uint32_t* dev_status,
                              cudaStream_t stream) {
  cosa_status st = check_shape(shape);
  if (st != COSA_OK) return st;
  const int G = shape->Hq / shape->Hkv;
  // one query head per group: the group's order is the head's order
  if (G == 1)
    return attend_impl(shape, q, k, v, page_table, order, count, kmax, skip_eps, out, lse, skip_bits, dev_status,
                       1000000000ull, 0, false, stream);
  if (G % 2) return COSA_EUNSUPPORTED;
  return attend_impl(shape, q, k, v, page_table, order, count, kmax, skip_eps, out, lse, skip_bits, dev_status,
                     1000000000ull, 0, true, stream);
}

cosa_status cosa_test_attend_wait_timeout(const cosa_shape* shape, const void* q, const void* k, const void* v,
                                          const int32_t* page_table, const int32_t* order, const int32_t* count,
                                          int kmax, void* out, uint32_t* dev_status, uint64_t wait_limit_ns,
                                          cudaStream_t stream) {
  if (!dev_status || wait_limit_ns < 1000ull || wait_limit_ns > 1000000000ull) return COSA_EINVAL;
  return attend_impl(shape, q, k, v, page_table, order, count, kmax, 0.0, out, nullptr, nullptr, dev_status,
                     wait_limit_ns, 1, false, stream);
}

const char* cosa_status_string(cosa_status status) {
  switch (status) {
    case COSA_OK: return "COSA_OK";
    case COSA_EINVAL: return "COSA_EINVAL: null required pointer or parameter out of range";
    case COSA_EALIGN: return "COSA_EALIGN: tensor pointer not 16-byte aligned (workspace: 256-byte)";
    case COSA_ESHAPE: return "COSA_ESHAPE: inconsistent shape";
    case COSA_EWORKSPACE: return "COSA_EWORKSPACE: workspace missing or too small";
    case COSA_ECUDA: return "COSA_ECUDA: CUDA call or kernel launch failed";
    case COSA_EUNSUPPORTED: return "COSA_EUNSUPPORTED: shape outside what the kernels implement";
  }
  return "COSA: unknown status";
}

int cosa_version(void) { return 101; }

}  // extern "C"
