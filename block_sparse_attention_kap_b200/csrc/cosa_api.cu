// Host front end of the C ABI declared in include/cosa.h: argument
// validation, workspace carving, TMA tensor-map encoding and kernel launch.
// No device memory is allocated here; every launch goes to the caller's
// stream.
#include <cudaTypedefs.h>
#include <cmath>
#include <cstring>
#include <mutex>

#include "cosa.h"
#include "internal.h"

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

struct Workspace {
  size_t qp, kp, rank, bs, total;
};

Workspace carve(const cosa_shape* s) {
  Workspace w;
  const long long rows_q = std::max<long long>((long long)s->B * s->Hq * (s->Nq / s->stride), 0) + 128;
  const long long rows_k = std::max<long long>((long long)s->B * s->Hkv * (s->Nkv / s->stride), 0) + 128;
  w.qp = 0;
  w.kp = align256(w.qp + (size_t)rows_q * kD * 2);
  w.rank = align256(w.kp + (size_t)rows_k * kD * 2);
  w.bs = align256(w.rank + (size_t)s->B * s->Hq * n_qblocks(s) * n_kblocks(s) * sizeof(float));
  const size_t row_tiles = (size_t)cdiv(s->Nq / s->stride, kTileRows);
  w.total = align256(w.bs + (size_t)s->B * s->Hq * row_tiles * n_kblocks(s) * kTileRows * sizeof(float));
  return w;
}

cosa_status launch_status(cudaError_t e) { return e == cudaSuccess ? COSA_OK : COSA_ECUDA; }

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
  cosa_status st = check_plan_shape(shape);
  if (st != COSA_OK) return st;
  if (!(budget > 0.0) || budget > 1.0) return COSA_EINVAL;
  const cosa_shape& s = *shape;
  const long long rows = (long long)s.B * s.Hq * n_qblocks(&s);
  if (rows == 0) return COSA_OK;
  if (!q || !k || !order || !count || (s.paged && !page_table)) return COSA_EINVAL;
  if (!aligned16(q) || !aligned16(k)) return COSA_EALIGN;
  if (kmax < cosa_kmax(&s, budget)) return COSA_EINVAL;
  const Workspace w = carve(&s);
  if (!workspace || ws_bytes < w.total) return COSA_EWORKSPACE;
  if (reinterpret_cast<uintptr_t>(workspace) & 255) return COSA_EALIGN;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  uint16_t* qp = reinterpret_cast<uint16_t*>(ws + w.qp);
  uint16_t* kp = reinterpret_cast<uint16_t*>(ws + w.kp);
  float* rank = reinterpret_cast<float*>(ws + w.rank);
  float* bs = reinterpret_cast<float*>(ws + w.bs);
  const int str = s.stride;

  PoolParams pp;
  pp.q = static_cast<const uint16_t*>(q);
  pp.k = static_cast<const uint16_t*>(k);
  pp.page_table = page_table;
  pp.qp = qp;
  pp.kp = kp;
  pp.B = s.B; pp.Hq = s.Hq; pp.Hkv = s.Hkv; pp.Nq = s.Nq; pp.Nkv = s.Nkv; pp.s = str; pp.bk = s.bk;
  pp.nkb = n_kblocks(&s); pp.paged = s.paged; pp.num_pages = s.num_pages;
  pp.q_items = (long long)s.B * s.Hq * (s.Nq / str);
  pp.k_items = (long long)s.B * s.Hkv * (s.Nkv / str);
  if ((st = launch_status(launch_kap_pool(pp, stream))) != COSA_OK) return st;

  CUtensorMap tm_qp, tm_kp;
  if ((st = make_map(&tm_qp, qp, pp.q_items + 128, 128)) != COSA_OK) return st;
  if ((st = make_map(&tm_kp, kp, pp.k_items + 128, 128)) != COSA_OK) return st;
  ScoreParams sp;
  sp.B = s.B; sp.Hq = s.Hq; sp.Hkv = s.Hkv; sp.G = s.Hq / s.Hkv;
  sp.nqp = s.Nq / str; sp.nkp = s.Nkv / str; sp.off_p = (s.Nkv - s.Nq) / str;
  sp.Nq = s.Nq; sp.Nkv = s.Nkv; sp.bq = s.bq; sp.bk = s.bk; sp.s = str;
  sp.nqb = n_qblocks(&s); sp.nkb = n_kblocks(&s);
  sp.kpb = s.bk / str; sp.rpq = s.bq / str;
  sp.n_row_tiles = cdiv(sp.nqp, kTileRows);
  sp.rank = rank; sp.bs = bs; sp.block_score = block_score; sp.hrm_flags = hrm_flags; sp.status = dev_status;
  if ((st = launch_status(launch_kap_score(tm_qp, tm_kp, sp, stream))) != COSA_OK) return st;

  SortParams so;
  so.B = s.B; so.Hq = s.Hq; so.nqb = sp.nqb; so.nkb = sp.nkb; so.Nq = s.Nq; so.Nkv = s.Nkv;
  so.bq = s.bq; so.bk = s.bk; so.bp = budget_bp(budget); so.kmax = kmax;
  so.rank = rank; so.order = order; so.count = count; so.hrm_count = hrm_count;
  so.block_score = block_score; so.hrm_flags = hrm_flags;
  return launch_status(launch_kap_sort(so, stream));
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

cosa_status cosa_attend(const cosa_shape* shape, const void* q, const void* k, const void* v,
                        const int32_t* page_table, const int32_t* order, const int32_t* count, int kmax,
                        double skip_eps, void* out, float* lse, uint32_t* skip_bits, uint32_t* dev_status,
                        cudaStream_t stream) {
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
  return launch_status(launch_osk(tm_q, tm_k, tm_v, p, s.bk, stream));
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

int cosa_version(void) { return 100; }

}  // extern "C"
