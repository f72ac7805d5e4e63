// api.cu -- the C ABI of libsattn.so: argument validation, workspace layout,
// tensor-map encoding and the launch sequence of each entry point.
//
// The library never allocates.  Each entry point carves its scratch out of
// the caller's workspace with the layout computed by plan_fwd / plan_seg,
// the same functions the *_workspace_size queries call.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <cstring>
#include <map>
#include <mutex>
#include <string>
#include <vector>

#include "../../include/sattn.h"
#include "kernels.cuh"
#include "prof.cuh"
#include "status.cuh"

using namespace sattn;

namespace {

constexpr int kVersion = 10000;  // 1.0.0

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

struct Region {
  size_t off = 0, bytes = 0;
};

struct FwdPlan {
  bool bf16 = true;
  int nQT = 0, Tpad = 0, npos = 0, n_sink = 0;
  bool need_qc = false, capped_sep = false;
  Region status, tab, qr, kr, qc, sink, kmax, prefix, sep_pos, sep_count, ranges, ks, vs, tk_idx, tk_z, fb,
      cand_idx, cand_thr, cand_cnt;
  size_t total = 0;
};

struct Alloc {
  size_t cur = 0;
  Region take(size_t bytes) {
    Region r;
    r.off = cur;
    r.bytes = bytes;
    cur = align256(cur + bytes);
    return r;
  }
};

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// bf16 with separators, a cap and a window below it: separators with
// w < i - j <= L are uncapped and go through the band tiles (which then
// reach back to i - L), those with i - j > L through the compacted capped
// tiles, so the block map's separator ranges are taken at distance L
bool sep_band_extended(const sattn_params* p) {
  return p->dtype == SATTN_DTYPE_BF16 && p->with_separators && p->L_pretrain > 0 && p->window < p->L_pretrain;
}
int sep_split_of(const sattn_params* p) { return sep_band_extended(p) ? p->L_pretrain : p->window; }

int check_common(const sattn_params* p) {
  if (!p) return SATTN_ERR_INVALID_ARG;
  if (p->B < 1 || p->Hq < 1 || p->Hkv < 1 || p->T < 1) return SATTN_ERR_INVALID_ARG;
  if (p->Hq % p->Hkv) return SATTN_ERR_INVALID_ARG;
  if (p->d != 64 && p->d != 128) return SATTN_ERR_UNSUPPORTED;
  if ((p->tile_m != 0 && p->tile_m != kTile) || (p->tile_n != 0 && p->tile_n != kTile)) return SATTN_ERR_UNSUPPORTED;
  if (p->dtype != SATTN_DTYPE_BF16 && p->dtype != SATTN_DTYPE_F32) return SATTN_ERR_INVALID_ARG;
  if (p->n_start < 0 || p->window < 0 || p->L_pretrain < 0 || p->topk < 0) return SATTN_ERR_INVALID_ARG;
  if (p->topk > 16) return SATTN_ERR_UNSUPPORTED;
  if (!(p->rope_theta >= 0.0) || !std::isfinite(p->rope_theta)) return SATTN_ERR_INVALID_ARG;
  if (!(p->rope_pos_scale >= 0.0) || p->rope_pos_scale > 1.0) return SATTN_ERR_INVALID_ARG;
  if (p->alibi && p->rope_theta != 0.0) return SATTN_ERR_INVALID_ARG;  // ALiBi replaces the rotation
  if ((int64_t)p->B * p->Hq * p->T > (int64_t)1 << 31) return SATTN_ERR_UNSUPPORTED;
  const int64_t* st[4] = {p->q_stride, p->k_stride, p->v_stride, p->o_stride};
  const int esz = p->dtype == SATTN_DTYPE_BF16 ? 2 : 4;
  for (int x = 0; x < 4; ++x) {
    for (int y = 0; y < 3; ++y)
      if (st[x][y] < 0) return SATTN_ERR_INVALID_ARG;
    if (st[x][2] < p->d && p->T > 1) return SATTN_ERR_INVALID_ARG;
    if (p->dtype == SATTN_DTYPE_BF16 && ((st[x][0] * esz) % 16 || (st[x][1] * esz) % 16 || (st[x][2] * esz) % 16))
      return SATTN_ERR_INVALID_ARG;
  }
  return SATTN_OK;
}

int check_fwd_rules(const sattn_params* p) {
  int rc = check_common(p);
  if (rc) return rc;
  // an unclipped ALiBi bias would change the top-k ranking and make the bias
  // of a gathered separator depend on its position: not supported
  if (p->alibi && p->L_pretrain == 0 && (p->topk > 0 || (p->with_separators && p->dtype == SATTN_DTYPE_BF16)))
    return SATTN_ERR_UNSUPPORTED;
  // top-k ranks by q.k; with ALiBi that is the logit's order only when every
  // candidate (i - j > window) is past the cap
  if (p->alibi && p->topk > 0 && p->window < p->L_pretrain) return SATTN_ERR_UNSUPPORTED;
  if (p->dtype == SATTN_DTYPE_BF16) {
    if (p->n_start > 256) return SATTN_ERR_UNSUPPORTED;
    if (p->L_pretrain > 0 && p->window > p->L_pretrain) return SATTN_ERR_UNSUPPORTED;
    if (p->Hq > 65535) return SATTN_ERR_UNSUPPORTED;
  }
  return SATTN_OK;
}

int plan_fwd(const sattn_params* p, FwdPlan* pl) {
  int rc = check_fwd_rules(p);
  if (rc) return rc;
  FwdPlan P;
  P.bf16 = p->dtype == SATTN_DTYPE_BF16;
  P.nQT = (p->T + kTile - 1) / kTile;
  P.Tpad = P.nQT * kTile;
  P.npos = std::max(p->T, p->L_pretrain + 1);
  P.n_sink = std::min(p->n_start, p->T);
  P.capped_sep = p->L_pretrain > 0;
  P.need_qc = P.bf16 && p->L_pretrain > 0 && (p->with_separators || p->topk > 0);
  const size_t B = p->B, Hq = p->Hq, Hkv = p->Hkv, T = p->T, d = p->d;
  Alloc A;
  P.status = A.take(kStatusBytes);
  if (p->rope_theta != 0.0) P.tab = A.take((size_t)P.npos * (d / 2) * sizeof(float2));
  P.prefix = A.take(blockmap_scratch_bytes(p->B, p->T, std::max(p->window, sep_split_of(p))));
  if (P.bf16) {
    P.qr = A.take(B * Hq * T * d * 2);
    P.kr = A.take(B * Hkv * T * d * 2);
    if (P.need_qc) P.qc = A.take(B * Hq * T * d * 2);
    if (P.n_sink > 0) P.sink = A.take(B * Hq * T * P.n_sink * 4);
  }
  if (p->with_separators) {
    P.sep_pos = A.take(B * T * 4);
    P.sep_count = A.take(B * 4);
    P.ranges = A.take(B * P.nQT * 2 * 4);
    if (P.bf16) {
      P.ks = A.take(B * Hkv * P.Tpad * d * 2);
      P.vs = A.take(B * Hkv * P.Tpad * d * 2);
    }
  }
  if (p->topk > 0) {
    P.tk_idx = A.take(B * Hq * T * p->topk * 4);
    P.tk_z = A.take(B * Hq * T * p->topk * 4);
    if (P.bf16) {
      P.kmax = A.take(B * Hkv * 4);
      P.fb = A.take(B * Hq * T * 4);
      P.cand_idx = A.take(B * Hq * T * kCandCap * 8);
      P.cand_thr = A.take(B * Hq * T * 4);
      P.cand_cnt = A.take(B * Hq * T * 4);
    }
  }
  P.total = A.cur;
  *pl = P;
  return SATTN_OK;
}

template <typename T>
T* at(void* ws, const Region& r) {
  return r.bytes ? reinterpret_cast<T*>(static_cast<uint8_t*>(ws) + r.off) : nullptr;
}

// ---------------------------------------------------------------------------
// tensor maps
// ---------------------------------------------------------------------------

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

PFN_cuTensorMapEncodeTiled_v12000 encoder() {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  return g_encode;
}

// bf16 [n3][n2][rows][d] with element strides (s3, s2, srow); box 64 x 128,
// 128-byte swizzle, zero fill outside the tensor.
bool make_map(CUtensorMap* m, const void* base, int d, int64_t rows, int64_t n2, int64_t n3, int64_t srow,
              int64_t s2, int64_t s3) {
  auto enc = encoder();
  if (!enc) return false;
  // strides of size-1 dimensions are never used; keep them legal
  if (n2 == 1) s2 = srow * rows;
  if (n3 == 1) s3 = s2 * n2;
  cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)rows, (cuuint64_t)n2, (cuuint64_t)n3};
  cuuint64_t strides[3] = {(cuuint64_t)srow * 2, (cuuint64_t)s2 * 2, (cuuint64_t)s3 * 2};
  for (int x = 0; x < 3; ++x)
    if (strides[x] == 0 || strides[x] % 16) return false;
  cuuint32_t box[4] = {64, (cuuint32_t)kTile, 1, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

int cuda_rc(cudaError_t e) { return e == cudaSuccess ? SATTN_OK : SATTN_ERR_CUDA; }

// rotary position scale (position interpolation); 0 means none
double pos_scale(const sattn_params* p) { return p->rope_pos_scale > 0.0 ? p->rope_pos_scale : 1.0; }

// ---------------------------------------------------------------------------
// optional event instrumentation of launch groups
// ---------------------------------------------------------------------------

struct ProfRec {
  const char* name;
  int kernels;
  cudaEvent_t a, b;
};

std::mutex g_prof_mu;
bool g_prof_on = false;
std::vector<ProfRec> g_prof_recs;
std::vector<cudaEvent_t> g_prof_pool;

cudaEvent_t prof_event() {
  {
    std::lock_guard<std::mutex> g(g_prof_mu);
    if (!g_prof_pool.empty()) {
      cudaEvent_t e = g_prof_pool.back();
      g_prof_pool.pop_back();
      return e;
    }
  }
  cudaEvent_t e = nullptr;
  cudaEventCreate(&e);
  return e;
}

}  // namespace

sattn::ProfScope::ProfScope(const char* name, int kernels, cudaStream_t st) : st_(st) {
  if (!g_prof_on) return;
  name_ = name;
  kernels_ = kernels;
  a_ = prof_event();
  b_ = prof_event();
  active_ = a_ && b_ && cudaEventRecord(a_, st_) == cudaSuccess;
}

sattn::ProfScope::~ProfScope() {
  if (!active_) return;
  if (cudaEventRecord(b_, st_) == cudaSuccess) {
    std::lock_guard<std::mutex> g(g_prof_mu);
    g_prof_recs.push_back(ProfRec{name_, kernels_, a_, b_});
  }
}

namespace {

#define SATTN_TRY(expr)                   \
  do {                                    \
    int _rc = cuda_rc(expr);              \
    if (_rc != SATTN_OK) return _rc;      \
  } while (0)

// ---------------------------------------------------------------------------
// shared launch steps
// ---------------------------------------------------------------------------

int run_prep_bf16(const sattn_params* p, const FwdPlan& P, const void* Q, const void* K, void* ws, bool with_sinks,
                  bool with_kmax, cudaStream_t st) {
  if (P.tab.bytes) {
    ProfScope ps("rope_table", 1, st);
    SATTN_TRY(launch_rope_table(at<float2>(ws, P.tab), P.npos, p->d, p->rope_theta, pos_scale(p), st));
  }
  if (with_kmax && P.kmax.bytes) SATTN_TRY(cudaMemsetAsync(at<uint8_t>(ws, P.kmax), 0, P.kmax.bytes, st));
  PrepArgs a{};
  a.B = p->B;
  a.Hq = p->Hq;
  a.Hkv = p->Hkv;
  a.T = p->T;
  a.d = p->d;
  a.Q = Q;
  a.K = K;
  a.q_sb = p->q_stride[0];
  a.q_sh = p->q_stride[1];
  a.q_st = p->q_stride[2];
  a.k_sb = p->k_stride[0];
  a.k_sh = p->k_stride[1];
  a.k_st = p->k_stride[2];
  a.f32 = false;
  a.tab = at<float2>(ws, P.tab);
  a.L = p->L_pretrain;
  a.Qr = at<__nv_bfloat16>(ws, P.qr);
  a.Qc = at<__nv_bfloat16>(ws, P.qc);
  a.Kr = at<__nv_bfloat16>(ws, P.kr);
  a.sink_z = with_sinks ? at<float>(ws, P.sink) : nullptr;
  a.n_sink = with_sinks ? P.n_sink : 0;
  a.alibi = p->alibi ? 1 : 0;
  a.kmax = with_kmax ? at<uint32_t>(ws, P.kmax) : nullptr;
  ProfScope ps("prep_rope", 1, st);
  return cuda_rc(launch_prep(a, st));
}

int run_blockmap(const sattn_params* p, const FwdPlan& P, const uint8_t* is_sep, uint8_t* cls, int32_t* sep_pos,
                 int32_t* sep_count, int32_t* ranges, void* ws, cudaStream_t st, int window = -1) {
  BlockmapArgs a{};
  a.B = p->B;
  a.T = p->T;
  a.n_start = p->n_start;
  a.window = window >= 0 ? window : p->window;
  a.is_sep = is_sep;
  a.scratch = at<uint8_t>(ws, P.prefix);
  a.sep_pos = sep_pos;
  a.sep_count = sep_count;
  a.ranges = ranges;
  a.cls = cls;
  ProfScope ps("blockmap", cls ? 2 : 1, st);  // the class kernel runs only when classes are asked for
  return cuda_rc(launch_blockmap(a, st));
}

TopkArgs topk_args(const sattn_params* p, const FwdPlan& P, const void* Q, const void* K, const uint8_t* is_sep,
                   int32_t* idx, float* z, void* ws) {
  TopkArgs a{};
  a.B = p->B;
  a.Hq = p->Hq;
  a.Hkv = p->Hkv;
  a.T = p->T;
  a.d = p->d;
  a.nQT = P.nQT;
  a.n_start = p->n_start;
  a.window = p->window;
  a.topk = p->topk;
  a.L = p->L_pretrain;
  a.is_sep = is_sep;
  a.Q = Q;
  a.K = K;
  a.f32 = !P.bf16;
  a.q_sb = p->q_stride[0];
  a.q_sh = p->q_stride[1];
  a.q_st = p->q_stride[2];
  a.k_sb = p->k_stride[0];
  a.k_sh = p->k_stride[1];
  a.k_st = p->k_stride[2];
  a.tab = at<float2>(ws, P.tab);
  a.kmax = at<uint32_t>(ws, P.kmax);
  a.idx = idx;
  a.z = z;
  a.fallback_rows = at<int32_t>(ws, P.fb);
  a.status = at<int32_t>(ws, P.status);
  a.cand_idx = at<int2>(ws, P.cand_idx);
  a.cand_thr = at<float>(ws, P.cand_thr);
  a.cand_cnt = at<int32_t>(ws, P.cand_cnt);
  return a;
}

// selection into (idx, z); prep must have run (bf16)
int run_topk(const sattn_params* p, const FwdPlan& P, const void* Q, const void* K, const uint8_t* is_sep,
             int32_t* idx, float* z, void* ws, cudaStream_t st) {
  TopkArgs a = topk_args(p, P, Q, K, is_sep, idx, z, ws);
  if (!P.bf16) {
    if (P.tab.bytes) SATTN_TRY(launch_rope_table(at<float2>(ws, P.tab), P.npos, p->d, p->rope_theta, pos_scale(p), st));
    ProfScope ps("topk_exact", 1, st);
    return cuda_rc(launch_topk_exact(a, true, st));
  }
  TopkMaps m;
  const size_t B = p->B, Hq = p->Hq, Hkv = p->Hkv, T = p->T, d = p->d;
  // uncapped operands (R(i) q, R(j) k): the only pair when L = 0, the pair of
  // the candidates within the cap when 0 < w < L
  if (!make_map(&m.qsel2, at<void>(ws, P.qr), p->d, p->T, Hq, B, d, T * d, Hq * T * d)) return SATTN_ERR_CUDA;
  if (!make_map(&m.ksel2, at<void>(ws, P.kr), p->d, p->T, Hkv, B, d, T * d, Hkv * T * d)) return SATTN_ERR_CUDA;
  if (p->L_pretrain > 0) {
    if (!make_map(&m.qsel, at<void>(ws, P.qc), p->d, p->T, Hq, B, d, T * d, Hq * T * d)) return SATTN_ERR_CUDA;
    if (!make_map(&m.ksel, K, p->d, p->T, Hkv, B, p->k_stride[2], p->k_stride[1], p->k_stride[0]))
      return SATTN_ERR_CUDA;
  } else {
    m.qsel = m.qsel2;
    m.ksel = m.ksel2;
  }
  {
    ProfScope ps("topk_score", 1, st);
    SATTN_TRY(launch_topk_score(a, m, st));
  }
  {
    ProfScope ps("topk_rerank", 1, st);
    SATTN_TRY(launch_topk_rerank(a, st));
  }
  ProfScope ps("topk_exact", 1, st);
  return cuda_rc(launch_topk_exact(a, false, st));
}

bool pointers_ok_bf16(const void* a, const void* b, const void* c) {
  return aligned16(a) && aligned16(b) && aligned16(c);
}

}  // namespace

// ===========================================================================
// exported
// ===========================================================================

extern "C" {

const char* sattn_strerror(int status) {
  switch (status) {
    case SATTN_OK: return "ok";
    case SATTN_ERR_INVALID_ARG: return "invalid argument";
    case SATTN_ERR_UNSUPPORTED: return "unsupported parameters";
    case SATTN_ERR_CUDA: return "CUDA error";
    case SATTN_ERR_TIMEOUT: return "device-side wait timed out";
    default: return "unknown status";
  }
}

int sattn_version(void) { return kVersion; }

int sattn_workspace_size(const sattn_params* p, size_t* bytes) {
  if (!bytes) return SATTN_ERR_INVALID_ARG;
  FwdPlan P;
  int rc = plan_fwd(p, &P);
  if (rc) return rc;
  *bytes = P.total;
  return SATTN_OK;
}

int sattn_build_blockmap(const sattn_params* p, const uint8_t* is_sep, uint8_t* cls, int32_t* sep_pos,
                         int32_t* sep_count, int32_t* qtile_sep_range, void* ws, size_t ws_bytes, void* stream) {
  FwdPlan P;
  int rc = plan_fwd(p, &P);
  if (rc) return rc;
  if (!ws || ws_bytes < P.total || (reinterpret_cast<uintptr_t>(ws) & 255u)) return SATTN_ERR_INVALID_ARG;
  if (!sep_pos || !sep_count || !qtile_sep_range) return SATTN_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  SATTN_TRY(cudaMemsetAsync(ws, 0, kStatusBytes, st));
  return run_blockmap(p, P, is_sep, cls, sep_pos, sep_count, qtile_sep_range, ws, st);
}

int sattn_topk_select(const sattn_params* p, const void* Q, const void* K, const uint8_t* is_sep, int32_t* idx,
                      float* logit, void* ws, size_t ws_bytes, void* stream) {
  FwdPlan P;
  int rc = plan_fwd(p, &P);
  if (rc) return rc;
  if (p->topk < 1 || !Q || !K || !idx || !logit) return SATTN_ERR_INVALID_ARG;
  if (is_sep && !p->with_separators) return SATTN_ERR_INVALID_ARG;
  if (!ws || ws_bytes < P.total || (reinterpret_cast<uintptr_t>(ws) & 255u)) return SATTN_ERR_INVALID_ARG;
  if (P.bf16 && !pointers_ok_bf16(Q, K, K)) return SATTN_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  SATTN_TRY(cudaMemsetAsync(ws, 0, kStatusBytes, st));
  if (P.bf16) {
    rc = run_prep_bf16(p, P, Q, K, ws, false, true, st);
    if (rc) return rc;
  }
  return run_topk(p, P, Q, K, is_sep, idx, logit, ws, st);
}

int sattn_fwd(const sattn_params* p, const void* Q, const void* K, const void* V, const uint8_t* is_sep,
              const int32_t* topk_idx, const float* topk_logit, void* O, float* lse, void* ws, size_t ws_bytes,
              void* stream) {
  FwdPlan P;
  int rc = plan_fwd(p, &P);
  if (rc) return rc;
  if (!Q || !K || !V || !O || !lse) return SATTN_ERR_INVALID_ARG;
  if (is_sep && !p->with_separators) return SATTN_ERR_INVALID_ARG;
  if ((topk_idx == nullptr) != (topk_logit == nullptr)) return SATTN_ERR_INVALID_ARG;
  if (!ws || ws_bytes < P.total || (reinterpret_cast<uintptr_t>(ws) & 255u)) return SATTN_ERR_INVALID_ARG;
  if (P.bf16 && (!pointers_ok_bf16(Q, K, V) || !aligned16(O))) return SATTN_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t B = p->B, Hq = p->Hq, Hkv = p->Hkv, T = p->T, d = p->d;
  SATTN_TRY(cudaMemsetAsync(ws, 0, kStatusBytes, st));

  int32_t* sep_pos = at<int32_t>(ws, P.sep_pos);
  int32_t* sep_count = at<int32_t>(ws, P.sep_count);
  int32_t* ranges = at<int32_t>(ws, P.ranges);
  const int32_t* tki = topk_idx;
  const float* tkz = topk_logit;

  if (!P.bf16) {
    // ---------------- fp32 path ----------------
    if (P.tab.bytes) {
      ProfScope ps("rope_table", 1, st);
      SATTN_TRY(launch_rope_table(at<float2>(ws, P.tab), P.npos, p->d, p->rope_theta, pos_scale(p), st));
    }
    if (is_sep) {
      rc = run_blockmap(p, P, is_sep, nullptr, sep_pos, sep_count, ranges, ws, st);
      if (rc) return rc;
    }
    if (p->topk > 0 && !tki) {
      TopkArgs ta = topk_args(p, P, Q, K, is_sep, at<int32_t>(ws, P.tk_idx), at<float>(ws, P.tk_z), ws);
      {
        ProfScope ps("topk_exact", 1, st);
        SATTN_TRY(launch_topk_exact(ta, true, st));
      }
      tki = at<int32_t>(ws, P.tk_idx);
      tkz = at<float>(ws, P.tk_z);
    }
    AttnF32Args a{};
    a.B = p->B;
    a.Hq = p->Hq;
    a.Hkv = p->Hkv;
    a.T = p->T;
    a.d = p->d;
    a.Q = static_cast<const float*>(Q);
    a.K = static_cast<const float*>(K);
    a.V = static_cast<const float*>(V);
    a.q_sb = p->q_stride[0];
    a.q_sh = p->q_stride[1];
    a.q_st = p->q_stride[2];
    a.k_sb = p->k_stride[0];
    a.k_sh = p->k_stride[1];
    a.k_st = p->k_stride[2];
    a.v_sb = p->v_stride[0];
    a.v_sh = p->v_stride[1];
    a.v_st = p->v_stride[2];
    a.tab = at<float2>(ws, P.tab);
    a.L = p->L_pretrain;
    a.alibi = p->alibi ? 1 : 0;
    a.n_start = p->n_start;
    a.window = p->window;
    a.sep_pos = is_sep ? sep_pos : nullptr;
    a.sep_count = sep_count;
    a.tk_idx = p->topk > 0 ? tki : nullptr;
    a.tk_z = tkz;
    a.topk = p->topk;
    a.O = static_cast<float*>(O);
    a.o_sb = p->o_stride[0];
    a.o_sh = p->o_stride[1];
    a.o_st = p->o_stride[2];
    a.lse = lse;
    ProfScope ps("attn_f32", 1, st);
    return cuda_rc(launch_attn_f32(a, st));
  }

  // ---------------- bf16 tensor-core path ----------------
  rc = run_prep_bf16(p, P, Q, K, ws, true, p->topk > 0 && !tki, st);
  if (rc) return rc;
  AttnMaps m;
  if (!make_map(&m.q, at<void>(ws, P.qr), p->d, p->T, Hq, B, d, T * d, Hq * T * d)) return SATTN_ERR_CUDA;
  if (!make_map(&m.k, at<void>(ws, P.kr), p->d, p->T, Hkv, B, d, T * d, Hkv * T * d)) return SATTN_ERR_CUDA;
  if (!make_map(&m.v, V, p->d, p->T, Hkv, B, p->v_stride[2], p->v_stride[1], p->v_stride[0])) return SATTN_ERR_CUDA;
  m.q2 = m.q;
  m.kg = m.k;
  m.vg = m.v;
  bool q2 = false;
  if (is_sep) {
    rc = run_blockmap(p, P, is_sep, nullptr, sep_pos, sep_count, ranges, ws, st, sep_split_of(p));
    if (rc) return rc;
    GatherArgs ga{};
    ga.B = p->B;
    ga.Hkv = p->Hkv;
    ga.T = p->T;
    ga.Tpad = P.Tpad;
    ga.d = p->d;
    if (P.capped_sep) {
      ga.Ksrc = static_cast<const __nv_bfloat16*>(K);
      ga.k_sb = p->k_stride[0];
      ga.k_sh = p->k_stride[1];
      ga.k_st = p->k_stride[2];
      q2 = true;
      if (!make_map(&m.q2, at<void>(ws, P.qc), p->d, p->T, Hq, B, d, T * d, Hq * T * d)) return SATTN_ERR_CUDA;
    } else {
      ga.Ksrc = at<__nv_bfloat16>(ws, P.kr);
      ga.k_sb = Hkv * T * d;
      ga.k_sh = T * d;
      ga.k_st = d;
    }
    ga.Vsrc = static_cast<const __nv_bfloat16*>(V);
    ga.v_sb = p->v_stride[0];
    ga.v_sh = p->v_stride[1];
    ga.v_st = p->v_stride[2];
    ga.sep_pos = sep_pos;
    ga.sep_count = sep_count;
    ga.Ks = at<__nv_bfloat16>(ws, P.ks);
    ga.Vs = at<__nv_bfloat16>(ws, P.vs);
    {
      ProfScope ps("sep_gather", 1, st);
      SATTN_TRY(launch_sep_gather(ga, st));
    }
    if (!make_map(&m.kg, ga.Ks, p->d, P.Tpad, Hkv, B, d, (int64_t)P.Tpad * d, Hkv * P.Tpad * d)) return SATTN_ERR_CUDA;
    if (!make_map(&m.vg, ga.Vs, p->d, P.Tpad, Hkv, B, d, (int64_t)P.Tpad * d, Hkv * P.Tpad * d)) return SATTN_ERR_CUDA;
  }
  if (p->topk > 0 && !tki) {
    rc = run_topk(p, P, Q, K, is_sep, at<int32_t>(ws, P.tk_idx), at<float>(ws, P.tk_z), ws, st);
    if (rc) return rc;
    tki = at<int32_t>(ws, P.tk_idx);
    tkz = at<float>(ws, P.tk_z);
  }
  AttnArgs a{};
  a.B = p->B;
  a.Hq = p->Hq;
  a.Hkv = p->Hkv;
  a.T = p->T;
  a.d = p->d;
  a.nQT = P.nQT;
  a.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)p->d));
  a.alibi = p->alibi ? 1 : 0;
  a.alibi_cap = p->L_pretrain;
  a.ns_band = p->n_start;
  a.w_eff = p->window;
  a.sink_z = at<float>(ws, P.sink);
  a.n_sink = P.n_sink;
  a.tk_idx = p->topk > 0 ? tki : nullptr;
  a.tk_z = p->topk > 0 ? tkz : nullptr;
  a.topk = p->topk > 0 ? p->topk : 0;
  a.V = static_cast<const __nv_bfloat16*>(V);
  a.v_sb = p->v_stride[0];
  a.v_sh = p->v_stride[1];
  a.v_st = p->v_stride[2];
  a.gather_mode = is_sep ? 1 : 0;
  a.q2 = q2;
  a.sep_pos = sep_pos;
  a.sep_words = at<uint2>(ws, P.prefix);
  a.ranges = ranges;
  a.window = sep_split_of(p);
  a.w_sepband = (is_sep && sep_band_extended(p)) ? p->L_pretrain : 0;
  for (int h = 0; h < kMaxHeads; ++h) a.long_slot[h] = -1;
  a.O = static_cast<__nv_bfloat16*>(O);
  a.o_sb = p->o_stride[0];
  a.o_sh = p->o_stride[1];
  a.o_st = p->o_stride[2];
  a.lse = lse;
  a.status = at<int32_t>(ws, P.status);
  ProfScope ps("attn_tc", 1, st);
  // capped separator tiles need the second (capped) query tile: one query
  // tile per CTA; otherwise two query tiles per CTA
  return cuda_rc(q2 ? launch_attn_tc3(a, m, st) : launch_attn_tc2(a, m, st));
}

// ---------------------------------------------------------------------------
// segmented execution
// ---------------------------------------------------------------------------

struct SegPlan {
  int nQT, N, Rpad, n_long, npos;
  Region status, tab, qr, kr, kpre, vpre, pcnt, score;
  size_t total;
};

static int plan_seg(const sattn_params* p, int32_t S, int32_t M, int32_t R, int32_t blk, const uint8_t* is_long,
                    SegPlan* out) {
  int rc = check_common(p);
  if (rc) return rc;
  if (p->dtype != SATTN_DTYPE_BF16) return SATTN_ERR_UNSUPPORTED;
  if (p->alibi) return SATTN_ERR_UNSUPPORTED;
  if (S < kTile || S % kTile || p->T % S || M < 0 || R < 0 || blk < 1 || R % blk) return SATTN_ERR_INVALID_ARG;
  if (R / blk > 1024 || p->Hq > kMaxHeads) return SATTN_ERR_UNSUPPORTED;
  if (!segment_retrieval_supported(p->T, S, blk)) return SATTN_ERR_UNSUPPORTED;
  SegPlan P;
  P.nQT = (p->T + kTile - 1) / kTile;
  P.N = p->T / S;
  P.Rpad = (R + kTile - 1) / kTile * kTile;
  P.n_long = 0;
  for (int h = 0; h < p->Hq; ++h) P.n_long += (is_long == nullptr || is_long[h]) ? 1 : 0;
  P.npos = p->T;
  const size_t B = p->B, Hq = p->Hq, Hkv = p->Hkv, T = p->T, d = p->d;
  Alloc A;
  P.status = A.take(kStatusBytes);
  if (p->rope_theta != 0.0) P.tab = A.take((size_t)P.npos * (d / 2) * sizeof(float2));
  P.qr = A.take(B * Hq * T * d * 2);
  P.kr = A.take(B * Hkv * T * d * 2);
  if (P.n_long > 0 && R > 0) {
    P.kpre = A.take(B * P.n_long * P.N * P.Rpad * d * 2);
    P.vpre = A.take(B * P.n_long * P.N * P.Rpad * d * 2);
  }
  P.pcnt = A.take(B * std::max(P.n_long, 1) * P.N * 4);
  if (P.n_long > 0 && R > 0) P.score = A.take(segment_score_bytes(p->B, P.n_long, P.N, p->T, blk));
  P.total = A.cur;
  *out = P;
  return SATTN_OK;
}

int sattn_segment_workspace_size(const sattn_params* p, int32_t S, int32_t M, int32_t R, int32_t retr_block,
                                 const uint8_t* is_long, size_t* bytes) {
  if (!bytes) return SATTN_ERR_INVALID_ARG;
  SegPlan P;
  int rc = plan_seg(p, S, M, R, retr_block, is_long, &P);
  if (rc) return rc;
  *bytes = P.total;
  return SATTN_OK;
}

int sattn_segment_fwd(const sattn_params* p, int32_t S, int32_t M, int32_t R, int32_t retr_block,
                      const uint8_t* is_long, const void* Q, const void* K, const void* V, void* O, float* lse,
                      int32_t* prefix_blocks, void* ws, size_t ws_bytes, void* stream) {
  if (!is_long) return SATTN_ERR_INVALID_ARG;
  SegPlan P;
  int rc = plan_seg(p, S, M, R, retr_block, is_long, &P);
  if (rc) return rc;
  if (!Q || !K || !V || !O || !lse || !prefix_blocks) return SATTN_ERR_INVALID_ARG;
  if (!ws || ws_bytes < P.total || (reinterpret_cast<uintptr_t>(ws) & 255u)) return SATTN_ERR_INVALID_ARG;
  if (!pointers_ok_bf16(Q, K, V) || !aligned16(O)) return SATTN_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t B = p->B, Hq = p->Hq, Hkv = p->Hkv, T = p->T, d = p->d;
  SATTN_TRY(cudaMemsetAsync(ws, 0, kStatusBytes, st));

  // prep: rotate Q and K at their global positions (only distances matter)
  FwdPlan F;
  F.bf16 = true;
  F.npos = P.npos;
  F.tab = P.tab;
  F.qr = P.qr;
  F.kr = P.kr;
  sattn_params pp = *p;
  pp.L_pretrain = 0;
  rc = run_prep_bf16(&pp, F, Q, K, ws, false, false, st);
  if (rc) return rc;

  const int nb = R / retr_block;
  if (nb > 0) SATTN_TRY(cudaMemsetAsync(prefix_blocks, 0xFF, B * Hq * P.N * nb * 4, st));
  SATTN_TRY(cudaMemsetAsync(at<uint8_t>(ws, P.pcnt), 0, P.pcnt.bytes, st));
  AttnArgs a{};
  for (int h = 0; h < kMaxHeads; ++h) a.long_slot[h] = -1;
  SegRetrArgs ra{};
  {
    int slot = 0;
    for (int h = 0; h < p->Hq; ++h)
      if (is_long[h]) {
        a.long_slot[h] = (int16_t)slot;
        ra.long_heads[slot] = (int16_t)h;
        ++slot;
      }
  }
  AttnMaps m;
  if (!make_map(&m.q, at<void>(ws, P.qr), p->d, p->T, Hq, B, d, T * d, Hq * T * d)) return SATTN_ERR_CUDA;
  if (!make_map(&m.k, at<void>(ws, P.kr), p->d, p->T, Hkv, B, d, T * d, Hkv * T * d)) return SATTN_ERR_CUDA;
  if (!make_map(&m.v, V, p->d, p->T, Hkv, B, p->v_stride[2], p->v_stride[1], p->v_stride[0])) return SATTN_ERR_CUDA;
  m.q2 = m.q;
  m.kg = m.k;
  m.vg = m.v;
  if (P.n_long > 0 && R > 0 && P.N > 1) {
    ra.B = p->B;
    ra.Hq = p->Hq;
    ra.Hkv = p->Hkv;
    ra.T = p->T;
    ra.d = p->d;
    ra.S = S;
    ra.N = P.N;
    ra.R = R;
    ra.blk = retr_block;
    ra.n_long = P.n_long;
    ra.s_lo = 1;  // every segment after the first, all of them held
    ra.s_base = 0;
    ra.Q = static_cast<const __nv_bfloat16*>(Q);
    ra.K = static_cast<const __nv_bfloat16*>(K);
    ra.V = static_cast<const __nv_bfloat16*>(V);
    ra.q_sb = p->q_stride[0];
    ra.q_sh = p->q_stride[1];
    ra.q_st = p->q_stride[2];
    ra.k_sb = p->k_stride[0];
    ra.k_sh = p->k_stride[1];
    ra.k_st = p->k_stride[2];
    ra.v_sb = p->v_stride[0];
    ra.v_sh = p->v_stride[1];
    ra.v_st = p->v_stride[2];
    ra.tab = at<float2>(ws, P.tab);
    ra.prefix_blocks = prefix_blocks;
    ra.prefix_cnt = at<int32_t>(ws, P.pcnt);
    ra.Kpre = at<__nv_bfloat16>(ws, P.kpre);
    ra.Vpre = at<__nv_bfloat16>(ws, P.vpre);
    ra.score = at<float>(ws, P.score);
    {
      ProfScope ps("segment_retrieval", 3, st);
      SATTN_TRY(launch_segment_retrieval(ra, st));
    }
    const int64_t planes = (int64_t)P.n_long * P.N;
    if (!make_map(&m.kg, ra.Kpre, p->d, P.Rpad, planes, B, d, (int64_t)P.Rpad * d, planes * P.Rpad * d))
      return SATTN_ERR_CUDA;
    if (!make_map(&m.vg, ra.Vpre, p->d, P.Rpad, planes, B, d, (int64_t)P.Rpad * d, planes * P.Rpad * d))
      return SATTN_ERR_CUDA;
  }
  a.B = p->B;
  a.Hq = p->Hq;
  a.Hkv = p->Hkv;
  a.T = p->T;
  a.d = p->d;
  a.nQT = P.nQT;
  a.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)p->d));
  a.ns_band = 0;
  a.w_eff = 0x3fffffff;
  a.V = static_cast<const __nv_bfloat16*>(V);
  a.v_sb = p->v_stride[0];
  a.v_sh = p->v_stride[1];
  a.v_st = p->v_stride[2];
  a.gather_mode = 2;
  a.q2 = false;
  a.seg_S = S;
  a.seg_M = M;
  a.seg_N = P.N;
  a.seg_R = R;
  a.prefix_cnt = at<int32_t>(ws, P.pcnt);
  a.n_long = std::max(P.n_long, 1);
  a.O = static_cast<__nv_bfloat16*>(O);
  a.o_sb = p->o_stride[0];
  a.o_sh = p->o_stride[1];
  a.o_st = p->o_stride[2];
  a.lse = lse;
  a.status = at<int32_t>(ws, P.status);
  ProfScope ps("attn_tc_segment", 1, st);
  return cuda_rc((S % (2 * kTile) == 0) ? launch_attn_tc2(a, m, st) : launch_attn_tc3(a, m, st));
}

// ---------------------------------------------------------------------------
// segmented execution one segment at a time (explicit carried state)
// ---------------------------------------------------------------------------

// The state of a layer of capacity p->T (a multiple of S): header, rotary
// table of every position, raw K and V and the keys rotated at their
// positions for every position taken, the last segment's last query.
struct SegStateLayout {
  Region header, tab, khist, vhist, krot, qend;
  size_t total = 0;
};

static int seg_stream_rules(const sattn_params* p, int32_t S, int32_t M, int32_t R, int32_t blk) {
  int rc = check_common(p);
  if (rc) return rc;
  if (p->dtype != SATTN_DTYPE_BF16 || p->alibi) return SATTN_ERR_UNSUPPORTED;
  if (S < kTile || S % kTile || p->T % S || M < 0 || R < 0 || blk < 1 || R % blk) return SATTN_ERR_INVALID_ARG;
  if (R / blk > 1024 || p->Hq > kMaxHeads) return SATTN_ERR_UNSUPPORTED;
  if (!segment_retrieval_supported(p->T, S, blk)) return SATTN_ERR_UNSUPPORTED;
  return SATTN_OK;
}

static int seg_state_layout(const sattn_params* p, int32_t S, int32_t M, int32_t R, int32_t blk,
                            SegStateLayout* out) {
  int rc = seg_stream_rules(p, S, M, R, blk);
  if (rc) return rc;
  SegStateLayout L;
  const size_t B = p->B, Hq = p->Hq, Hkv = p->Hkv, T = p->T, d = p->d;
  Alloc A;
  L.header = A.take(256);
  if (p->rope_theta != 0.0) L.tab = A.take(T * (d / 2) * sizeof(float2));
  L.khist = A.take(B * Hkv * T * d * 2);
  L.vhist = A.take(B * Hkv * T * d * 2);
  L.krot = A.take(B * Hkv * T * d * 2);
  L.qend = A.take(B * Hq * d * 2);
  L.total = A.cur;
  *out = L;
  return SATTN_OK;
}

struct SegStepPlan {
  int n_long = 0, Rpad = 0;
  Region status, qr, pcnt, score, kpre, vpre;
  size_t total = 0;
};

static int plan_seg_step(const sattn_params* p, int32_t S, int32_t M, int32_t R, int32_t blk, const uint8_t* is_long,
                         SegStepPlan* out) {
  int rc = seg_stream_rules(p, S, M, R, blk);
  if (rc) return rc;
  SegStepPlan P;
  for (int h = 0; h < p->Hq; ++h) P.n_long += (is_long == nullptr || is_long[h]) ? 1 : 0;
  P.Rpad = (R + kTile - 1) / kTile * kTile;
  const size_t B = p->B, Hq = p->Hq, d = p->d;
  Alloc A;
  P.status = A.take(kStatusBytes);
  P.qr = A.take(B * Hq * (size_t)S * d * 2);
  P.pcnt = A.take(B * std::max(P.n_long, 1) * 4);
  if (P.n_long > 0 && R > 0) {
    P.score = A.take(segment_score_bytes(p->B, P.n_long, 1, p->T, blk));
    P.kpre = A.take(B * P.n_long * (size_t)P.Rpad * d * 2);
    P.vpre = A.take(B * P.n_long * (size_t)P.Rpad * d * 2);
  }
  P.total = A.cur;
  *out = P;
  return SATTN_OK;
}

int sattn_segment_state_size(const sattn_params* p, int32_t S, int32_t M, int32_t R, int32_t retr_block,
                             size_t* bytes) {
  if (!bytes) return SATTN_ERR_INVALID_ARG;
  SegStateLayout L;
  int rc = seg_state_layout(p, S, M, R, retr_block, &L);
  if (rc) return rc;
  *bytes = L.total;
  return SATTN_OK;
}

int sattn_segment_state_reset(const sattn_params* p, int32_t S, int32_t M, int32_t R, int32_t retr_block,
                              void* state, size_t state_bytes, void* stream) {
  SegStateLayout L;
  int rc = seg_state_layout(p, S, M, R, retr_block, &L);
  if (rc) return rc;
  if (!state || state_bytes < L.total || (reinterpret_cast<uintptr_t>(state) & 255u)) return SATTN_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  SATTN_TRY(cudaMemsetAsync(state, 0, L.header.bytes, st));
  SATTN_TRY(launch_segstate_reset(at<int32_t>(state, L.header), S, p->T, st));
  if (L.tab.bytes)
    SATTN_TRY(launch_rope_table(at<float2>(state, L.tab), p->T, p->d, p->rope_theta, pos_scale(p), st));
  return SATTN_OK;
}

int sattn_segment_step_workspace_size(const sattn_params* p, int32_t S, int32_t M, int32_t R, int32_t retr_block,
                                      const uint8_t* is_long, size_t* bytes) {
  if (!bytes) return SATTN_ERR_INVALID_ARG;
  SegStepPlan P;
  int rc = plan_seg_step(p, S, M, R, retr_block, is_long, &P);
  if (rc) return rc;
  *bytes = P.total;
  return SATTN_OK;
}

int sattn_segment_step(const sattn_params* p, int32_t S, int32_t M, int32_t R, int32_t retr_block,
                       const uint8_t* is_long, int32_t seg, const void* Q, const void* K, const void* V, void* state,
                       size_t state_bytes, void* O, float* lse, int32_t* prefix_blocks, void* ws, size_t ws_bytes,
                       void* stream) {
  if (!is_long) return SATTN_ERR_INVALID_ARG;
  SegStateLayout L;
  int rc = seg_state_layout(p, S, M, R, retr_block, &L);
  if (rc) return rc;
  SegStepPlan P;
  rc = plan_seg_step(p, S, M, R, retr_block, is_long, &P);
  if (rc) return rc;
  if (seg < 0 || (int64_t)(seg + 1) * S > p->T) return SATTN_ERR_INVALID_ARG;
  if (!Q || !K || !V || !O || !lse || (R > 0 && !prefix_blocks)) return SATTN_ERR_INVALID_ARG;
  if (!state || state_bytes < L.total || (reinterpret_cast<uintptr_t>(state) & 255u)) return SATTN_ERR_INVALID_ARG;
  if (!ws || ws_bytes < P.total || (reinterpret_cast<uintptr_t>(ws) & 255u)) return SATTN_ERR_INVALID_ARG;
  if (!pointers_ok_bf16(Q, K, V) || !aligned16(O)) return SATTN_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t B = p->B, Hq = p->Hq, Hkv = p->Hkv, Tcap = p->T, d = p->d;
  const int Tnow = (seg + 1) * S;  // positions taken once this segment is in
  SATTN_TRY(cudaMemsetAsync(ws, 0, kStatusBytes, st));
  int32_t* status = at<int32_t>(ws, P.status);

  // 1. the segment joins the history (after checking it is the next one)
  SegStateArgs sa{};
  sa.B = p->B;
  sa.Hq = p->Hq;
  sa.Hkv = p->Hkv;
  sa.d = p->d;
  sa.S = S;
  sa.T_cap = p->T;
  sa.seg = seg;
  sa.header = at<int32_t>(state, L.header);
  sa.Q = static_cast<const __nv_bfloat16*>(Q);
  sa.K = static_cast<const __nv_bfloat16*>(K);
  sa.V = static_cast<const __nv_bfloat16*>(V);
  sa.q_sb = p->q_stride[0];
  sa.q_sh = p->q_stride[1];
  sa.q_st = p->q_stride[2];
  sa.k_sb = p->k_stride[0];
  sa.k_sh = p->k_stride[1];
  sa.k_st = p->k_stride[2];
  sa.v_sb = p->v_stride[0];
  sa.v_sh = p->v_stride[1];
  sa.v_st = p->v_stride[2];
  sa.Khist = at<__nv_bfloat16>(state, L.khist);
  sa.Vhist = at<__nv_bfloat16>(state, L.vhist);
  sa.q_end = at<__nv_bfloat16>(state, L.qend);
  sa.status = status;
  {
    ProfScope ps("segment_state_append", 1, st);
    SATTN_TRY(launch_segstate_append(sa, st));
  }
  // 2. rotation at the global positions: the segment's queries into the
  //    workspace, its keys into the state's rotated history
  {
    PrepArgs pa{};
    pa.B = p->B;
    pa.Hq = p->Hq;
    pa.Hkv = p->Hkv;
    pa.T = S;
    pa.d = p->d;
    pa.Q = Q;
    pa.K = K;
    pa.q_sb = p->q_stride[0];
    pa.q_sh = p->q_stride[1];
    pa.q_st = p->q_stride[2];
    pa.k_sb = p->k_stride[0];
    pa.k_sh = p->k_stride[1];
    pa.k_st = p->k_stride[2];
    pa.tab = L.tab.bytes ? at<float2>(state, L.tab) : nullptr;
    pa.Qr = at<__nv_bfloat16>(ws, P.qr);
    pa.Kr = at<__nv_bfloat16>(state, L.krot);
    pa.pos0 = seg * S;
    pa.kr_rows = p->T;
    pa.kr_row0 = seg * S;
    pa.status = status;
    ProfScope ps("prep_rope", 1, st);
    SATTN_TRY(launch_prep(pa, st));
  }
  // 3. retrieval for the long heads from the pool [0, seg S) with the carried query
  const int nb = R / retr_block;
  if (nb > 0) SATTN_TRY(cudaMemsetAsync(prefix_blocks, 0xFF, B * Hq * nb * 4, st));
  SATTN_TRY(cudaMemsetAsync(at<uint8_t>(ws, P.pcnt), 0, P.pcnt.bytes, st));
  AttnArgs a{};
  for (int h = 0; h < kMaxHeads; ++h) a.long_slot[h] = -1;
  SegRetrArgs ra{};
  {
    int slot = 0;
    for (int h = 0; h < p->Hq; ++h)
      if (is_long[h]) {
        a.long_slot[h] = (int16_t)slot;
        ra.long_heads[slot] = (int16_t)h;
        ++slot;
      }
  }
  AttnMaps m;
  if (!make_map(&m.q, at<void>(ws, P.qr), p->d, S, Hq, B, d, (int64_t)S * d, Hq * S * d)) return SATTN_ERR_CUDA;
  if (!make_map(&m.k, at<void>(state, L.krot), p->d, p->T, Hkv, B, d, Tcap * d, Hkv * Tcap * d)) return SATTN_ERR_CUDA;
  if (!make_map(&m.v, at<void>(state, L.vhist), p->d, p->T, Hkv, B, d, Tcap * d, Hkv * Tcap * d)) return SATTN_ERR_CUDA;
  m.q2 = m.q;
  m.kg = m.k;
  m.vg = m.v;
  if (P.n_long > 0 && R > 0 && seg > 0) {
    ra.B = p->B;
    ra.Hq = p->Hq;
    ra.Hkv = p->Hkv;
    ra.T = Tnow;
    ra.d = p->d;
    ra.S = S;
    ra.N = seg + 1;
    ra.R = R;
    ra.blk = retr_block;
    ra.n_long = P.n_long;
    ra.s_lo = seg;  // this segment alone, its arrays the only ones held
    ra.s_base = seg;
    ra.Q = nullptr;
    ra.q_end = at<__nv_bfloat16>(state, L.qend);
    ra.qe_sb = (int64_t)Hq * d;
    ra.qe_sh = d;
    ra.K = at<__nv_bfloat16>(state, L.khist);
    ra.V = at<__nv_bfloat16>(state, L.vhist);
    ra.k_sb = ra.v_sb = (int64_t)Hkv * Tcap * d;
    ra.k_sh = ra.v_sh = (int64_t)Tcap * d;
    ra.k_st = ra.v_st = d;
    ra.tab = L.tab.bytes ? at<float2>(state, L.tab) : nullptr;
    ra.prefix_blocks = prefix_blocks;
    ra.prefix_cnt = at<int32_t>(ws, P.pcnt);
    ra.Kpre = at<__nv_bfloat16>(ws, P.kpre);
    ra.Vpre = at<__nv_bfloat16>(ws, P.vpre);
    ra.score = at<float>(ws, P.score);
    {
      ProfScope ps("segment_retrieval", 3, st);
      SATTN_TRY(launch_segment_retrieval(ra, st));
    }
    const int64_t planes = P.n_long;
    if (!make_map(&m.kg, ra.Kpre, p->d, P.Rpad, planes, B, d, (int64_t)P.Rpad * d, planes * P.Rpad * d))
      return SATTN_ERR_CUDA;
    if (!make_map(&m.vg, ra.Vpre, p->d, P.Rpad, planes, B, d, (int64_t)P.Rpad * d, planes * P.Rpad * d))
      return SATTN_ERR_CUDA;
  }
  // 4. attention of the segment's rows over the state
  a.B = p->B;
  a.Hq = p->Hq;
  a.Hkv = p->Hkv;
  a.T = Tnow;
  a.d = p->d;
  a.nQT = S / kTile;
  a.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)p->d));
  a.ns_band = 0;
  a.w_eff = 0x3fffffff;
  a.V = at<__nv_bfloat16>(state, L.vhist);
  a.v_sb = (int64_t)Hkv * Tcap * d;
  a.v_sh = (int64_t)Tcap * d;
  a.v_st = d;
  a.gather_mode = 2;
  a.q2 = false;
  a.seg_S = S;
  a.seg_M = M;
  a.seg_N = seg + 1;
  a.seg_R = R;
  a.seg_s0 = seg;
  a.q_pos0 = seg * S;
  a.T_q = S;
  a.prefix_cnt = at<int32_t>(ws, P.pcnt);
  a.n_long = std::max(P.n_long, 1);
  a.O = static_cast<__nv_bfloat16*>(O);
  a.o_sb = p->o_stride[0];
  a.o_sh = p->o_stride[1];
  a.o_st = p->o_stride[2];
  a.lse = lse;
  a.status = status;
  {
    ProfScope ps("attn_tc_segment", 1, st);
    SATTN_TRY((S % (2 * kTile) == 0) ? launch_attn_tc2(a, m, st) : launch_attn_tc3(a, m, st));
  }
  // 5. the segment's last query is carried to the next step
  ProfScope ps("segment_state_finish", 1, st);
  return cuda_rc(launch_segstate_finish(sa, st));
}

// ---------------------------------------------------------------------------
// segmented execution: backward
// ---------------------------------------------------------------------------

struct SegBwdPlan {
  Region status, tab, dsum;
  size_t total = 0;
};

static int plan_seg_bwd(const sattn_params* p, int32_t S, int32_t M, int32_t R, int32_t blk, SegBwdPlan* out) {
  SegPlan F;
  int rc = plan_seg(p, S, M, R, blk, nullptr, &F);  // the forward's rules
  if (rc) return rc;
  SegBwdPlan P;
  Alloc A;
  P.status = A.take(kStatusBytes);
  if (p->rope_theta != 0.0) P.tab = A.take((size_t)p->T * (p->d / 2) * sizeof(float2));
  P.dsum = A.take((size_t)p->B * p->Hq * p->T * 4);
  P.total = A.cur;
  *out = P;
  return SATTN_OK;
}

int sattn_segment_bwd_workspace_size(const sattn_params* p, int32_t S, int32_t M, int32_t R, int32_t retr_block,
                                     size_t* bytes) {
  if (!bytes) return SATTN_ERR_INVALID_ARG;
  SegBwdPlan P;
  int rc = plan_seg_bwd(p, S, M, R, retr_block, &P);
  if (rc) return rc;
  *bytes = P.total;
  return SATTN_OK;
}

int sattn_segment_bwd(const sattn_params* p, int32_t S, int32_t M, int32_t R, int32_t retr_block,
                      const uint8_t* is_long, const void* Q, const void* K, const void* V, const void* O,
                      const float* lse, const int32_t* prefix_blocks, const void* dO, void* dQ, void* dK, void* dV,
                      void* ws, size_t ws_bytes, void* stream) {
  if (!is_long) return SATTN_ERR_INVALID_ARG;
  SegBwdPlan P;
  int rc = plan_seg_bwd(p, S, M, R, retr_block, &P);
  if (rc) return rc;
  if (!Q || !K || !V || !O || !lse || !dO || !dQ || !dK || !dV) return SATTN_ERR_INVALID_ARG;
  if (R > 0 && !prefix_blocks) return SATTN_ERR_INVALID_ARG;
  if (!ws || ws_bytes < P.total || (reinterpret_cast<uintptr_t>(ws) & 255u)) return SATTN_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  SATTN_TRY(cudaMemsetAsync(ws, 0, kStatusBytes, st));
  if (P.tab.bytes) {
    ProfScope ps("rope_table", 1, st);
    SATTN_TRY(launch_rope_table(at<float2>(ws, P.tab), p->T, p->d, p->rope_theta, pos_scale(p), st));
  }
  SegBwdArgs a{};
  a.B = p->B;
  a.Hq = p->Hq;
  a.Hkv = p->Hkv;
  a.T = p->T;
  a.d = p->d;
  a.S = S;
  a.N = p->T / S;
  a.M = M;
  a.R = R;
  a.blk = retr_block;
  a.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)p->d));
  a.Q = static_cast<const __nv_bfloat16*>(Q);
  a.K = static_cast<const __nv_bfloat16*>(K);
  a.V = static_cast<const __nv_bfloat16*>(V);
  a.O = static_cast<const __nv_bfloat16*>(O);
  a.dO = static_cast<const __nv_bfloat16*>(dO);
  a.q_sb = p->q_stride[0];
  a.q_sh = p->q_stride[1];
  a.q_st = p->q_stride[2];
  a.k_sb = p->k_stride[0];
  a.k_sh = p->k_stride[1];
  a.k_st = p->k_stride[2];
  a.v_sb = p->v_stride[0];
  a.v_sh = p->v_stride[1];
  a.v_st = p->v_stride[2];
  a.o_sb = p->o_stride[0];
  a.o_sh = p->o_stride[1];
  a.o_st = p->o_stride[2];
  a.lse = lse;
  a.prefix_blocks = prefix_blocks;
  for (int h = 0; h < kMaxHeads; ++h) a.long_slot[h] = -1;
  {
    int slot = 0;
    for (int h = 0; h < p->Hq; ++h)
      if (is_long[h]) a.long_slot[h] = (int16_t)slot++;
  }
  a.tab = P.tab.bytes ? at<float2>(ws, P.tab) : nullptr;
  a.Dsum = at<float>(ws, P.dsum);
  a.dQ = static_cast<__nv_bfloat16*>(dQ);
  a.dK = static_cast<__nv_bfloat16*>(dK);
  a.dV = static_cast<__nv_bfloat16*>(dV);
  a.dq_sb = p->q_stride[0];
  a.dq_sh = p->q_stride[1];
  a.dq_st = p->q_stride[2];
  a.dk_sb = p->k_stride[0];
  a.dk_sh = p->k_stride[1];
  a.dk_st = p->k_stride[2];
  a.dv_sb = p->v_stride[0];
  a.dv_sh = p->v_stride[1];
  a.dv_st = p->v_stride[2];
  ProfScope ps("segment_bwd", 2, st);
  return cuda_rc(launch_segment_bwd(a, st));
}

// ---------------------------------------------------------------------------
// SharedLLM tree cross-attention
// ---------------------------------------------------------------------------

struct TreePlan {
  int n_kept = 0, S = 0, Spad = 0, nQT = 0, npos = 0;
  Region status, tab, qr, kt, vt;
  size_t total = 0;
};

static int plan_tree(const sattn_params* p, int32_t n_chunks, int32_t chunk_len, int32_t depth, int32_t alpha_leaf,
                     TreePlan* out) {
  int rc = check_common(p);
  if (rc) return rc;
  if (p->dtype != SATTN_DTYPE_BF16) return SATTN_ERR_UNSUPPORTED;
  if (p->topk != 0 || p->L_pretrain != 0 || p->alibi || p->with_separators) return SATTN_ERR_INVALID_ARG;
  if (n_chunks < 1 || chunk_len < 1) return SATTN_ERR_INVALID_ARG;
  TreePlan P;
  P.n_kept = tree_kept_count(chunk_len, depth, alpha_leaf);
  if (P.n_kept < 1) return SATTN_ERR_INVALID_ARG;
  if ((int64_t)n_chunks * chunk_len > ((int64_t)1 << 30) || (int64_t)n_chunks * P.n_kept > ((int64_t)1 << 28))
    return SATTN_ERR_UNSUPPORTED;
  P.S = n_chunks * P.n_kept;
  P.Spad = (P.S + kTile - 1) / kTile * kTile;
  P.nQT = (p->T + kTile - 1) / kTile;
  P.npos = n_chunks + 1;
  const size_t B = p->B, Hq = p->Hq, Hkv = p->Hkv, T = p->T, d = p->d;
  Alloc A;
  P.status = A.take(kStatusBytes);
  if (p->rope_theta != 0.0) P.tab = A.take((size_t)P.npos * (d / 2) * sizeof(float2));
  P.qr = A.take(B * Hq * T * d * 2);
  P.kt = A.take(B * Hkv * (size_t)P.Spad * d * 2);
  P.vt = A.take(B * Hkv * (size_t)P.Spad * d * 2);
  P.total = A.cur;
  *out = P;
  return SATTN_OK;
}

// ---------------------------------------------------------------------------
// decoding step
// ---------------------------------------------------------------------------

struct DecPlan {
  int nQT, npos, n_chunks;
  Region status, prefix, sep_pos, sep_count, ranges, part, tk_cz, tk_cj, tk_idx, tk_z, tk_part;
  int tk_nchunks = 0;
  size_t total;
};

// the decoding step's rotation: theta^(-2c/d) per pair in double (the
// prefill table's values) and the position scale
static void set_decode_rope(DecodeArgs& a, const sattn_params* p) {
  a.rope = p->rope_theta != 0.0 ? 1 : 0;
  a.rope_scale = pos_scale(p);
  for (int c = 0; c < p->d / 2 && c < 64; ++c) a.inv_freq[c] = std::pow(p->rope_theta, -2.0 * (double)c / (double)p->d);
}

static int plan_decode(const sattn_params* p, DecPlan* out) {
  int rc = check_common(p);
  if (rc) return rc;
  if (p->dtype != SATTN_DTYPE_BF16) return SATTN_ERR_UNSUPPORTED;
  // top-k with ALiBi ranks by q.k only when every candidate is past the cap
  if (p->alibi && p->topk > 0 && (p->L_pretrain == 0 || p->window < p->L_pretrain)) return SATTN_ERR_UNSUPPORTED;
  const int rep = p->Hq / p->Hkv;
  if (rep != 1 && rep != 2 && rep != 4 && rep != 8) return SATTN_ERR_UNSUPPORTED;
  if (p->L_pretrain > 0 && p->window > p->L_pretrain) return SATTN_ERR_UNSUPPORTED;
  if (p->T > decode_max_len()) return SATTN_ERR_UNSUPPORTED;
  DecPlan P;
  P.nQT = (p->T + kTile - 1) / kTile;
  P.npos = std::max(p->T, p->L_pretrain + 1);
  P.n_chunks = decode_chunks(p->T);
  const size_t B = p->B, Hq = p->Hq, T = p->T, d = p->d;
  Alloc A;
  P.status = A.take(kStatusBytes);
  if (p->with_separators) {
    P.prefix = A.take(blockmap_scratch_bytes(p->B, p->T, p->window));
    P.sep_pos = A.take(B * T * 4);
    P.sep_count = A.take(B * 4);
    P.ranges = A.take(B * P.nQT * 2 * 4);
  }
  P.part = A.take(B * Hq * (size_t)P.n_chunks * (d + 2) * 4);
  if (p->topk > 0) {
    P.tk_nchunks = decode_topk_chunks(p->T - 1 - p->window - p->n_start);
    const size_t nc = (size_t)std::max(P.tk_nchunks, 1) * p->topk;
    P.tk_cz = A.take(B * Hq * nc * 4);
    P.tk_cj = A.take(B * Hq * nc * 4);
    P.tk_idx = A.take(B * Hq * (size_t)p->topk * 4);
    P.tk_z = A.take(B * Hq * (size_t)p->topk * 4);
    P.tk_part = A.take(B * Hq * (d + 2) * 4);
  }
  P.total = A.cur;
  *out = P;
  return SATTN_OK;
}

int sattn_decode_workspace_size(const sattn_params* p, size_t* bytes) {
  if (!bytes) return SATTN_ERR_INVALID_ARG;
  DecPlan P;
  int rc = plan_decode(p, &P);
  if (rc) return rc;
  *bytes = P.total;
  return SATTN_OK;
}

int sattn_decode_fwd(const sattn_params* p, const void* Q, const void* K, const void* V, const uint8_t* is_sep,
                     void* O, float* lse, void* ws, size_t ws_bytes, void* stream) {
  return sattn_decode_topk_fwd(p, Q, K, V, is_sep, O, lse, nullptr, nullptr, ws, ws_bytes, stream);
}

int sattn_decode_topk_fwd(const sattn_params* p, const void* Q, const void* K, const void* V, const uint8_t* is_sep,
                          void* O, float* lse, int32_t* topk_idx, float* topk_logit, void* ws, size_t ws_bytes,
                          void* stream) {
  DecPlan P;
  int rc = plan_decode(p, &P);
  if (rc) return rc;
  if (!Q || !K || !V || !O || !lse) return SATTN_ERR_INVALID_ARG;
  if (is_sep && !p->with_separators) return SATTN_ERR_INVALID_ARG;
  if (!ws || ws_bytes < P.total || (reinterpret_cast<uintptr_t>(ws) & 255u)) return SATTN_ERR_INVALID_ARG;
  if (!pointers_ok_bf16(Q, K, V) || !aligned16(O)) return SATTN_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  SATTN_TRY(cudaMemsetAsync(ws, 0, kStatusBytes, st));
  if (is_sep) {
    FwdPlan F;
    F.prefix = P.prefix;
    rc = run_blockmap(p, F, is_sep, nullptr, at<int32_t>(ws, P.sep_pos), at<int32_t>(ws, P.sep_count),
                      at<int32_t>(ws, P.ranges), ws, st);
    if (rc) return rc;
  }
  DecodeArgs a{};
  a.B = p->B;
  a.Hq = p->Hq;
  a.Hkv = p->Hkv;
  a.T = p->T;
  a.d = p->d;
  a.n_start = p->n_start;
  a.window = p->window;
  a.L = p->L_pretrain;
  a.alibi = p->alibi ? 1 : 0;
  a.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)p->d));
  a.Q = static_cast<const __nv_bfloat16*>(Q);
  a.q_sb = p->q_stride[0];
  a.q_sh = p->q_stride[1];
  a.K = static_cast<const __nv_bfloat16*>(K);
  a.k_sb = p->k_stride[0];
  a.k_sh = p->k_stride[1];
  a.k_st = p->k_stride[2];
  a.V = static_cast<const __nv_bfloat16*>(V);
  a.v_sb = p->v_stride[0];
  a.v_sh = p->v_stride[1];
  a.v_st = p->v_stride[2];
  set_decode_rope(a, p);
  a.sep_words = is_sep ? at<uint2>(ws, P.prefix) : nullptr;
  a.sep_pos = is_sep ? at<int32_t>(ws, P.sep_pos) : nullptr;
  a.part = at<float>(ws, P.part);
  a.status = at<int32_t>(ws, P.status);
  a.n_chunks = P.n_chunks;
  if (p->topk > 0) {
    a.topk = p->topk;
    a.tk_nchunks = P.tk_nchunks;
    a.tk_cz = at<float>(ws, P.tk_cz);
    a.tk_cj = at<int32_t>(ws, P.tk_cj);
    a.tk_idx = topk_idx ? topk_idx : at<int32_t>(ws, P.tk_idx);
    a.tk_z = topk_logit ? topk_logit : at<float>(ws, P.tk_z);
    a.tk_part = at<float>(ws, P.tk_part);
  }
  a.O = static_cast<__nv_bfloat16*>(O);
  a.o_sb = p->o_stride[0];
  a.o_sh = p->o_stride[1];
  a.lse = lse;
  const int n_topk_kernels = p->topk > 0 ? (p->T - 1 - p->window - p->n_start > 0 ? 2 : 1) : 0;
  ProfScope ps("decode", 2 + n_topk_kernels, st);
  return cuda_rc(launch_decode(a, st));
}

// ---------------------------------------------------------------------------
// backward pass
// ---------------------------------------------------------------------------

struct BwdPlan {
  FwdPlan F;  // regions shared with the forward's steps (status, table, prep products, block map, gather)
  int nRB = 0;
  Region dsum, nlse2, sink_ds, sink_p, sink_part, dq_side, dk_band, dv_band, dk_sep, dv_sep, tk_ds, tk_p, tk_cnt,
      tk_off, tk_cur, tk_code, tk_sorted;
  size_t total = 0;
};

static int plan_bwd(const sattn_params* p, BwdPlan* out) {
  int rc = check_fwd_rules(p);
  if (rc) return rc;
  BwdPlan P;
  FwdPlan& F = P.F;
  F.bf16 = p->dtype == SATTN_DTYPE_BF16;
  // top-k key lists are indexed in 32 bits
  if (F.bf16 && p->topk > 0 && (int64_t)p->B * p->Hq * p->T * p->topk >= ((int64_t)1 << 31))
    return SATTN_ERR_UNSUPPORTED;
  F.nQT = (p->T + kTile - 1) / kTile;
  F.Tpad = F.nQT * kTile;
  F.npos = std::max(p->T, p->L_pretrain + 1);
  F.n_sink = std::min(p->n_start, p->T);
  F.capped_sep = p->L_pretrain > 0 && p->with_separators;
  F.need_qc = F.bf16 && F.capped_sep;
  const size_t B = p->B, Hq = p->Hq, Hkv = p->Hkv, T = p->T, d = p->d, Tpad = F.Tpad;
  Alloc A;
  F.status = A.take(kStatusBytes);
  if (p->rope_theta != 0.0) F.tab = A.take((size_t)F.npos * (d / 2) * sizeof(float2));
  if (p->with_separators) {
    F.prefix = A.take(blockmap_scratch_bytes(p->B, p->T, std::max(p->window, sep_split_of(p))));
    F.sep_pos = A.take(B * T * 4);
    F.sep_count = A.take(B * 4);
    F.ranges = A.take(B * F.nQT * 2 * 4);
  }
  if (!F.bf16) {
    P.dsum = A.take(B * Hq * T * 4);
  } else {
    F.qr = A.take(B * Hq * T * d * 2);
    F.kr = A.take(B * Hkv * T * d * 2);
    if (F.need_qc) F.qc = A.take(B * Hq * T * d * 2);
    if (p->with_separators) {
      F.ks = A.take(B * Hkv * Tpad * d * 2);
      F.vs = A.take(B * Hkv * Tpad * d * 2);
      P.dk_sep = A.take(B * Hkv * Tpad * d * 4);
      P.dv_sep = A.take(B * Hkv * Tpad * d * 4);
    }
    P.dsum = A.take(B * Hq * Tpad * 4);
    P.nlse2 = A.take(B * Hq * Tpad * 4);
    if (F.n_sink > 0) {
      F.sink = A.take(B * Hq * T * F.n_sink * 4);
      P.sink_ds = A.take(B * Hq * T * F.n_sink * 4);
      P.sink_p = A.take(B * Hq * T * F.n_sink * 4);
      P.nRB = (int)((T + bwd_sink_row_block() - 1) / bwd_sink_row_block());
      P.sink_part = A.take(B * Hkv * F.n_sink * (size_t)P.nRB * 2 * d * 4);
    }
    // the capped separators' dq (first dq pass) and the top-k pairs' dq
    if (F.capped_sep || p->topk > 0) P.dq_side = A.take(B * Hq * T * d * 4);
    P.dk_band = A.take(B * Hkv * T * d * 4);
    P.dv_band = A.take(B * Hkv * T * d * 4);
    if (p->topk > 0) {
      const size_t sel = B * Hq * T * (size_t)p->topk;
      P.tk_ds = A.take(sel * 4);
      P.tk_p = A.take(sel * 4);
      P.tk_cnt = A.take(B * Hkv * T * 4);
      P.tk_off = A.take(B * Hkv * T * 4);
      P.tk_cur = A.take(B * Hkv * T * 4);
      P.tk_code = A.take(sel * 4);
      P.tk_sorted = A.take(sel * 4);
    }
  }
  P.total = A.cur;
  *out = P;
  return SATTN_OK;
}

static int run_bwd_bf16(const sattn_params* p, const BwdPlan& P, const void* Q, const void* K, const void* V,
                        const uint8_t* is_sep, const int32_t* topk_idx, const void* O, const float* lse,
                        const void* dO, void* dQ, void* dK, void* dV, void* ws, cudaStream_t st) {
  const FwdPlan& F = P.F;
  const int64_t B = p->B, Hq = p->Hq, Hkv = p->Hkv, T = p->T, d = p->d;
  int rc = run_prep_bf16(p, F, Q, K, ws, F.n_sink > 0, false, st);
  if (rc) return rc;
  BwdMaps m;
  if (!make_map(&m.q, at<void>(ws, F.qr), p->d, p->T, Hq, B, d, T * d, Hq * T * d)) return SATTN_ERR_CUDA;
  if (!make_map(&m.k, at<void>(ws, F.kr), p->d, p->T, Hkv, B, d, T * d, Hkv * T * d)) return SATTN_ERR_CUDA;
  if (!make_map(&m.v, V, p->d, p->T, Hkv, B, p->v_stride[2], p->v_stride[1], p->v_stride[0])) return SATTN_ERR_CUDA;
  if (!make_map(&m.dO, dO, p->d, p->T, Hq, B, p->o_stride[2], p->o_stride[1], p->o_stride[0])) return SATTN_ERR_CUDA;
  m.qc = m.q;
  m.kg = m.k;
  m.vg = m.v;
  int32_t* sep_pos = at<int32_t>(ws, F.sep_pos);
  int32_t* sep_count = at<int32_t>(ws, F.sep_count);
  int32_t* ranges = at<int32_t>(ws, F.ranges);
  if (is_sep) {
    rc = run_blockmap(p, F, is_sep, nullptr, sep_pos, sep_count, ranges, ws, st, sep_split_of(p));
    if (rc) return rc;
    GatherArgs ga{};
    ga.B = p->B;
    ga.Hkv = p->Hkv;
    ga.T = p->T;
    ga.Tpad = F.Tpad;
    ga.d = p->d;
    if (F.capped_sep) {
      ga.Ksrc = static_cast<const __nv_bfloat16*>(K);
      ga.k_sb = p->k_stride[0];
      ga.k_sh = p->k_stride[1];
      ga.k_st = p->k_stride[2];
      if (!make_map(&m.qc, at<void>(ws, F.qc), p->d, p->T, Hq, B, d, T * d, Hq * T * d)) return SATTN_ERR_CUDA;
    } else {
      ga.Ksrc = at<__nv_bfloat16>(ws, F.kr);
      ga.k_sb = Hkv * T * d;
      ga.k_sh = T * d;
      ga.k_st = d;
    }
    ga.Vsrc = static_cast<const __nv_bfloat16*>(V);
    ga.v_sb = p->v_stride[0];
    ga.v_sh = p->v_stride[1];
    ga.v_st = p->v_stride[2];
    ga.sep_pos = sep_pos;
    ga.sep_count = sep_count;
    ga.Ks = at<__nv_bfloat16>(ws, F.ks);
    ga.Vs = at<__nv_bfloat16>(ws, F.vs);
    {
      ProfScope ps("sep_gather", 1, st);
      SATTN_TRY(launch_sep_gather(ga, st));
    }
    if (!make_map(&m.kg, ga.Ks, p->d, F.Tpad, Hkv, B, d, (int64_t)F.Tpad * d, Hkv * F.Tpad * d)) return SATTN_ERR_CUDA;
    if (!make_map(&m.vg, ga.Vs, p->d, F.Tpad, Hkv, B, d, (int64_t)F.Tpad * d, Hkv * F.Tpad * d)) return SATTN_ERR_CUDA;
  }
  BwdArgs a{};
  a.B = p->B;
  a.Hq = p->Hq;
  a.Hkv = p->Hkv;
  a.T = p->T;
  a.d = p->d;
  a.nQT = F.nQT;
  a.Tpad = F.Tpad;
  a.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)p->d));
  a.n_start = p->n_start;
  a.window = p->window;
  a.L = p->L_pretrain;
  a.sep_split = sep_split_of(p);
  a.w_sepband = (is_sep && sep_band_extended(p)) ? p->L_pretrain : 0;
  a.alibi = p->alibi ? 1 : 0;
  a.alibi_cap = p->L_pretrain;
  a.tab = F.tab.bytes ? at<float2>(ws, F.tab) : nullptr;
  a.Q = static_cast<const __nv_bfloat16*>(Q);
  a.K = static_cast<const __nv_bfloat16*>(K);
  a.V = static_cast<const __nv_bfloat16*>(V);
  a.O = static_cast<const __nv_bfloat16*>(O);
  a.dO = static_cast<const __nv_bfloat16*>(dO);
  a.q_sb = p->q_stride[0];
  a.q_sh = p->q_stride[1];
  a.q_st = p->q_stride[2];
  a.k_sb = p->k_stride[0];
  a.k_sh = p->k_stride[1];
  a.k_st = p->k_stride[2];
  a.v_sb = p->v_stride[0];
  a.v_sh = p->v_stride[1];
  a.v_st = p->v_stride[2];
  a.o_sb = p->o_stride[0];
  a.o_sh = p->o_stride[1];
  a.o_st = p->o_stride[2];
  a.lse = lse;
  a.Qr = at<__nv_bfloat16>(ws, F.qr);
  a.Qc = F.qc.bytes ? at<__nv_bfloat16>(ws, F.qc) : nullptr;
  a.sink_z = F.n_sink > 0 ? at<float>(ws, F.sink) : nullptr;
  a.n_sink = F.n_sink;
  a.gather = is_sep ? 1 : 0;
  a.capped_sep = (is_sep && F.capped_sep) ? 1 : 0;
  a.sep_pos = is_sep ? sep_pos : nullptr;
  a.sep_count = is_sep ? sep_count : nullptr;
  a.sep_words = is_sep ? at<uint2>(ws, F.prefix) : nullptr;
  a.ranges = is_sep ? ranges : nullptr;
  a.Dsum = at<float>(ws, P.dsum);
  a.nlse2 = at<float>(ws, P.nlse2);
  a.sink_ds = F.n_sink > 0 ? at<float>(ws, P.sink_ds) : nullptr;
  a.sink_p = F.n_sink > 0 ? at<float>(ws, P.sink_p) : nullptr;
  a.sink_part = F.n_sink > 0 ? at<float>(ws, P.sink_part) : nullptr;
  a.nRB = P.nRB;
  a.dq_side = P.dq_side.bytes ? at<float>(ws, P.dq_side) : nullptr;
  a.dk_band = at<float>(ws, P.dk_band);
  a.dv_band = at<float>(ws, P.dv_band);
  a.dk_sep = is_sep ? at<float>(ws, P.dk_sep) : nullptr;
  a.dv_sep = is_sep ? at<float>(ws, P.dv_sep) : nullptr;
  a.dQ = static_cast<__nv_bfloat16*>(dQ);
  a.dK = static_cast<__nv_bfloat16*>(dK);
  a.dV = static_cast<__nv_bfloat16*>(dV);
  a.status = at<int32_t>(ws, F.status);
  a.topk = p->topk;
  a.tk_idx = p->topk > 0 ? topk_idx : nullptr;
  a.tk_ds = at<float>(ws, P.tk_ds);
  a.tk_p = at<float>(ws, P.tk_p);
  a.tk_cnt = at<int>(ws, P.tk_cnt);
  a.tk_off = at<int>(ws, P.tk_off);
  a.tk_cur = at<int>(ws, P.tk_cur);
  a.tk_code = at<int>(ws, P.tk_code);
  a.tk_sorted = at<int>(ws, P.tk_sorted);
  {
    ProfScope ps("bwd_rows", 1, st);
    SATTN_TRY(launch_bwd_rows(a, st));
  }
  // capped separators: a first dq pass writes their part to dq_side, the
  // second adds it; the top-k pairs' dq joins dq_side in between; the sink
  // pairs' dq is formed in the second pass's epilogue
  a.side_valid = false;
  a.fold_sinks = 0;
  if (a.capped_sep) {
    a.dq_mode = 1;
    ProfScope ps("bwd_dq", 1, st);
    SATTN_TRY(launch_bwd_dq(a, m, st));
    a.side_valid = true;
  }
  if (p->topk > 0) {
    ProfScope ps("bwd_topk_rows", 1, st);
    SATTN_TRY(launch_bwd_topk_rows(a, a.side_valid, st));
    a.side_valid = true;
  }
  a.dq_mode = 0;
  a.fold_sinks = F.n_sink > 0 ? 1 : 0;
  {
    ProfScope ps("bwd_dq", 1, st);
    SATTN_TRY(launch_bwd_dq(a, m, st));
  }
  {
    ProfScope ps("bwd_dkv", 1, st);
    SATTN_TRY(launch_bwd_dkv(a, m, st));
  }
  if (p->topk > 0) {
    ProfScope ps("bwd_topk_keys", 5, st);
    SATTN_TRY(launch_bwd_topk_keys(a, st));
  }
  if (F.n_sink > 0) {
    ProfScope ps("bwd_sink_keys", 1, st);
    SATTN_TRY(launch_bwd_sink_keys(a, st));
  }
  ProfScope ps("bwd_combine", 1, st);
  return cuda_rc(launch_bwd_combine(a, st));
}

int sattn_bwd_workspace_size(const sattn_params* p, size_t* bytes) {
  if (!bytes) return SATTN_ERR_INVALID_ARG;
  BwdPlan P;
  int rc = plan_bwd(p, &P);
  if (rc) return rc;
  *bytes = P.total;
  return SATTN_OK;
}

int sattn_bwd(const sattn_params* p, const void* Q, const void* K, const void* V, const uint8_t* is_sep,
              const int32_t* topk_idx, const void* O, const float* lse, const void* dO, void* dQ, void* dK, void* dV,
              void* ws, size_t ws_bytes, void* stream) {
  BwdPlan P;
  int rc = plan_bwd(p, &P);
  if (rc) return rc;
  if (!Q || !K || !V || !O || !lse || !dO || !dQ || !dK || !dV) return SATTN_ERR_INVALID_ARG;
  if (is_sep && !p->with_separators) return SATTN_ERR_INVALID_ARG;
  if (p->topk > 0 && !topk_idx) return SATTN_ERR_INVALID_ARG;  // the forward's selection is an input
  if (!ws || ws_bytes < P.total || (reinterpret_cast<uintptr_t>(ws) & 255u)) return SATTN_ERR_INVALID_ARG;
  const FwdPlan& F = P.F;
  if (F.bf16 && (!pointers_ok_bf16(Q, K, V) || !pointers_ok_bf16(O, dO, dQ) || !aligned16(dK) || !aligned16(dV)))
    return SATTN_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  SATTN_TRY(cudaMemsetAsync(ws, 0, kStatusBytes, st));
  if (F.bf16) return run_bwd_bf16(p, P, Q, K, V, is_sep, topk_idx, O, lse, dO, dQ, dK, dV, ws, st);
  if (F.tab.bytes) {
    ProfScope ps("rope_table", 1, st);
    SATTN_TRY(launch_rope_table(at<float2>(ws, F.tab), F.npos, p->d, p->rope_theta, pos_scale(p), st));
  }
  if (is_sep) {
    rc = run_blockmap(p, F, is_sep, nullptr, at<int32_t>(ws, F.sep_pos), at<int32_t>(ws, F.sep_count),
                      at<int32_t>(ws, F.ranges), ws, st);
    if (rc) return rc;
  }
  BwdF32Args a{};
  a.B = p->B;
  a.Hq = p->Hq;
  a.Hkv = p->Hkv;
  a.T = p->T;
  a.d = p->d;
  a.Q = static_cast<const float*>(Q);
  a.K = static_cast<const float*>(K);
  a.V = static_cast<const float*>(V);
  a.O = static_cast<const float*>(O);
  a.dO = static_cast<const float*>(dO);
  a.q_sb = p->q_stride[0];
  a.q_sh = p->q_stride[1];
  a.q_st = p->q_stride[2];
  a.k_sb = p->k_stride[0];
  a.k_sh = p->k_stride[1];
  a.k_st = p->k_stride[2];
  a.v_sb = p->v_stride[0];
  a.v_sh = p->v_stride[1];
  a.v_st = p->v_stride[2];
  a.o_sb = p->o_stride[0];
  a.o_sh = p->o_stride[1];
  a.o_st = p->o_stride[2];
  a.lse = lse;
  a.tab = F.tab.bytes ? at<float2>(ws, F.tab) : nullptr;
  a.L = p->L_pretrain;
  a.n_start = p->n_start;
  a.window = p->window;
  a.is_sep = is_sep;
  a.sep_pos = is_sep ? at<int32_t>(ws, F.sep_pos) : nullptr;
  a.sep_count = is_sep ? at<int32_t>(ws, F.sep_count) : nullptr;
  a.tk_idx = p->topk > 0 ? topk_idx : nullptr;
  a.topk = p->topk;
  a.alibi = p->alibi ? 1 : 0;
  a.Dsum = at<float>(ws, P.dsum);
  a.dQ = static_cast<float*>(dQ);
  a.dK = static_cast<float*>(dK);
  a.dV = static_cast<float*>(dV);
  a.dq_sb = p->q_stride[0];
  a.dq_sh = p->q_stride[1];
  a.dq_st = p->q_stride[2];
  a.dk_sb = p->k_stride[0];
  a.dk_sh = p->k_stride[1];
  a.dk_st = p->k_stride[2];
  a.dv_sb = p->v_stride[0];
  a.dv_sh = p->v_stride[1];
  a.dv_st = p->v_stride[2];
  ProfScope ps("bwd_f32", 2, st);
  return cuda_rc(launch_bwd_f32(a, st));
}

int sattn_tree_cross_workspace_size(const sattn_params* p, int32_t n_chunks, int32_t chunk_len, int32_t depth,
                                    int32_t alpha_leaf, size_t* bytes) {
  if (!bytes) return SATTN_ERR_INVALID_ARG;
  TreePlan P;
  int rc = plan_tree(p, n_chunks, chunk_len, depth, alpha_leaf, &P);
  if (rc) return rc;
  *bytes = P.total;
  return SATTN_OK;
}

int sattn_tree_cross_fwd(const sattn_params* p, int32_t n_chunks, int32_t chunk_len, int32_t depth,
                         int32_t alpha_leaf, const void* Q, const void* K, const void* V, void* O, float* lse,
                         int32_t* kept_index, void* ws, size_t ws_bytes, void* stream) {
  TreePlan P;
  int rc = plan_tree(p, n_chunks, chunk_len, depth, alpha_leaf, &P);
  if (rc) return rc;
  if (!Q || !K || !V || !O || !lse) return SATTN_ERR_INVALID_ARG;
  if (!ws || ws_bytes < P.total || (reinterpret_cast<uintptr_t>(ws) & 255u)) return SATTN_ERR_INVALID_ARG;
  if (!pointers_ok_bf16(Q, K, V) || !aligned16(O)) return SATTN_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  SATTN_TRY(cudaMemsetAsync(ws, 0, kStatusBytes, st));
  if (P.tab.bytes) {
    ProfScope ps("rope_table", 1, st);
    SATTN_TRY(launch_rope_table(at<float2>(ws, P.tab), P.npos, p->d, p->rope_theta, pos_scale(p), st));
  }
  TreeArgs t{};
  t.B = p->B;
  t.Hq = p->Hq;
  t.Hkv = p->Hkv;
  t.Tq = p->T;
  t.d = p->d;
  t.n_chunks = n_chunks;
  t.chunk_len = chunk_len;
  t.depth = depth;
  t.alpha_leaf = alpha_leaf;
  t.n_kept = P.n_kept;
  t.Spad = P.Spad;
  t.tab = at<float2>(ws, P.tab);
  t.Q = static_cast<const __nv_bfloat16*>(Q);
  t.q_sb = p->q_stride[0];
  t.q_sh = p->q_stride[1];
  t.q_st = p->q_stride[2];
  t.K = static_cast<const __nv_bfloat16*>(K);
  t.V = static_cast<const __nv_bfloat16*>(V);
  t.k_sb = p->k_stride[0];
  t.k_sh = p->k_stride[1];
  t.k_st = p->k_stride[2];
  t.v_sb = p->v_stride[0];
  t.v_sh = p->v_stride[1];
  t.v_st = p->v_stride[2];
  t.Qr = at<__nv_bfloat16>(ws, P.qr);
  t.Kt = at<__nv_bfloat16>(ws, P.kt);
  t.Vt = at<__nv_bfloat16>(ws, P.vt);
  t.kept_index = kept_index;
  {
    ProfScope ps("tree_prep", 1, st);
    SATTN_TRY(launch_tree_prep(t, st));
  }
  const int64_t B = p->B, Hq = p->Hq, Hkv = p->Hkv, T = p->T, d = p->d;
  AttnMaps m;
  if (!make_map(&m.q, t.Qr, p->d, p->T, Hq, B, d, T * d, Hq * T * d)) return SATTN_ERR_CUDA;
  if (!make_map(&m.kg, t.Kt, p->d, P.Spad, Hkv, B, d, (int64_t)P.Spad * d, Hkv * P.Spad * d)) return SATTN_ERR_CUDA;
  if (!make_map(&m.vg, t.Vt, p->d, P.Spad, Hkv, B, d, (int64_t)P.Spad * d, Hkv * P.Spad * d)) return SATTN_ERR_CUDA;
  m.q2 = m.q;
  m.k = m.kg;
  m.v = m.vg;
  AttnArgs a{};
  a.B = p->B;
  a.Hq = p->Hq;
  a.Hkv = p->Hkv;
  a.T = p->T;
  a.d = p->d;
  a.nQT = P.nQT;
  a.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)p->d));
  a.ns_band = 0;
  a.w_eff = 0;
  a.V = t.Vt;
  a.v_sb = Hkv * P.Spad * d;
  a.v_sh = (int64_t)P.Spad * d;
  a.v_st = d;
  a.gather_mode = 3;
  a.cross_len = P.S;
  a.q2 = false;
  a.O = static_cast<__nv_bfloat16*>(O);
  a.o_sb = p->o_stride[0];
  a.o_sh = p->o_stride[1];
  a.o_st = p->o_stride[2];
  a.lse = lse;
  a.status = at<int32_t>(ws, P.status);
  ProfScope ps("attn_tc_cross", 1, st);
  return cuda_rc(launch_attn_tc2(a, m, st));
}

// ---------------------------------------------------------------------------
// streaming KV cache
// ---------------------------------------------------------------------------

struct StreamLayout {
  Region sizes, len, ctrl, pos, flag, dst, k, v, ks, vs, pos_s, flag_s;
  size_t total = 0;
};

static int stream_layout(const sattn_stream_config* cfg, StreamLayout* out) {
  if (!cfg) return SATTN_ERR_INVALID_ARG;
  if (cfg->B < 1 || cfg->Hkv < 1 || cfg->a < 0 || cfg->s < 0 || cfg->w < 1) return SATTN_ERR_INVALID_ARG;
  if ((int64_t)cfg->a + cfg->s + cfg->w >= cfg->c) return SATTN_ERR_INVALID_ARG;  // a full cache could not shrink
  if (cfg->d != 64 && cfg->d != 128) return SATTN_ERR_UNSUPPORTED;
  if (cfg->c > (1 << 24)) return SATTN_ERR_UNSUPPORTED;
  const size_t B = cfg->B, H = cfg->Hkv, c = cfg->c, d = cfg->d;
  StreamLayout L;
  Alloc A;
  L.sizes = A.take(B * 4 * 4);
  L.len = A.take(B * 4);
  L.ctrl = A.take(B * 2 * 4);
  L.pos = A.take(B * c * 4);
  L.flag = A.take(B * c);
  L.dst = A.take(B * c * 4);
  L.k = A.take(B * H * c * d * 2);
  L.v = A.take(B * H * c * d * 2);
  L.ks = A.take(B * H * c * d * 2);
  L.vs = A.take(B * H * c * d * 2);
  L.pos_s = A.take(B * c * 4);
  L.flag_s = A.take(B * c);
  L.total = A.cur;
  *out = L;
  return SATTN_OK;
}

static StreamArgs stream_args(const sattn_stream_config* cfg, const StreamLayout& L, void* state) {
  StreamArgs a{};
  a.B = cfg->B;
  a.Hkv = cfg->Hkv;
  a.d = cfg->d;
  a.a = cfg->a;
  a.s = cfg->s;
  a.w = cfg->w;
  a.c = cfg->c;
  a.sizes = at<int32_t>(state, L.sizes);
  a.len = at<int32_t>(state, L.len);
  a.ctrl = at<int32_t>(state, L.ctrl);
  a.pos = at<int32_t>(state, L.pos);
  a.flag = at<uint8_t>(state, L.flag);
  a.dst = at<int32_t>(state, L.dst);
  a.K = at<__nv_bfloat16>(state, L.k);
  a.V = at<__nv_bfloat16>(state, L.v);
  a.Ks = at<__nv_bfloat16>(state, L.ks);
  a.Vs = at<__nv_bfloat16>(state, L.vs);
  a.pos_s = at<int32_t>(state, L.pos_s);
  a.flag_s = at<uint8_t>(state, L.flag_s);
  return a;
}

int sattn_stream_state_size(const sattn_stream_config* cfg, size_t* bytes) {
  if (!bytes) return SATTN_ERR_INVALID_ARG;
  StreamLayout L;
  int rc = stream_layout(cfg, &L);
  if (rc) return rc;
  *bytes = L.total;
  return SATTN_OK;
}

static int stream_check_state(const sattn_stream_config* cfg, const void* state, size_t state_bytes,
                              StreamLayout* L) {
  int rc = stream_layout(cfg, L);
  if (rc) return rc;
  if (!state || state_bytes < L->total || (reinterpret_cast<uintptr_t>(state) & 255u)) return SATTN_ERR_INVALID_ARG;
  return SATTN_OK;
}

int sattn_stream_reset(const sattn_stream_config* cfg, void* state, size_t state_bytes, void* stream) {
  StreamLayout L;
  int rc = stream_check_state(cfg, state, state_bytes, &L);
  if (rc) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // sizes, lengths and plan flags start at zero (the three regions are contiguous)
  SATTN_TRY(cudaMemsetAsync(state, 0, L.pos.off, st));
  return SATTN_OK;
}

int sattn_stream_append(const sattn_stream_config* cfg, void* state, size_t state_bytes, const void* K_new,
                        const void* V_new, const uint8_t* is_sep, int64_t position, void* stream) {
  StreamLayout L;
  int rc = stream_check_state(cfg, state, state_bytes, &L);
  if (rc) return rc;
  if (!K_new || !V_new || !aligned16(K_new) || !aligned16(V_new)) return SATTN_ERR_INVALID_ARG;
  if (position < 0 || position > INT32_MAX) return SATTN_ERR_INVALID_ARG;
  StreamArgs a = stream_args(cfg, L, state);
  a.position = position;
  a.K_new = static_cast<const __nv_bfloat16*>(K_new);
  a.V_new = static_cast<const __nv_bfloat16*>(V_new);
  a.sep_new = is_sep;
  ProfScope ps("stream_append", 4, static_cast<cudaStream_t>(stream));
  return cuda_rc(launch_stream_append(a, static_cast<cudaStream_t>(stream)));
}

int sattn_stream_read(const sattn_stream_config* cfg, const void* state, size_t state_bytes, int32_t* sizes,
                      int32_t* positions, void* stream) {
  StreamLayout L;
  int rc = stream_check_state(cfg, state, state_bytes, &L);
  if (rc) return rc;
  if (!sizes) return SATTN_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return SATTN_ERR_CUDA;
  const uint8_t* base = static_cast<const uint8_t*>(state);
  if (cudaMemcpy(sizes, base + L.sizes.off, (size_t)cfg->B * 4 * 4, cudaMemcpyDeviceToHost) != cudaSuccess)
    return SATTN_ERR_CUDA;
  if (positions && cudaMemcpy(positions, base + L.pos.off, (size_t)cfg->B * cfg->c * 4, cudaMemcpyDeviceToHost) !=
                       cudaSuccess)
    return SATTN_ERR_CUDA;
  return SATTN_OK;
}

static int plan_stream_decode(const sattn_stream_config* cfg, const sattn_params* p, DecPlan* out) {
  StreamLayout L;
  int rc = stream_layout(cfg, &L);
  if (rc) return rc;
  if (!p || p->B != cfg->B || p->Hkv != cfg->Hkv || p->d != cfg->d || p->dtype != SATTN_DTYPE_BF16)
    return SATTN_ERR_INVALID_ARG;
  if (p->Hq < 1 || p->Hq % p->Hkv) return SATTN_ERR_INVALID_ARG;
  const int rep = p->Hq / p->Hkv;
  if (rep != 1 && rep != 2 && rep != 4 && rep != 8) return SATTN_ERR_UNSUPPORTED;
  if (!(p->rope_theta >= 0.0) || !(p->rope_pos_scale >= 0.0) || p->rope_pos_scale > 1.0) return SATTN_ERR_INVALID_ARG;
  if (cfg->c > decode_max_len()) return SATTN_ERR_UNSUPPORTED;
  DecPlan P{};
  P.nQT = (cfg->c + kTile - 1) / kTile;
  P.npos = cfg->c;
  P.n_chunks = decode_chunks(cfg->c);
  Alloc A;
  P.status = A.take(kStatusBytes);
  P.part = A.take((size_t)p->B * p->Hq * (size_t)P.n_chunks * (p->d + 2) * 4);
  P.total = A.cur;
  *out = P;
  return SATTN_OK;
}

int sattn_stream_decode_workspace_size(const sattn_stream_config* cfg, const sattn_params* p, size_t* bytes) {
  if (!bytes) return SATTN_ERR_INVALID_ARG;
  DecPlan P;
  int rc = plan_stream_decode(cfg, p, &P);
  if (rc) return rc;
  *bytes = P.total;
  return SATTN_OK;
}

int sattn_stream_decode(const sattn_stream_config* cfg, const sattn_params* p, const void* state, size_t state_bytes,
                        const void* Q, void* O, float* lse, void* ws, size_t ws_bytes, void* stream) {
  DecPlan P;
  int rc = plan_stream_decode(cfg, p, &P);
  if (rc) return rc;
  StreamLayout L;
  rc = stream_check_state(cfg, state, state_bytes, &L);
  if (rc) return rc;
  if (!Q || !O || !lse || !aligned16(Q) || !aligned16(O)) return SATTN_ERR_INVALID_ARG;
  if (!ws || ws_bytes < P.total || (reinterpret_cast<uintptr_t>(ws) & 255u)) return SATTN_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  SATTN_TRY(cudaMemsetAsync(ws, 0, kStatusBytes, st));
  void* sp = const_cast<void*>(state);
  const int64_t H = cfg->Hkv, c = cfg->c, d = cfg->d;
  DecodeArgs a{};
  a.B = p->B;
  a.Hq = p->Hq;
  a.Hkv = p->Hkv;
  a.T = cfg->c;
  a.d = p->d;
  a.n_start = 0;
  a.window = cfg->c;  // every cached entry is kept
  a.L = 0;
  a.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)p->d));
  a.Q = static_cast<const __nv_bfloat16*>(Q);
  a.q_sb = p->q_stride[0];
  a.q_sh = p->q_stride[1];
  a.K = at<__nv_bfloat16>(sp, L.k);
  a.k_sb = H * c * d;
  a.k_sh = c * d;
  a.k_st = d;
  a.V = at<__nv_bfloat16>(sp, L.v);
  a.v_sb = H * c * d;
  a.v_sh = c * d;
  a.v_st = d;
  set_decode_rope(a, p);
  a.seq_len = at<int32_t>(sp, L.len);
  a.part = at<float>(ws, P.part);
  a.status = at<int32_t>(ws, P.status);
  a.n_chunks = P.n_chunks;
  a.O = static_cast<__nv_bfloat16*>(O);
  a.o_sb = p->o_stride[0];
  a.o_sh = p->o_stride[1];
  a.lse = lse;
  ProfScope ps("stream_decode", 2, st);
  return cuda_rc(launch_decode(a, st));
}

int sattn_stream_status(void* stream, const void* ws, int32_t* device_status) {
  if (!ws || !device_status) return SATTN_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return SATTN_ERR_CUDA;
  int32_t v = 0;
  if (cudaMemcpy(&v, ws, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return SATTN_ERR_CUDA;
  *device_status = v;
  return SATTN_OK;
}

int sattn_profile_enable(int on) {
  std::lock_guard<std::mutex> g(g_prof_mu);
  g_prof_on = on != 0;
  return SATTN_OK;
}

int sattn_profile_collect(char* names, int32_t* launches, double* total_ms, int32_t max_groups, int32_t* n_groups) {
  if (!names || !launches || !total_ms || !n_groups || max_groups < 0) return SATTN_ERR_INVALID_ARG;
  std::vector<ProfRec> recs;
  {
    std::lock_guard<std::mutex> g(g_prof_mu);
    recs.swap(g_prof_recs);
  }
  std::map<std::string, std::pair<int64_t, double>> acc;
  std::vector<std::string> order;
  int rc = SATTN_OK;
  for (const ProfRec& r : recs) {
    float ms = 0.f;
    if (cudaEventSynchronize(r.b) != cudaSuccess || cudaEventElapsedTime(&ms, r.a, r.b) != cudaSuccess) rc = SATTN_ERR_CUDA;
    auto it = acc.find(r.name);
    if (it == acc.end()) {
      order.push_back(r.name);
      acc[r.name] = {r.kernels, (double)ms};
    } else {
      it->second.first += r.kernels;
      it->second.second += ms;
    }
  }
  {
    std::lock_guard<std::mutex> g(g_prof_mu);
    for (const ProfRec& r : recs) {
      g_prof_pool.push_back(r.a);
      g_prof_pool.push_back(r.b);
    }
  }
  int n = 0;
  for (const std::string& k : order) {
    if (n >= max_groups) break;
    std::strncpy(names + 32 * n, k.c_str(), 31);
    names[32 * n + 31] = 0;
    launches[n] = (int32_t)acc[k].first;
    total_ms[n] = acc[k].second;
    ++n;
  }
  *n_groups = n;
  return rc;
}

}  // extern "C"
