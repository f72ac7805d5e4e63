// topk.cu -- K4: per-head top-k middle-token selection.
//
// "LM-Infinite" (section 方法, optional top-k) adds, per attention head, the
// k middle tokens with the largest attention logit.  Candidates of row i are
// n_start <= j < i - w that are not separators; the score is the unscaled
// capped logit z_ij; ties go to the smaller j.
//
// Three passes:
//  1. scoring on the tensor cores: S = Qsel Ksel^T in bf16 x bf16 -> fp32
//     (Qsel/Ksel = R(L)q / raw k when capped, R(i)q / R(j)k otherwise); each
//     row keeps a shortlist of the `short_len` best coarse scores;
//  2. exact re-rank: one warp per row recomputes the shortlisted logits in
//     fp32 from the exact inputs and certifies the result: every key left
//     out has a coarse score <= the last shortlisted one, and the coarse
//     score differs from the fp32 one by at most eps (operand rounding bound
//     ||q - bf16(q)|| * max||k|| plus the accumulation bound), so if the
//     k-th re-ranked logit exceeds that score + eps the top-k is exact;
//  3. rows that fail the certificate (rare) are rescanned exactly in fp32
//     over all their candidates.
#include <cuda_bf16.h>
#include <math_constants.h>

#include "kernels.cuh"
#include "sm100.cuh"

namespace sattn {

namespace {

constexpr int kThreads = 192;
constexpr int kStages = 4;
constexpr int kScratchStride = 33;  // floats per scan thread's scratch row (odd: no bank conflicts)

template <typename Tin>
__device__ __forceinline__ float ld_in(const Tin* p);
template <>
__device__ __forceinline__ float ld_in<__nv_bfloat16>(const __nv_bfloat16* p) {
  return __bfloat162float(*p);
}
template <>
__device__ __forceinline__ float ld_in<float>(const float* p) {
  return *p;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ bool mbar_wait_raw(uint64_t* bar, uint32_t parity) {
  uint32_t a = smem_u32(bar);
  uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(a, parity)) {
    if (globaltimer_ns() - t0 > 100000000ull) return false;
  }
  return true;
}

// insert (v, j) into the descending list (vals, idxs); strict > keeps the
// earlier (smaller j) entry first among equal scores
template <int KC>
__device__ __forceinline__ void list_insert(float v, int j, float (&vals)[KC], int (&idxs)[KC]) {
#pragma unroll
  for (int x = 0; x < KC; ++x) {
    if (v > vals[x]) {
      const float tv = vals[x];
      const int tj = idxs[x];
      vals[x] = v;
      idxs[x] = j;
      v = tv;
      j = tj;
    }
  }
}

// ---------------------------------------------------------------------------
// pass 1: tensor-core scoring with a per-row shortlist
// ---------------------------------------------------------------------------
template <int D, int KC>
__global__ void __launch_bounds__(kThreads, 1)
    topk_score_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                      const TopkArgs a) {
  constexpr uint32_t kTileBytes = D * kTile * 2;
  constexpr int kChunks = D / 64;
  constexpr uint32_t kChunkBytes = kTile * 128;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sq = base;
  uint8_t* sk[kStages];
  for (int s = 0; s < kStages; ++s) sk[s] = base + kTileBytes * (1 + s);
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + kTileBytes * (1 + kStages));
  uint64_t* q_full = bars;
  uint64_t* k_full = bars + 1;
  uint64_t* k_empty = bars + 1 + kStages;
  uint64_t* s_full = bars + 1 + 2 * kStages;
  uint64_t* s_free = bars + 1 + 3 * kStages;
  uint64_t* drain = bars + 1 + 4 * kStages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 + 4 * kStages);
  int* abort_i = reinterpret_cast<int*>(tmem_slot + 1);
  int* early = abort_i + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x % a.nQT;
  const int bh = blockIdx.x / a.nQT;
  const int h = bh % a.Hq, b = bh / a.Hq;
  const int g = h / (a.Hq / a.Hkv);
  const int i0 = t * kTile;
  const int i1 = min(a.T - 1, i0 + kTile - 1);
  const int hi_key = i1 - a.window - 1;
  int u_lo = 0, ntiles = 0;
  if (hi_key >= a.n_start) {
    u_lo = a.n_start / kTile;
    ntiles = hi_key / kTile - u_lo + 1;
  }

  if (threadIdx.x == 0) {
    *early = status_failed(a.status) ? 1 : 0;
    *abort_i = 0;
    mbar_init(q_full, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(k_full + s, 1);
      mbar_init(k_empty + s, 1);
      mbar_init(s_full + s, 1);
      mbar_init(s_free + s, 128);
    }
    mbar_init(drain, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (*early) return;
  if (warp == 5) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  volatile int* abort_flag = abort_i;

  if (warp == 4) {
    if (lane == 0 && ntiles > 0) {
      mbar_expect_tx(q_full, kTileBytes);
      for (int c = 0; c < kChunks; ++c) tma_load_4d(sq + c * kChunkBytes, &tmQ, q_full, c * 64, i0, h, b);
      int issued = 0;
      bool ok = true;
      for (int it = 0; it < ntiles; ++it) {
        const int st = it % kStages;
        if (it >= kStages) ok = mbar_wait(k_empty + st, ((it / kStages) - 1) & 1, abort_flag, a.status, 21);
        if (!ok) break;
        mbar_expect_tx(k_full + st, kTileBytes);
        for (int c = 0; c < kChunks; ++c)
          tma_load_4d(sk[st] + c * kChunkBytes, &tmK, k_full + st, c * 64, (u_lo + it) * kTile, g, b);
        ++issued;
      }
      if (!ok) {
        mbar_wait_raw(q_full, 0);
        for (int it = max(0, issued - kStages); it < issued; ++it) mbar_wait_raw(k_full + it % kStages, (it / kStages) & 1);
      }
    }
  } else if (warp == 5) {
    if (lane == 0 && ntiles > 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(128, 128, false);
      const uint32_t q_addr = smem_u32(sq);
      bool ok = mbar_wait(q_full, 0, abort_flag, a.status, 22);
      for (int it = 0; it < ntiles && ok; ++it) {
        const int st = it % kStages;
        ok = mbar_wait(k_full + st, (it / kStages) & 1, abort_flag, a.status, 23);
        if (ok && it >= kStages) ok = mbar_wait(s_free + st, ((it / kStages) - 1) & 1, abort_flag, a.status, 24);
        if (!ok) break;
        tc_fence_after();
        const uint32_t k_addr = smem_u32(sk[st]);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * kChunkBytes + (kk & 3) * 32;
          tc_mma_ss(tmem + st * 128, smem_desc_sw128(q_addr + off, 16, 1024), smem_desc_sw128(k_addr + off, 16, 1024),
                    idesc, kk > 0 ? 1u : 0u);
        }
        tc_commit(s_full + st);
        tc_commit(k_empty + st);
      }
      tc_commit(drain);
      mbar_wait_raw(drain, 0);
    }
    __syncwarp();
  } else {
    // scan warps: thread r owns query row i0 + r (TMEM lane r)
    const int r = threadIdx.x;
    const int i = i0 + r;
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    // candidates of this row: n_start <= j <= i - w - 1; of the warp's rows,
    // the smallest upper bound decides which tiles need no per-column mask
    const int j_hi = i - a.window - 1;
    float* my_scratch = reinterpret_cast<float*>(base + kTileBytes * (1 + kStages) + 1024) + r * kScratchStride;
    const int warp_j_hi = i0 + warp * 32 - a.window - 1;
    float vals[KC];
    int idxs[KC];
#pragma unroll
    for (int x = 0; x < KC; ++x) {
      vals[x] = -CUDART_INF_F;
      idxs[x] = -1;
    }
    int ncand = 0;
    bool ok = true;
    const uint8_t* flags = a.is_sep ? a.is_sep + (size_t)b * a.T : nullptr;
    for (int it = 0; it < ntiles; ++it) {
      const int st = it % kStages;
      ok = ok && mbar_wait(s_full + st, (it / kStages) & 1, abort_flag, a.status, 25);
      tc_fence_after();
      float v[128];
#pragma unroll
      for (int c4 = 0; c4 < 4; ++c4) tmem_ld32(tmem + st * 128 + lane_off + c4 * 32, v + c4 * 32);
      tc_wait_ld();
      // the scores are in registers: hand the TMEM buffer back to the MMA warp
      tc_fence_before();
      if (ok) mbar_arrive(s_free + st);
      const int j0 = (u_lo + it) * kTile;
      const bool interior = (j0 >= a.n_start) && (j0 + kTile - 1 <= warp_j_hi);
      if (!interior || flags) {
        const int c_lo = max(0, a.n_start - j0);
        const int c_hi = min(kTile - 1, j_hi - j0);
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) {
          uint32_t sepm = 0;
          if (flags) {
            const int jj = j0 + c4 * 32 + lane;
            sepm = __ballot_sync(0xffffffffu, jj < a.T && flags[jj] != 0);
          }
          const int lo = max(c_lo - c4 * 32, 0);
          const int hi = min(c_hi - c4 * 32, 31);
          uint32_t vm = 0;
          if (lo <= hi) vm = (hi == 31 ? 0xffffffffu : ((1u << (hi + 1)) - 1u)) & ~((1u << lo) - 1u);
          vm &= ~sepm;
          ncand += __popc(vm);
#pragma unroll
          for (int x = 0; x < 32; ++x) v[c4 * 32 + x] = ((vm >> x) & 1u) ? v[c4 * 32 + x] : -CUDART_INF_F;
        }
      } else {
        ncand += kTile;
      }
      // per 32-column chunk maxima (independent chains), then the insertion
      // path only for chunks that beat the row's current threshold
      float cm[4];
#pragma unroll
      for (int c4 = 0; c4 < 4; ++c4) {
        float pm[8];
#pragma unroll
        for (int y = 0; y < 8; ++y) pm[y] = v[c4 * 32 + y];
#pragma unroll
        for (int x = 8; x < 32; ++x) pm[x & 7] = fmaxf(pm[x & 7], v[c4 * 32 + x]);
        cm[c4] = fmaxf(fmaxf(fmaxf(pm[0], pm[1]), fmaxf(pm[2], pm[3])), fmaxf(fmaxf(pm[4], pm[5]), fmaxf(pm[6], pm[7])));
      }
      // a chunk that beats the threshold goes through this thread's shared
      // scratch row, so one copy of the insertion code serves every column
      // (an unrolled insertion per column would not fit the instruction cache)
#pragma unroll
      for (int c4 = 0; c4 < 4; ++c4) {
        if (cm[c4] > vals[KC - 1]) {
          uint32_t msk = 0;
#pragma unroll
          for (int x = 0; x < 32; ++x) {
            my_scratch[x] = v[c4 * 32 + x];
            msk |= (v[c4 * 32 + x] > vals[KC - 1]) ? (1u << x) : 0u;
          }
          while (msk) {
            const int x = __ffs(msk) - 1;
            msk &= msk - 1;
            const float z = my_scratch[x];
            if (z > vals[KC - 1]) list_insert<KC>(z, j0 + c4 * 32 + x, vals, idxs);
          }
        }
      }
    }
    if (i < a.T) {
      const size_t row = ((size_t)b * a.Hq + h) * a.T + i;
#pragma unroll
      for (int x = 0; x < KC; ++x) a.short_idx[row * KC + x] = idxs[x];
      a.short_thr[row] = (ncand > KC) ? vals[KC - 1] : -CUDART_INF_F;
      a.n_cand[row] = ncand;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------------------
// shared fp32 helpers for passes 2 and 3
// ---------------------------------------------------------------------------

// Query rotated to the row position (qi) and to the cap (qc), fp32, lane
// owns pairs c = lane*PP + e.
template <typename Tin, int PP>
struct RowQuery {
  float qi0[PP], qi1[PP], qc0[PP], qc1[PP];
  __device__ __forceinline__ void load(const TopkArgs& a, const Tin* qp, int i, int lane) {
    const int half = a.d / 2;
#pragma unroll
    for (int e = 0; e < PP; ++e) {
      const int c = lane * PP + e;
      const float x0 = ld_in(qp + c), x1 = ld_in(qp + c + half);
      const float2 cs = a.tab ? a.tab[(int64_t)i * half + c] : make_float2(1.f, 0.f);
      qi0[e] = x0 * cs.x - x1 * cs.y;
      qi1[e] = x1 * cs.x + x0 * cs.y;
      const float2 cl = (a.tab && a.L > 0) ? a.tab[(int64_t)a.L * half + c] : make_float2(1.f, 0.f);
      qc0[e] = x0 * cl.x - x1 * cl.y;
      qc1[e] = x1 * cl.x + x0 * cl.y;
    }
  }
  // this lane's part of z_ij (capped rule)
  __device__ __forceinline__ float partial(const TopkArgs& a, const Tin* kp, int i, int j, int lane) const {
    const int half = a.d / 2;
    const bool capped = a.L > 0 && (i - j) > a.L;
    float acc = 0.f;
#pragma unroll
    for (int e = 0; e < PP; ++e) {
      const int c = lane * PP + e;
      const float k0 = ld_in(kp + c), k1 = ld_in(kp + c + half);
      if (capped) {
        acc = fmaf(qc0[e], k0, fmaf(qc1[e], k1, acc));
      } else {
        const float2 cs = a.tab ? a.tab[(int64_t)j * half + c] : make_float2(1.f, 0.f);
        acc = fmaf(qi0[e], k0 * cs.x - k1 * cs.y, fmaf(qi1[e], k1 * cs.x + k0 * cs.y, acc));
      }
    }
    return acc;
  }
};

// ---------------------------------------------------------------------------
// pass 2: exact re-rank of the shortlist + certificate (warp per row)
// ---------------------------------------------------------------------------
template <int PP, int KC>
__global__ void topk_rerank_kernel(const TopkArgs a) {
  const int lane = threadIdx.x & 31;
  const int64_t row = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;
  const int64_t nrows = (int64_t)a.B * a.Hq * a.T;
  if (row >= nrows) return;
  const int i = (int)(row % a.T);
  const int64_t bh = row / a.T;
  const int h = (int)(bh % a.Hq), b = (int)(bh / a.Hq);
  const int g = h / (a.Hq / a.Hkv);
  const __nv_bfloat16* Q = reinterpret_cast<const __nv_bfloat16*>(a.Q);
  const __nv_bfloat16* K = reinterpret_cast<const __nv_bfloat16*>(a.K);
  RowQuery<__nv_bfloat16, PP> rq;
  rq.load(a, Q + b * a.q_sb + h * a.q_sh + (int64_t)i * a.q_st, i, lane);
  // the bf16 operand the scoring pass used, and its rounding error
  const bool capped_all = a.L > 0;  // capped scoring requires L == window
  float dq2 = 0.f, qn2 = 0.f;
#pragma unroll
  for (int e = 0; e < PP; ++e) {
    const float u0 = capped_all ? rq.qc0[e] : rq.qi0[e];
    const float u1 = capped_all ? rq.qc1[e] : rq.qi1[e];
    const float b0 = __bfloat162float(__float2bfloat16_rn(u0));
    const float b1 = __bfloat162float(__float2bfloat16_rn(u1));
    dq2 += (u0 - b0) * (u0 - b0) + (u1 - b1) * (u1 - b1);
    qn2 += b0 * b0 + b1 * b1;
  }
  dq2 = warp_sum(dq2);
  qn2 = warp_sum(qn2);
  const float kmax = __uint_as_float(a.kmax[(size_t)b * a.Hkv + g]) * (1.f + 1.f / 128.f);
  const float qn = sqrtf(qn2);
  float eps = sqrtf(dq2) * kmax + qn * kmax * (1.f / 32768.f);
  if (!capped_all) eps += qn * kmax * (1.f / 256.f);  // rotated keys were rounded too
  eps *= 1.0625f;

  const int32_t* sl = a.short_idx + row * KC;
  const __nv_bfloat16* kb = K + b * a.k_sb + g * a.k_sh;
  float zs[KC];
  int js[KC];
#pragma unroll
  for (int x = 0; x < KC; ++x) {
    const int j = sl[x];
    js[x] = j;
    zs[x] = (j >= 0) ? warp_sum(rq.partial(a, kb + (int64_t)j * a.k_st, i, j, lane)) : -CUDART_INF_F;
  }
  // sort (z desc, j asc); invalid entries (-1) last
#pragma unroll
  for (int x = 1; x < KC; ++x) {
#pragma unroll
    for (int y = x; y > 0; --y) {
      const bool less = (js[y - 1] < 0 && js[y] >= 0) ||
                        (js[y] >= 0 && js[y - 1] >= 0 &&
                         (zs[y] > zs[y - 1] || (zs[y] == zs[y - 1] && js[y] < js[y - 1])));
      if (less) {
        const float tz = zs[y];
        zs[y] = zs[y - 1];
        zs[y - 1] = tz;
        const int tj = js[y];
        js[y] = js[y - 1];
        js[y - 1] = tj;
      }
    }
  }
  const int n = a.n_cand[row];
  const float thr = a.short_thr[row];
  const int k = a.topk;
  float zk = -CUDART_INF_F;
#pragma unroll
  for (int x = 0; x < KC; ++x)
    if (x == k - 1) zk = zs[x];
  const bool certified = (n <= KC) || (zk > thr + eps);
  if (lane == 0) {
    if (certified) {
#pragma unroll
      for (int x = 0; x < KC; ++x) {
        if (x < k) {
          a.idx[row * k + x] = (x < n) ? js[x] : -1;
          a.z[row * k + x] = (x < n) ? zs[x] : -CUDART_INF_F;
        }
      }
    } else {
      const int pos = atomicAdd(a.status + 2, 1);
      a.fallback_rows[pos] = (int32_t)row;
    }
  }
}

// ---------------------------------------------------------------------------
// pass 3: exact fp32 scan of all candidates of a row (block per row)
// ---------------------------------------------------------------------------
constexpr int kExactThreads = 256;
constexpr int kMaxK = 16;

template <typename Tin, int PP>
__global__ void __launch_bounds__(kExactThreads) topk_exact_kernel(const TopkArgs a, int all_rows) {
  __shared__ float red_z[kExactThreads / 32];
  __shared__ int red_j[kExactThreads / 32];
  __shared__ float s_q[2][128 * 2];  // qi, qc (d <= 256 would fit; d <= 128 used)
  const int64_t nrows = (int64_t)a.B * a.Hq * a.T;
  const int64_t count = all_rows ? nrows : (int64_t)(*reinterpret_cast<volatile int32_t*>(a.status + 2));
  const Tin* Q = reinterpret_cast<const Tin*>(a.Q);
  const Tin* K = reinterpret_cast<const Tin*>(a.K);
  const int half = a.d / 2;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int64_t x = blockIdx.x; x < count; x += gridDim.x) {
    const int64_t row = all_rows ? x : a.fallback_rows[x];
    const int i = (int)(row % a.T);
    const int64_t bh = row / a.T;
    const int h = (int)(bh % a.Hq), b = (int)(bh / a.Hq);
    const int g = h / (a.Hq / a.Hkv);
    const Tin* qp = Q + b * a.q_sb + h * a.q_sh + (int64_t)i * a.q_st;
    __syncthreads();
    for (int c = threadIdx.x; c < half; c += blockDim.x) {
      const float x0 = ld_in(qp + c), x1 = ld_in(qp + c + half);
      const float2 cs = a.tab ? a.tab[(int64_t)i * half + c] : make_float2(1.f, 0.f);
      s_q[0][c] = x0 * cs.x - x1 * cs.y;
      s_q[0][c + half] = x1 * cs.x + x0 * cs.y;
      const float2 cl = (a.tab && a.L > 0) ? a.tab[(int64_t)a.L * half + c] : make_float2(1.f, 0.f);
      s_q[1][c] = x0 * cl.x - x1 * cl.y;
      s_q[1][c + half] = x1 * cl.x + x0 * cl.y;
    }
    __syncthreads();
    float vals[kMaxK];
    int idxs[kMaxK];
#pragma unroll
    for (int y = 0; y < kMaxK; ++y) {
      vals[y] = -CUDART_INF_F;
      idxs[y] = -1;
    }
    const Tin* kb = K + b * a.k_sb + g * a.k_sh;
    const uint8_t* flags = a.is_sep ? a.is_sep + (size_t)b * a.T : nullptr;
    const int jend = i - a.window;  // candidates j < i - w
    for (int j = a.n_start + threadIdx.x; j < jend; j += blockDim.x) {
      if (flags && flags[j]) continue;
      const Tin* kp = kb + (int64_t)j * a.k_st;
      const bool capped = a.L > 0 && (i - j) > a.L;
      float acc = 0.f;
      for (int c = 0; c < half; ++c) {
        const float k0 = ld_in(kp + c), k1 = ld_in(kp + c + half);
        if (capped) {
          acc = fmaf(s_q[1][c], k0, fmaf(s_q[1][c + half], k1, acc));
        } else {
          const float2 cs = a.tab ? a.tab[(int64_t)j * half + c] : make_float2(1.f, 0.f);
          acc = fmaf(s_q[0][c], k0 * cs.x - k1 * cs.y, fmaf(s_q[0][c + half], k1 * cs.x + k0 * cs.y, acc));
        }
      }
      if (acc > vals[kMaxK - 1] || (acc == vals[kMaxK - 1] && j < idxs[kMaxK - 1]))
        list_insert<kMaxK>(acc, j, vals, idxs);
    }
    // k rounds of block-wide argmax over (z desc, j asc)
    int head = 0;  // next unused entry of this thread's sorted list
    for (int r = 0; r < a.topk; ++r) {
      float bz = -CUDART_INF_F;
      int bj = -1;
#pragma unroll
      for (int y = 0; y < kMaxK; ++y)
        if (y == head) {
          bz = vals[y];
          bj = idxs[y];
        }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const float oz = __shfl_xor_sync(0xffffffffu, bz, o);
        const int oj = __shfl_xor_sync(0xffffffffu, bj, o);
        if (oj >= 0 && (bj < 0 || oz > bz || (oz == bz && oj < bj))) {
          bz = oz;
          bj = oj;
        }
      }
      if (lane == 0) {
        red_z[warp] = bz;
        red_j[warp] = bj;
      }
      __syncthreads();
      float wz = red_z[0];
      int wj = red_j[0];
      for (int w = 1; w < kExactThreads / 32; ++w) {
        const float oz = red_z[w];
        const int oj = red_j[w];
        if (oj >= 0 && (wj < 0 || oz > wz || (oz == wz && oj < wj))) {
          wz = oz;
          wj = oj;
        }
      }
      __syncthreads();
      if (wj >= 0 && head < kMaxK) {
        int hj = -2;
#pragma unroll
        for (int y = 0; y < kMaxK; ++y)
          if (y == head) hj = idxs[y];
        if (hj == wj) ++head;
      }
      if (threadIdx.x == 0) {
        a.idx[row * a.topk + r] = wj;
        a.z[row * a.topk + r] = (wj >= 0) ? wz : -CUDART_INF_F;
      }
    }
  }
}

template <int D, int KC>
cudaError_t launch_score(const TopkArgs& a, const TopkMaps& m, cudaStream_t st) {
  const size_t tile = (size_t)D * kTile * 2;
  // at least 116 KB: one CTA per SM, so the 512-column TMEM allocation never waits
  const size_t bytes = std::max<size_t>(116 * 1024, 1024 + tile * (1 + kStages) + 1024 + 128 * kScratchStride * 4);
  cudaError_t e = cudaFuncSetAttribute(topk_score_kernel<D, KC>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e != cudaSuccess) return e;
  topk_score_kernel<D, KC><<<(unsigned)(a.B * a.Hq * a.nQT), kThreads, bytes, st>>>(m.qsel, m.ksel, a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int64_t rows = (int64_t)a.B * a.Hq * a.T;
  const unsigned blocks = (unsigned)((rows * 32 + 255) / 256);
  topk_rerank_kernel<D / 64, KC><<<blocks, 256, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_topk_tc(const TopkArgs& a, const TopkMaps& m, cudaStream_t st) {
  if ((int64_t)a.B * a.Hq * a.T == 0) return cudaSuccess;
  if (a.d == 128) {
    if (a.short_len == 8) return launch_score<128, 8>(a, m, st);
    if (a.short_len == 16) return launch_score<128, 16>(a, m, st);
    if (a.short_len == 32) return launch_score<128, 32>(a, m, st);
  } else if (a.d == 64) {
    if (a.short_len == 8) return launch_score<64, 8>(a, m, st);
    if (a.short_len == 16) return launch_score<64, 16>(a, m, st);
    if (a.short_len == 32) return launch_score<64, 32>(a, m, st);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_topk_exact(const TopkArgs& a, bool all_rows, cudaStream_t st) {
  const int64_t rows = (int64_t)a.B * a.Hq * a.T;
  if (rows == 0) return cudaSuccess;
  const unsigned grid = all_rows ? (unsigned)std::min<int64_t>(rows, 148 * 16) : 148u * 4u;
  if (a.f32) {
    if (a.d == 128) topk_exact_kernel<float, 2><<<grid, kExactThreads, 0, st>>>(a, all_rows ? 1 : 0);
    else topk_exact_kernel<float, 1><<<grid, kExactThreads, 0, st>>>(a, all_rows ? 1 : 0);
  } else {
    if (a.d == 128) topk_exact_kernel<__nv_bfloat16, 2><<<grid, kExactThreads, 0, st>>>(a, all_rows ? 1 : 0);
    else topk_exact_kernel<__nv_bfloat16, 1><<<grid, kExactThreads, 0, st>>>(a, all_rows ? 1 : 0);
  }
  return cudaGetLastError();
}

}  // namespace sattn
