// topk.cu -- K4: per-head top-k middle-token selection.
//
// "LM-Infinite" (section 方法, optional top-k) adds, per attention head, the
// k middle tokens with the largest attention logit.  Candidates of row i are
// n_start <= j < i - w that are not separators; the score is the unscaled
// capped logit z_ij; ties go to the smaller j.
//
// Three passes:
//  1. scoring on the tensor cores: S = Qsel Ksel^T in bf16 x bf16 -> fp32
//     (Qsel/Ksel = R(L)q / raw k when capped, R(i)q / R(j)k otherwise).  A
//     CTA takes two 128-row query tiles; each K tile is loaded once and
//     multiplied into both tiles' TMEM score buffers; one scan warpgroup per
//     tile keeps, per row, a shortlist of the `short_len` best coarse scores;
//  2. exact re-rank: a group of short_len lanes per row recomputes the
//     shortlisted logits in fp32 from the exact inputs and certifies the
//     result: every key left out has a coarse score <= the last shortlisted
//     one, and the coarse score differs from the fp32 one by at most eps
//     (operand rounding bound ||q - bf16(q)|| * max||k|| plus the
//     accumulation bound), so if the k-th re-ranked logit exceeds that
//     score + eps the top-k is exact;
//  3. rows that fail the certificate (rare) are rescanned exactly in fp32
//     over all their candidates.
#include <cuda_bf16.h>
#include <math_constants.h>

#include "kernels.cuh"
#include "simt.cuh"
#include "sm100.cuh"

namespace sattn {

namespace {

constexpr int kThreads = 320;  // 8 scan warps (two query tiles), TMA warp, MMA warp
constexpr int kStages = 3;     // K tiles in flight
constexpr int kSBuf = 2;       // TMEM score buffers per query tile
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
                      const TopkArgs a, int nQB) {
  constexpr uint32_t kTileBytes = D * kTile * 2;
  constexpr int kChunks = D / 64;
  constexpr uint32_t kChunkBytes = kTile * 128;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sq = base;  // Q0 | Q1
  uint8_t* sk = base + 2 * kTileBytes;  // kStages K tiles
  uint64_t* bars = reinterpret_cast<uint64_t*>(sk + kStages * kTileBytes);
  uint64_t* q_full = bars;
  uint64_t* k_full = bars + 1;
  uint64_t* k_empty = k_full + kStages;
  uint64_t* s_full = k_empty + kStages;  // [2 tiles][kSBuf]
  uint64_t* s_free = s_full + 2 * kSBuf;  // [2 tiles][kSBuf]
  uint64_t* drain = s_free + 2 * kSBuf;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  int* abort_i = reinterpret_cast<int*>(tmem_slot + 1);
  int* early = abort_i + 1;
  float* scratch = reinterpret_cast<float*>(sk + kStages * kTileBytes + 1024);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qb = blockIdx.x % nQB;
  const int bh = blockIdx.x / nQB;
  const int h = bh % a.Hq, b = bh / a.Hq;
  const int g = h / (a.Hq / a.Hkv);
  // key tiles each query tile scans: [u_lo, u_lo + nt[x]); the union is the longer
  const int u_lo = a.n_start / kTile;
  int nt[2];
  for (int x = 0; x < 2; ++x) {
    const int i0x = (2 * qb + x) * kTile;
    nt[x] = 0;
    if (i0x < a.T) {
      const int hi_key = min(a.T - 1, i0x + kTile - 1) - a.window - 1;
      if (hi_key >= a.n_start) nt[x] = hi_key / kTile - u_lo + 1;
    }
  }
  const int ntiles = max(nt[0], nt[1]);

  if (threadIdx.x == 0) {
    *early = status_failed(a.status) ? 1 : 0;
    *abort_i = 0;
    mbar_init(q_full, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(k_full + s, 1);
      mbar_init(k_empty + s, 1);
    }
    for (int s = 0; s < 2 * kSBuf; ++s) {
      mbar_init(s_full + s, 1);
      mbar_init(s_free + s, 128);
    }
    mbar_init(drain, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (*early) return;
  if (warp == 9) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  volatile int* abort_flag = abort_i;

  if (warp == 8) {
    // ===== TMA producer: both query tiles once, then the K ring =====
    if (lane == 0 && ntiles > 0) {
      mbar_expect_tx(q_full, 2 * kTileBytes);
      for (int x = 0; x < 2; ++x)
        for (int c = 0; c < kChunks; ++c)
          tma_load_4d(sq + x * kTileBytes + c * kChunkBytes, &tmQ, q_full, c * 64, (2 * qb + x) * kTile, h, b);
      int issued = 0;
      bool ok = true;
      for (int it = 0; it < ntiles; ++it) {
        const int st = it % kStages;
        if (it >= kStages) ok = mbar_wait(k_empty + st, ((it / kStages) - 1) & 1, abort_flag, a.status, 21);
        if (!ok) break;
        mbar_expect_tx(k_full + st, kTileBytes);
        for (int c = 0; c < kChunks; ++c)
          tma_load_4d(sk + st * kTileBytes + c * kChunkBytes, &tmK, k_full + st, c * 64, (u_lo + it) * kTile, g, b);
        ++issued;
      }
      if (!ok) {
        mbar_wait_raw(q_full, 0);
        for (int it = max(0, issued - kStages); it < issued; ++it) mbar_wait_raw(k_full + it % kStages, (it / kStages) & 1);
      }
    }
  } else if (warp == 9) {
    // ===== MMA issuer: per K tile, S_x = Q_x K^T for each query tile still scanning =====
    if (lane == 0 && ntiles > 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(128, 128, false);
      const uint32_t q_addr = smem_u32(sq);
      bool ok = mbar_wait(q_full, 0, abort_flag, a.status, 22);
      for (int it = 0; it < ntiles && ok; ++it) {
        const int st = it % kStages;
        const int sb = it % kSBuf;
        ok = mbar_wait(k_full + st, (it / kStages) & 1, abort_flag, a.status, 23);
        if (!ok) break;
        const uint32_t k_addr = smem_u32(sk + st * kTileBytes);
        for (int x = 0; x < 2 && ok; ++x) {
          if (it >= nt[x]) continue;
          if (it >= kSBuf) ok = mbar_wait(s_free + x * kSBuf + sb, ((it / kSBuf) - 1) & 1, abort_flag, a.status, 24);
          if (!ok) break;
          tc_fence_after();
          const uint32_t qx = q_addr + x * kTileBytes;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * kChunkBytes + (kk & 3) * 32;
            tc_mma_ss(tmem + (x * kSBuf + sb) * 128, smem_desc_sw128(qx + off, 16, 1024),
                      smem_desc_sw128(k_addr + off, 16, 1024), idesc, kk > 0 ? 1u : 0u);
          }
          tc_commit(s_full + x * kSBuf + sb);
        }
        tc_commit(k_empty + st);
      }
      tc_commit(drain);
      mbar_wait_raw(drain, 0);
    }
    __syncwarp();
  } else if (warp < 8) {
    // scan warps: warpgroup qt = warp / 4 scans query tile qt; thread r of the
    // warpgroup owns query row i0 + r (TMEM lane r)
    const int qt = warp >> 2;
    const int r = threadIdx.x & 127;
    const int i0 = (2 * qb + qt) * kTile;
    const int i = i0 + r;
    const int ntx = nt[qt];
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    // candidates of this row: n_start <= j <= i - w - 1; of the warp's rows,
    // the smallest upper bound decides which tiles need no per-column mask
    const int j_hi = i - a.window - 1;
    float* my_scratch = scratch + threadIdx.x * kScratchStride;
    const int warp_j_hi = i0 + (warp & 3) * 32 - a.window - 1;
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
    for (int it = 0; it < ntx; ++it) {
      const int sb = it % kSBuf;
      ok = ok && mbar_wait(s_full + qt * kSBuf + sb, (it / kSBuf) & 1, abort_flag, a.status, 25);
      tc_fence_after();
      const int j0 = (u_lo + it) * kTile;
      const bool interior = (j0 >= a.n_start) && (j0 + kTile - 1 <= warp_j_hi);
      const int c_lo = max(0, a.n_start - j0);
      const int c_hi = min(kTile - 1, j_hi - j0);
      // the row's 128 scores in two halves of 64 (keeps the scan within its
      // register budget); the TMEM buffer goes back to the MMA warp as soon
      // as the second half is in registers
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        float v[64];
        tmem_ld32(tmem + (qt * kSBuf + sb) * 128 + lane_off + hf * 64, v);
        tmem_ld32(tmem + (qt * kSBuf + sb) * 128 + lane_off + hf * 64 + 32, v + 32);
        tc_wait_ld();
        if (hf == 1) {
          tc_fence_before();
          if (ok) mbar_arrive(s_free + qt * kSBuf + sb);
        }
        if (!interior || flags) {
#pragma unroll
          for (int c2 = 0; c2 < 2; ++c2) {
            const int cb = hf * 64 + c2 * 32;  // first column of this 32-column chunk
            uint32_t sepm = 0;
            if (flags) {
              const int jj = j0 + cb + lane;
              sepm = __ballot_sync(0xffffffffu, jj < a.T && flags[jj] != 0);
            }
            const int lo = max(c_lo - cb, 0);
            const int hi = min(c_hi - cb, 31);
            uint32_t vm = 0;
            if (lo <= hi) vm = (hi == 31 ? 0xffffffffu : ((1u << (hi + 1)) - 1u)) & ~((1u << lo) - 1u);
            vm &= ~sepm;
            ncand += __popc(vm);
#pragma unroll
            for (int y = 0; y < 32; ++y) v[c2 * 32 + y] = ((vm >> y) & 1u) ? v[c2 * 32 + y] : -CUDART_INF_F;
          }
        } else {
          ncand += 64;
        }
        // per 32-column chunk maxima (independent chains), then the insertion
        // path only for chunks that beat the row's current threshold; such a
        // chunk goes through this thread's shared scratch row, so one copy of
        // the insertion code serves every column (an unrolled insertion per
        // column would not fit the instruction cache)
#pragma unroll
        for (int c2 = 0; c2 < 2; ++c2) {
          float pm[8];
#pragma unroll
          for (int y = 0; y < 8; ++y) pm[y] = v[c2 * 32 + y];
#pragma unroll
          for (int y = 8; y < 32; ++y) pm[y & 7] = fmaxf(pm[y & 7], v[c2 * 32 + y]);
          const float cm =
              fmaxf(fmaxf(fmaxf(pm[0], pm[1]), fmaxf(pm[2], pm[3])), fmaxf(fmaxf(pm[4], pm[5]), fmaxf(pm[6], pm[7])));
          if (cm > vals[KC - 1]) {
            uint32_t msk = 0;
#pragma unroll
            for (int y = 0; y < 32; ++y) {
              my_scratch[y] = v[c2 * 32 + y];
              msk |= (v[c2 * 32 + y] > vals[KC - 1]) ? (1u << y) : 0u;
            }
            while (msk) {
              const int y = __ffs(msk) - 1;
              msk &= msk - 1;
              const float z = my_scratch[y];
              if (z > vals[KC - 1]) list_insert<KC>(z, j0 + hf * 64 + c2 * 32 + y, vals, idxs);
            }
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
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------------------
// pass 2: exact re-rank of the shortlist + certificate
// ---------------------------------------------------------------------------
// A group of KC lanes per row (KC = shortlist length, 16 or 32): the group
// stages the row's fp32 scoring query (R(L) q when capped, R(i) q otherwise)
// in shared memory, lane x recomputes the fp32 logit of shortlist entry x
// from the exact inputs (16-byte key loads), and a bitonic network over the
// group's lanes orders the entries by (logit desc, j asc).  The certificate:
// every key left out of the shortlist has a coarse score <= the row's
// threshold (the last shortlisted coarse score), and a coarse score differs
// from the fp32 logit by at most eps (query rounding ||q - bf16(q)|| * max||k||,
// accumulation, and for rotated keys their rounding), so the top k are exact
// when the k-th re-ranked logit exceeds threshold + eps.
template <int D, int KC>
__global__ void __launch_bounds__(256) topk_rerank_kernel(const TopkArgs a) {
  constexpr int half = D / 2;
  constexpr int RPB = 256 / KC;          // rows per block
  constexpr int PPL = half / KC;         // rotary pairs staged per lane (2 or 4 for d=128)
  __shared__ __align__(16) float sq[RPB][D];
  const int grp = threadIdx.x / KC, x = threadIdx.x % KC;
  const int lane = threadIdx.x & 31;
  const unsigned gmask = (KC == 32) ? 0xffffffffu : (0xffffu << (lane & 16));
  const int64_t nrows = (int64_t)a.B * a.Hq * a.T;
  const int64_t row_raw = (int64_t)blockIdx.x * RPB + grp;
  const bool live = row_raw < nrows;
  const int64_t row = live ? row_raw : nrows - 1;  // dead groups compute a copy and write nothing
  const int i = (int)(row % a.T);
  const int64_t bh = row / a.T;
  const int h = (int)(bh % a.Hq), b = (int)(bh / a.Hq);
  const int g = h / (a.Hq / a.Hkv);
  const bool capped_all = a.L > 0;  // capped scoring requires L == window: every candidate is capped
  const __nv_bfloat16* qp = reinterpret_cast<const __nv_bfloat16*>(a.Q) + b * a.q_sb + h * a.q_sh +
                            (int64_t)i * a.q_st;
  // stage the scoring query and measure its bf16 rounding
  float dq2 = 0.f, qn2 = 0.f;
#pragma unroll
  for (int e = 0; e < PPL; ++e) {
    const int c = x * PPL + e;
    const float x0 = __bfloat162float(qp[c]), x1 = __bfloat162float(qp[c + half]);
    const int64_t pos = capped_all ? a.L : i;
    const float2 cs = a.tab ? a.tab[pos * half + c] : make_float2(1.f, 0.f);
    const float u0 = x0 * cs.x - x1 * cs.y, u1 = x1 * cs.x + x0 * cs.y;
    sq[grp][c] = u0;
    sq[grp][c + half] = u1;
    const float b0 = __bfloat162float(__float2bfloat16_rn(u0)), b1 = __bfloat162float(__float2bfloat16_rn(u1));
    dq2 += (u0 - b0) * (u0 - b0) + (u1 - b1) * (u1 - b1);
    qn2 += b0 * b0 + b1 * b1;
  }
#pragma unroll
  for (int o = KC / 2; o > 0; o >>= 1) {
    dq2 += __shfl_xor_sync(gmask, dq2, o);
    qn2 += __shfl_xor_sync(gmask, qn2, o);
  }
  __syncwarp();
  const float kmax = __uint_as_float(a.kmax[(size_t)b * a.Hkv + g]) * (1.f + 1.f / 128.f);
  const float qn = sqrtf(qn2);
  float eps = sqrtf(dq2) * kmax + qn * kmax * (1.f / 32768.f);
  if (!capped_all) eps += qn * kmax * (1.f / 256.f);  // rotated keys were rounded too
  eps *= 1.0625f;

  // lane x: fp32 logit of shortlist entry x
  const int j = a.short_idx[row * KC + x];
  float z = -CUDART_INF_F;
  if (j >= 0) {
    const __nv_bfloat16* kp = reinterpret_cast<const __nv_bfloat16*>(a.K) + b * a.k_sb + g * a.k_sh +
                              (int64_t)j * a.k_st;
    const float* qv = sq[grp];
    float A0 = 0.f, A1 = 0.f;
#pragma unroll
    for (int c0 = 0; c0 < half; c0 += 8) {
      float k0[8], k1[8];
      const uint4 lo = *reinterpret_cast<const uint4*>(kp + c0);
      const uint4 hi = *reinterpret_cast<const uint4*>(kp + c0 + half);
      const __nv_bfloat162* l2 = reinterpret_cast<const __nv_bfloat162*>(&lo);
      const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&hi);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 p = __bfloat1622float2(l2[e]), r = __bfloat1622float2(h2[e]);
        k0[2 * e] = p.x;
        k0[2 * e + 1] = p.y;
        k1[2 * e] = r.x;
        k1[2 * e + 1] = r.y;
      }
      if (!capped_all && a.tab) {
        const float4* t = reinterpret_cast<const float4*>(a.tab + (int64_t)j * half + c0);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float4 cs = t[e];
          const float a0 = k0[2 * e], a1 = k0[2 * e + 1], r0 = k1[2 * e], r1 = k1[2 * e + 1];
          k0[2 * e] = a0 * cs.x - r0 * cs.y;
          k1[2 * e] = r0 * cs.x + a0 * cs.y;
          k0[2 * e + 1] = a1 * cs.z - r1 * cs.w;
          k1[2 * e + 1] = r1 * cs.z + a1 * cs.w;
        }
      }
#pragma unroll
      for (int e = 0; e < 8; e += 2) {
        fma2(A0, A1, qv[c0 + e], qv[c0 + e + 1], k0[e], k0[e + 1], A0, A1);
        fma2(A0, A1, qv[half + c0 + e], qv[half + c0 + e + 1], k1[e], k1[e + 1], A0, A1);
      }
    }
    z = A0 + A1;
  }
  // bitonic sort over the group's lanes: (z desc, j asc), invalid (j < 0) last
  int jj = j;
#pragma unroll
  for (int k = 2; k <= KC; k <<= 1) {
#pragma unroll
    for (int o = k >> 1; o > 0; o >>= 1) {
      const float oz = __shfl_xor_sync(gmask, z, o);
      const int oj = __shfl_xor_sync(gmask, jj, o);
      // does the partner's entry come before ours in the order?
      const bool other_first = (oj >= 0) && (jj < 0 || oz > z || (oz == z && oj < jj));
      const bool mine_first = (jj >= 0) && (oj < 0 || z > oz || (z == oz && jj < oj));
      // in a run of ascending rank the lower lane of a pair keeps the earlier entry
      const bool want_earlier = ((x & o) == 0) == ((x & k) == 0);
      const bool take = want_earlier ? other_first : mine_first;
      if (take) {
        z = oz;
        jj = oj;
      }
    }
  }
  const int n = a.n_cand[row];
  const float thr = a.short_thr[row];
  const int k = a.topk;
  const float zk = __shfl_sync(gmask, z, (lane & ~(KC - 1)) + k - 1);
  const bool certified = (n <= KC) || (zk > thr + eps);
  if (!live) return;
  if (certified) {
    if (x < k) {
      a.idx[row * k + x] = (x < n) ? jj : -1;
      a.z[row * k + x] = (x < n) ? z : -CUDART_INF_F;
    }
  } else if (x == 0) {
    const int pos = atomicAdd(a.status + 2, 1);
    a.fallback_rows[pos] = (int32_t)row;
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
  const size_t bytes = std::max<size_t>(116 * 1024, 1024 + tile * (2 + kStages) + 1024 + 256 * kScratchStride * 4);
  cudaError_t e = cudaFuncSetAttribute(topk_score_kernel<D, KC>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e != cudaSuccess) return e;
  const int nQB = (a.nQT + 1) / 2;
  topk_score_kernel<D, KC><<<(unsigned)(a.B * a.Hq * nQB), kThreads, bytes, st>>>(m.qsel, m.ksel, a, nQB);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int64_t rows = (int64_t)a.B * a.Hq * a.T;
  const unsigned blocks = (unsigned)((rows * KC + 255) / 256);
  topk_rerank_kernel<D, KC><<<blocks, 256, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_topk_tc(const TopkArgs& a, const TopkMaps& m, cudaStream_t st) {
  if ((int64_t)a.B * a.Hq * a.T == 0) return cudaSuccess;
  if (a.d == 128) {
    if (a.short_len == 16) return launch_score<128, 16>(a, m, st);
    if (a.short_len == 32) return launch_score<128, 32>(a, m, st);
  } else if (a.d == 64) {
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
