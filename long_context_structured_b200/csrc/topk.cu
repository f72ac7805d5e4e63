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
//     multiplied into both tiles' TMEM score buffers (with the window below
//     the cap, one query tile per CTA whose two slots hold R(L)q and R(i)q,
//     a key tile straddling the cap scored against both).  A sample of the key
//     tiles is scored first and sets each row's threshold tau; then every
//     candidate tile is scored and each key whose coarse score exceeds tau
//     is appended to the row's candidate list (kCandCap entries);
//  2. exact re-rank: a warp per row recomputes the listed keys' logits in
//     fp32 from the exact inputs, takes the top k and certifies them: every
//     key left out has a coarse score <= tau, and a coarse score differs from
//     the fp32 logit by at most eps (operand rounding bound ||q - bf16(q)|| *
//     max||k|| plus the accumulation bound), so the top k are exact when the
//     k-th fp32 logit exceeds tau + eps;
//  3. rows that fail the certificate or overflow their list (rare) are
//     rescanned exactly in fp32 over all their candidates.
#include <cuda_bf16.h>

#include <type_traits>
#include <math_constants.h>

#include "kernels.cuh"
#include "select.cuh"
#include "simt.cuh"
#include "sm100.cuh"

namespace sattn {

namespace {

constexpr int kThreads = 576;  // 16 scan warps (two query tiles x two column halves), TMA warp, MMA warp
constexpr int kTmaWarp = 16, kMmaWarp = 17;
constexpr int kSBuf = 2;       // TMEM score buffers per query tile

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

// ---------------------------------------------------------------------------
// pass 1: tensor-core scoring with a per-row candidate list
// ---------------------------------------------------------------------------
// Key tiles are scored in two phases.  The sample phase scores every
// stride-th key tile of the row's candidate range and keeps, per row, the 16
// largest group maxima; the r-th of them becomes the row's threshold tau.
// With a sample of 1/stride of the row, about r * stride candidates score
// above the r-th largest 32-column chunk maximum (a Gamma(r)-distributed
// count, scaled by the stride); the (stride, r) pairs below keep both "fewer
// than about seven above tau" (the certificate would fail) and "more than
// kCandCap above tau" (the list would overflow) near or below 0.03% of rows,
// each of which then takes the exact rescan.  CTAs with few key tiles sample
// every tile and take groups of 4 columns (the y = g mod 8 columns of a
// 32-column chunk): the 16th largest group maximum leaves at least 15 and at
// most 15 * 4 keys above it, so the list never overflows.  The main phase
// scores every candidate tile in key order and appends each key above tau to
// the row's list: per 32-column chunk a thread first takes the chunk
// maximum, and only when some row of the warp has a chunk maximum above its
// threshold does the warp build bit masks and append.
constexpr int kSampleKeep = 16;  // group maxima kept per row in the sample phase
constexpr int kStagesK = 2;      // K tiles in flight
// floats per scan thread's scratch row: a multiple of 4 (16-byte stores) that
// puts the eight rows of a quarter-warp on distinct bank groups
constexpr int kScratchStride = 36;

// Sample stride and rank for a CTA whose longer query tile scans `ntiles`
// key tiles; `fine`: 4-column groups instead of 32-column chunks.
__device__ __forceinline__ void sample_plan(int ntiles, int& stride, int& r, bool& fine) {
  fine = false;
  if (ntiles >= 48) { stride = 6; r = 8; }
  else if (ntiles >= 16) { stride = 3; r = 12; }
  else { stride = 1; r = 16; fine = true; }
}

// max of three (one instruction on sm_100)
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// (m << 2) | [v_hi > t] << 1 | [v_lo > t]: t - v has its sign bit set exactly
// when v > t (t - v is +0 for v == t and a positive NaN for -inf - -inf); one
// packed subtraction for the pair, one funnel shift per bit
__device__ __forceinline__ uint32_t push_above2(uint32_t m, float v_lo, float v_hi, unsigned long long tt) {
  uint32_t r;
  asm("{\n\t.reg .b64 t, d;\n\t.reg .b32 lo, hi;\n\t"
      "mov.b64 t, {%2, %3};\n\t"
      "sub.rn.f32x2 d, %4, t;\n\t"
      "mov.b64 {lo, hi}, d;\n\t"
      "shf.l.clamp.b32 %0, hi, %1, 1;\n\t"
      "shf.l.clamp.b32 %0, lo, %0, 1;\n\t}"
      : "=r"(r)
      : "r"(m), "f"(v_lo), "f"(v_hi), "l"(tt));
  return r;
}

// insert v into the descending list s (values only)
template <int R>
__device__ __forceinline__ void insert_val(float v, float (&s)[R]) {
#pragma unroll
  for (int x = 0; x < R; ++x) {
    if (v > s[x]) {
      const float t = s[x];
      s[x] = v;
      v = t;
    }
  }
}

// kDual (a cap with the window below it, 0 < w < L): candidates with
// i - j <= L take the uncapped logit <R(i) q, R(j) k>, the farther ones the
// capped <R(L) q, k>.  A CTA then takes ONE query tile and stages both of
// its scoring queries (Qc in the first query slot, Qr in the second); a key
// tile whose pairs are all capped is scored as Qc K^T, one whose pairs are
// all within the cap as Qr Kr^T, and a tile that straddles the cap both ways
// (two K ring entries, the products in the first and the idle second query
// tile's TMEM buffers), the scan warps taking each column from the product
// that holds its row's logit.
template <int D, bool kDual>
__global__ void __launch_bounds__(kThreads, 1)
    topk_score_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmQ2, const __grid_constant__ CUtensorMap tmK2,
                      const TopkArgs a, int nQB) {
  constexpr int kSt = kStagesK;
  constexpr int kR = kSampleKeep;
  constexpr uint32_t kTileBytes = D * kTile * 2;
  constexpr int kChunks = D / 64;
  constexpr uint32_t kChunkBytes = kTile * 128;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sq = base;  // Q0 | Q1
  uint8_t* sk = base + 2 * kTileBytes;  // kSt K tiles
  float* scratch = reinterpret_cast<float*>(sk + kSt * kTileBytes);  // [512 scan threads][kScratchStride]
  int* rcnt = reinterpret_cast<int*>(scratch + 512 * kScratchStride);  // [256 rows] keys above tau
  uint64_t* bars = reinterpret_cast<uint64_t*>(rcnt + 256);
  uint64_t* q_full = bars;
  uint64_t* k_full = bars + 1;
  uint64_t* k_empty = k_full + kSt;
  uint64_t* s_full = k_empty + kSt;  // [2 tiles][kSBuf]
  uint64_t* s_free = s_full + 2 * kSBuf;  // [2 tiles][kSBuf]
  uint64_t* drain = s_free + 2 * kSBuf;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  int* abort_i = reinterpret_cast<int*>(tmem_slot + 1);
  int* early = abort_i + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qb = blockIdx.x % nQB;
  const int bh = blockIdx.x / nQB;
  const int h = bh % a.Hq, b = bh / a.Hq;
  const int g = h / (a.Hq / a.Hkv);
  // query tiles of this CTA: 2 qb and 2 qb + 1, or the one tile qb (kDual)
  auto qtile = [&](int x) { return kDual ? qb : 2 * qb + x; };
  // key tiles each query tile scans: [u_lo, u_lo + nt[x]); the union is the longer
  const int u_lo = a.n_start / kTile;
  int nt[2];
  for (int x = 0; x < 2; ++x) {
    const int i0x = qtile(x) * kTile;
    nt[x] = 0;
    if ((!kDual || x == 0) && i0x < a.T) {
      const int hi_key = min(a.T - 1, i0x + kTile - 1) - a.window - 1;
      if (hi_key >= a.n_start) nt[x] = hi_key / kTile - u_lo + 1;
    }
  }
  const int ntiles = max(nt[0], nt[1]);
  // step sequence: the sample tiles 0, S, 2S, ... then every tile in order
  int stride, r_tau;
  bool fine;
  sample_plan(ntiles, stride, r_tau, fine);
  const int n_s = (ntiles + stride - 1) / stride;
  const int n_steps = ntiles > 0 ? n_s + ntiles : 0;
  auto tile_of = [&](int it) { return it < n_s ? it * stride : it - n_s; };
  // kDual: 0 = every pair of the key tile capped, 1 = every pair within the
  // cap, 2 = both (rows past the sequence end count as rows; they keep nothing)
  auto ttype = [&](int t) -> int {
    if (!kDual) return 0;
    const int i0d = qb * kTile;
    const int j0 = (u_lo + t) * kTile;
    if (i0d - (j0 + kTile - 1) > a.L) return 0;
    if (i0d + kTile - 1 - j0 <= a.L) return 1;
    return 2;
  };

  if (threadIdx.x == 0) {
    *early = status_failed(a.status) ? 1 : 0;
    *abort_i = 0;
    mbar_init(q_full, 1);
    for (int s = 0; s < kSt; ++s) {
      mbar_init(k_full + s, 1);
      mbar_init(k_empty + s, 1);
    }
    for (int s = 0; s < 2 * kSBuf; ++s) {
      mbar_init(s_full + s, 1);
      mbar_init(s_free + s, 256);  // both column halves of the tile's 128 rows
    }
    mbar_init(drain, 1);
    fence_mbar_init();
  }
  for (int x = threadIdx.x; x < 256; x += blockDim.x) rcnt[x] = 0;
  __syncthreads();
  if (*early) return;
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  volatile int* abort_flag = abort_i;

  if (warp == kTmaWarp) {
    // ===== TMA producer: both query tiles once, then the K ring =====
    if (lane == 0 && n_steps > 0) {
      mbar_expect_tx(q_full, 2 * kTileBytes);
      for (int x = 0; x < 2; ++x)
        for (int c = 0; c < kChunks; ++c)
          tma_load_4d(sq + x * kTileBytes + c * kChunkBytes, (kDual && x == 1) ? &tmQ2 : &tmQ, q_full, c * 64,
                      qtile(x) * kTile, h, b);
      // ring entries: one K tile per step (raw K, or Kr for a tile within
      // the cap), two for a straddling tile (raw K, then Kr)
      int issued = 0;
      bool ok = true;
      for (int it = 0; it < n_steps && ok; ++it) {
        const int ty = ttype(tile_of(it));
        for (int e = 0; e < (ty == 2 ? 2 : 1); ++e) {
          const int st = issued % kSt;
          if (issued >= kSt) ok = mbar_wait(k_empty + st, ((issued / kSt) - 1) & 1, abort_flag, a.status, 21);
          if (!ok) break;
          mbar_expect_tx(k_full + st, kTileBytes);
          const CUtensorMap* km = (ty == 1 || e == 1) ? &tmK2 : &tmK;
          for (int c = 0; c < kChunks; ++c)
            tma_load_4d(sk + st * kTileBytes + c * kChunkBytes, km, k_full + st, c * 64,
                        (u_lo + tile_of(it)) * kTile, g, b);
          ++issued;
        }
      }
      if (!ok) {
        mbar_wait_raw(q_full, 0);
        for (int it = max(0, issued - kSt); it < issued; ++it) mbar_wait_raw(k_full + it % kSt, (it / kSt) & 1);
      }
    }
  } else if (warp == kMmaWarp) {
    // ===== MMA issuer: per K tile, S_x = Q_x K^T for each query tile that needs it =====
    if (lane == 0 && n_steps > 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(128, 128, false);
      const uint32_t q_addr = smem_u32(sq);
      bool ok = mbar_wait(q_full, 0, abort_flag, a.status, 22);
      int cnt[2] = {0, 0};  // score tiles produced per query tile
      int used = 0;         // K ring entries consumed
      auto mma_tile = [&](uint32_t d_tmem, uint32_t qa, uint32_t ka) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * kChunkBytes + (kk & 3) * 32;
          tc_mma_ss(d_tmem, smem_desc_sw128(qa + off, 16, 1024), smem_desc_sw128(ka + off, 16, 1024), idesc,
                    kk > 0 ? 1u : 0u);
        }
      };
      for (int it = 0; it < n_steps && ok; ++it) {
        const int t = tile_of(it);
        const int ty = ttype(t);
        const int st = used % kSt, st2 = (used + 1) % kSt;
        ok = mbar_wait(k_full + st, (used / kSt) & 1, abort_flag, a.status, 23);
        if (ok && ty == 2) ok = mbar_wait(k_full + st2, ((used + 1) / kSt) & 1, abort_flag, a.status, 23);
        if (!ok) break;
        const uint32_t k_addr = smem_u32(sk + st * kTileBytes);
        for (int x = 0; x < (kDual ? 1 : 2) && ok; ++x) {
          if (t >= nt[x]) continue;
          const int c = cnt[x]++;
          const int sb = c % kSBuf;
          if (c >= kSBuf) ok = mbar_wait(s_free + x * kSBuf + sb, ((c / kSBuf) - 1) & 1, abort_flag, a.status, 24);
          if (!ok) break;
          tc_fence_after();
          // the query slot: the tile's own, or in kDual Qc (slot 0) / Qr (slot 1)
          const int slot = kDual ? (ty == 1 ? 1 : 0) : x;
          mma_tile(tmem + (x * kSBuf + sb) * 128, q_addr + slot * kTileBytes, k_addr);
          if (kDual && ty == 2)  // the within-cap product into the idle second tile's buffer
            mma_tile(tmem + (kSBuf + sb) * 128, q_addr + kTileBytes, smem_u32(sk + st2 * kTileBytes));
          tc_commit(s_full + x * kSBuf + sb);
        }
        tc_commit(k_empty + st);
        if (ty == 2) tc_commit(k_empty + st2);
        used += ty == 2 ? 2 : 1;
      }
      tc_commit(drain);
      mbar_wait_raw(drain, 0);
    }
    __syncwarp();
  } else if (warp < 16 && !(kDual && ((warp >> 2) & 1))) {
    // scan warps: warp w scans query tile qt = (w / 4) % 2, rows 32 (w % 4)
    // .. + 31 of it (TMEM lanes of the warp's quarter), columns 64 ch .. + 63
    // of every key tile, ch = w / 8; the two threads of a row (warps w and
    // w ^ 8) share the row's threshold and its candidate list (kDual: the
    // second tile's warps idle)
    const int qt = (warp >> 2) & 1;
    const int ch = warp >> 3;
    const int rl = (warp & 3) * 32 + lane;  // row within the query tile
    const int i0 = qtile(qt) * kTile;
    const int i = i0 + rl;
    const int ntx = nt[qt];
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    // candidates of this row: n_start <= j <= i - w - 1; of the warp's rows,
    // the smallest upper bound decides which tiles need no per-column mask
    // (rows past the sequence end keep nothing)
    const int j_hi = i < a.T ? i - a.window - 1 : -1;
    const int warp_j_hi = (i0 + (warp & 3) * 32 + 31 < a.T) ? i0 + (warp & 3) * 32 - a.window - 1 : -1;
    const size_t row = ((size_t)b * a.Hq + h) * a.T + (i < a.T ? i : a.T - 1);
    int2* list = a.cand_idx + row * kCandCap;
    int* my_cnt = rcnt + qt * 128 + rl;
    float* my_scratch = scratch + (threadIdx.x & 511) * kScratchStride;
    const float* partner_scratch = scratch + ((threadIdx.x ^ 256) & 511) * kScratchStride;
    const int bar_id = 1 + qt;  // named barrier of the query tile's 256 scan threads
    float samp[kR];
#pragma unroll
    for (int x = 0; x < kR; ++x) samp[x] = -CUDART_INF_F;
    float tau = -CUDART_INF_F;
    int cx = 0; // score tiles consumed
    bool ok = true;
    const uint8_t* flags = a.is_sep ? a.is_sep + (size_t)b * a.T : nullptr;
    for (int it = 0; it < n_steps; ++it) {
      if (it == n_s) {
        // end of the sample phase: tau = the r-th largest of the maxima both
        // halves of the row sampled (a merge of the two sorted lists)
#pragma unroll
        for (int x = 0; x < kR; ++x) my_scratch[x] = samp[x];
        asm volatile("bar.sync %0, 256;" ::"r"(bar_id) : "memory");
        int pa = 0, pb = 0;
        float other = partner_scratch[0];
        for (int x = 0; x < r_tau; ++x) {
          float mine = -CUDART_INF_F;
#pragma unroll
          for (int y = 0; y < kR; ++y)
            if (y == pa) mine = samp[y];
          if (mine >= other) {
            tau = mine;
            ++pa;
          } else {
            tau = other;
            ++pb;
            other = pb < kR ? partner_scratch[pb] : -CUDART_INF_F;
          }
        }
        asm volatile("bar.sync %0, 256;" ::"r"(bar_id) : "memory");  // scratch rows are reused below
      }
      const int t = tile_of(it);
      if (t >= ntx) continue;
      const int ty = ttype(t);
      const bool sample = it < n_s;
      const int sb = cx % kSBuf;
      ok = ok && mbar_wait(s_full + qt * kSBuf + sb, (cx / kSBuf) & 1, abort_flag, a.status, 25);
      ++cx;
      tc_fence_after();
      const int j0 = (u_lo + t) * kTile;
      const bool interior = (j0 >= a.n_start) && (j0 + kTile - 1 <= warp_j_hi);
      const int c_lo = max(0, a.n_start - j0);
      const int c_hi = min(kTile - 1, j_hi - j0);
      // this thread's 64 columns as two chunks of 32; the TMEM buffer goes
      // back to the MMA warp once the second chunk is in registers
#pragma unroll
      for (int c2 = 0; c2 < 2; ++c2) {
        const int cb = ch * 64 + c2 * 32;  // first column of this 32-column chunk
        float v[32];
        const uint32_t tb = tmem + (qt * kSBuf + sb) * 128 + lane_off + cb;
        if (kDual && ty == 2) {
          // columns j >= i - L hold their logit in the second product
          const int yc = i - a.L - (j0 + cb);
          if (__all_sync(0xffffffffu, yc <= 0)) {
            tmem_ld32(tb + kSBuf * 128, v);
            tc_wait_ld();
          } else {
            tmem_ld32(tb, v);
            if (__any_sync(0xffffffffu, yc < 32)) {
#pragma unroll
              for (int hh = 0; hh < 2; ++hh) {
                float w16[16];
                tmem_ld16(tb + kSBuf * 128 + 16 * hh, w16);
                tc_wait_ld();
#pragma unroll
                for (int y = 0; y < 16; ++y)
                  if (16 * hh + y >= yc) v[16 * hh + y] = w16[y];
              }
            } else {
              tc_wait_ld();
            }
          }
        } else {
          tmem_ld32(tb, v);
          tc_wait_ld();
        }
        if (c2 == 1) {
          tc_fence_before();
          if (ok) mbar_arrive(s_free + qt * kSBuf + sb);
        }
        if (!interior || flags) {
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
#pragma unroll
          for (int y = 0; y < 32; ++y) v[y] = ((vm >> y) & 1u) ? v[y] : -CUDART_INF_F;
        }
        // group maxima pm[g] over columns g, g + 8, g + 16, g + 24, then the chunk maximum
        float pm[8];
#pragma unroll
        for (int y = 0; y < 8; ++y) pm[y] = fmaxf(fmax3(v[y], v[y + 8], v[y + 16]), v[y + 24]);
        const float cm = fmax3(fmax3(pm[0], pm[1], pm[2]), fmax3(pm[3], pm[4], pm[5]), fmaxf(pm[6], pm[7]));
        if (sample) {
          if (fine) {
#pragma unroll
            for (int y = 0; y < 8; ++y)
              if (pm[y] > samp[kR - 1]) insert_val<kR>(pm[y], samp);
          } else if (cm > samp[kR - 1]) {
            insert_val<kR>(cm, samp);
          }
          continue;
        }
        if (__any_sync(0xffffffffu, cm > tau) && cm > tau) {
          // append this row's keys above tau with their coarse scores (the
          // chunk goes through the thread's scratch row so that a score can
          // be picked by a run-time column)
          const unsigned long long tt = (unsigned long long)__float_as_uint(tau) << 32 | __float_as_uint(tau);
          // bit y: column y above tau (four independent 8-bit chains)
          uint32_t mq[4] = {0u, 0u, 0u, 0u};
#pragma unroll
          for (int y = 7; y > 0; y -= 2)
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) mq[q4] = push_above2(mq[q4], v[8 * q4 + y - 1], v[8 * q4 + y], tt);
          uint32_t m = mq[0] | mq[1] << 8 | mq[2] << 16 | mq[3] << 24;
#pragma unroll
          for (int q4 = 0; q4 < 8; ++q4)
            reinterpret_cast<float4*>(my_scratch)[q4] =
                make_float4(v[4 * q4], v[4 * q4 + 1], v[4 * q4 + 2], v[4 * q4 + 3]);
          const int jbase = j0 + cb;
          while (m) {
            const int y = __ffs(m) - 1;
            m &= m - 1;
            const int pos = atomicAdd(my_cnt, 1);
            if (pos < kCandCap) list[pos] = make_int2(jbase + y, __float_as_int(my_scratch[y]));
          }
        }
      }
    }
    asm volatile("bar.sync %0, 256;" ::"r"(bar_id) : "memory");  // both halves have appended
    if (ch == 0 && i < a.T) {
      a.cand_thr[row] = tau;
      a.cand_cnt[row] = *my_cnt;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// fp32 logit of key row kp (bf16, unrotated) against the staged fp32 query qv
// (R(L) q when `capped`, else R(i) q, whose partner is the key rotated by
// R(j) from the table); 16-byte key loads, two accumulators
template <int HALF>
__device__ __forceinline__ float exact_logit_bf16(const __nv_bfloat16* kp, const float* qv, bool capped,
                                                  const float2* tab, int64_t j) {
  float A0 = 0.f, A1 = 0.f;
#pragma unroll
  for (int c0 = 0; c0 < HALF; c0 += 8) {
    float k0[8], k1[8];
    const uint4 lo = *reinterpret_cast<const uint4*>(kp + c0);
    const uint4 hi = *reinterpret_cast<const uint4*>(kp + c0 + HALF);
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
    if (!capped && tab) {
      const float4* t = reinterpret_cast<const float4*>(tab + j * HALF + c0);
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
      fma2(A0, A1, qv[HALF + c0 + e], qv[HALF + c0 + e + 1], k1[e], k1[e + 1], A0, A1);
    }
  }
  return A0 + A1;
}

// ---------------------------------------------------------------------------
// pass 2: exact re-rank of the candidate list + certificate
// ---------------------------------------------------------------------------
// Per row: a coarse score c differs from the key's fp32 logit z by at
// most eps (query rounding ||q - bf16(q)|| * max||k||, accumulation, and for
// rotated keys their rounding).  If c' <= the k-th largest coarse score of the
// list, at least k listed keys have z >= c' - eps, so the k-th fp32 logit
// z_(k) >= c' - eps and only listed keys with c >= c' - 2 eps can be among the
// top k.  c' is the k-th largest of the lanes' maxima (k distinct entries are
// >= it).  The row's lanes compact the entries above the cut into shared memory,
// recomputes their logits in fp32 from the exact inputs (four lanes per key,
// each a quarter of the rotary pairs, 16-byte key loads; the row's fp32
// scoring query, R(L) q when capped and R(i) q otherwise, staged in shared
// memory), and ranks them by (logit desc, j asc) by counting.  Certificate:
// every key left out of the list has a coarse score <= tau, hence
// z <= tau + eps; the top k are exact when z_(k) > tau + eps (or tau = -inf:
// the list holds every candidate).  Rows that fail, or whose list overflowed,
// go to the exact rescan.
// kRerankG lanes per row, 32 / kRerankG rows per warp: the per-row work that
// does not grow with the list (the k rounds that find c', the query staging
// and its rounding measure, the ranking, the certificate) is shared by the
// warp's rows per instruction; every shuffle stays inside its lane group.
constexpr int kRerankG = 16;                   // lanes per row (8 measured slower: 0.94 vs 0.74 ms)
constexpr int kRerankRows = 12;                // rows per block (the dual case's static shared memory < 48 KB)
constexpr int kRerankWarps = kRerankRows * kRerankG / 32;
constexpr int kPerLane = kCandCap / kRerankG;
static_assert(kRerankRows * kRerankG % 32 == 0 && kCandCap % kRerankG == 0, "re-rank tiling");

template <int D, bool kDual>
__global__ void __launch_bounds__(kRerankWarps * 32) topk_rerank_kernel(const TopkArgs a) {
  constexpr int half = D / 2;
  constexpr int G = kRerankG;
  constexpr int PPL = half / G;    // rotary pairs staged per lane
  constexpr int QP = half / 4;     // rotary pairs per lane of a 4-lane group
  __shared__ __align__(16) float sq[kRerankRows][D];
  __shared__ __align__(16) float sqc[kDual ? kRerankRows : 1][kDual ? D : 4];  // R(L) q when 0 < w < L
  __shared__ int sj[kRerankRows][kCandCap];
  __shared__ float2 se[kRerankRows][kCandCap];
  const int wid = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int grp = lane / G, gl = lane % G;  // the row group of the lane and its lane in it
  const int slot = (32 / G) * wid + grp;
  const uint32_t lt = (1u << gl) - 1u;        // this lane's predecessors in its group
  auto group_bits = [&](uint32_t ballot) { return (ballot >> (G * grp)) & ((1u << G) - 1u); };
  const int64_t nrows = (int64_t)a.B * a.Hq * a.T;
  const int64_t row0 = (int64_t)blockIdx.x * kRerankRows + slot;
  const bool live = row0 < nrows;  // both groups of a warp take part in every shuffle
  const int64_t row = live ? row0 : nrows - 1;
  const int i = (int)(row % a.T);
  const int64_t bh = row / a.T;
  const int h = (int)(bh % a.Hq), b = (int)(bh / a.Hq);
  const int g = h / (a.Hq / a.Hkv);
  // w >= L: every candidate is capped; 0 < w < L: those with i - j <= L are not
  constexpr bool dual = kDual;  // the launch picks it: a.L > 0 && a.window < a.L
  const bool capped_all = a.L > 0 && !dual;
  const int cnt = live ? a.cand_cnt[row] : 0;
  const float tau = a.cand_thr[row];
  const int k = a.topk;
  const int n = min(cnt, kCandCap);
  const int2* list = a.cand_idx + row * kCandCap;
  float c[kPerLane];
  int jl[kPerLane];
  float lm = -CUDART_INF_F;
#pragma unroll
  for (int x = 0; x < kPerLane; ++x) {
    const int e = gl + G * x;
    jl[x] = -1;
    c[x] = -CUDART_INF_F;
    if (e < n) {
      const int2 v = list[e];
      jl[x] = v.x;
      c[x] = __int_as_float(v.y);
      lm = fmaxf(lm, c[x]);
    }
  }
  const __nv_bfloat16* qp = reinterpret_cast<const __nv_bfloat16*>(a.Q) + b * a.q_sb + h * a.q_sh +
                            (int64_t)i * a.q_st;
  // stage the scoring query (and with 0 < w < L the capped one as well) and
  // measure their bf16 rounding
  float dq2 = 0.f, qn2 = 0.f, dq2c = 0.f, qn2c = 0.f;
#pragma unroll
  for (int e = 0; e < PPL; ++e) {
    const int cc = gl * PPL + e;
    const float x0 = __bfloat162float(qp[cc]), x1 = __bfloat162float(qp[cc + half]);
    const int64_t pos = capped_all ? a.L : i;
    const float2 cs = a.tab ? a.tab[pos * half + cc] : make_float2(1.f, 0.f);
    const float u0 = x0 * cs.x - x1 * cs.y, u1 = x1 * cs.x + x0 * cs.y;
    sq[slot][cc] = u0;
    sq[slot][cc + half] = u1;
    const float b0 = __bfloat162float(__float2bfloat16_rn(u0)), b1 = __bfloat162float(__float2bfloat16_rn(u1));
    dq2 += (u0 - b0) * (u0 - b0) + (u1 - b1) * (u1 - b1);
    qn2 += b0 * b0 + b1 * b1;
    if constexpr (kDual) {
      const float2 cl = a.tab ? a.tab[(int64_t)a.L * half + cc] : make_float2(1.f, 0.f);
      const float w0 = x0 * cl.x - x1 * cl.y, w1 = x1 * cl.x + x0 * cl.y;
      sqc[slot][cc] = w0;
      sqc[slot][cc + half] = w1;
      const float c0 = __bfloat162float(__float2bfloat16_rn(w0)), c1 = __bfloat162float(__float2bfloat16_rn(w1));
      dq2c += (w0 - c0) * (w0 - c0) + (w1 - c1) * (w1 - c1);
      qn2c += c0 * c0 + c1 * c1;
    }
  }
#pragma unroll
  for (int o = G / 2; o > 0; o >>= 1) {
    dq2 += __shfl_xor_sync(0xffffffffu, dq2, o);
    qn2 += __shfl_xor_sync(0xffffffffu, qn2, o);
    if constexpr (kDual) {
      dq2c += __shfl_xor_sync(0xffffffffu, dq2c, o);
      qn2c += __shfl_xor_sync(0xffffffffu, qn2c, o);
    }
  }
  const float kmax = __uint_as_float(a.kmax[(size_t)b * a.Hkv + g]) * (1.f + 1.f / 128.f);
  const float qn = sqrtf(qn2);
  float eps = sqrtf(dq2) * kmax + qn * kmax * (1.f / 32768.f);
  if (!capped_all) eps += qn * kmax * (1.f / 256.f);  // rotated keys were rounded too
  if constexpr (kDual) {
    // the capped scores' bound (unrotated keys are exact)
    const float qnc = sqrtf(qn2c);
    eps = fmaxf(eps, sqrtf(dq2c) * kmax + qnc * kmax * (1.f / 32768.f));
  }
  eps *= 1.0625f;

  // c' = the k-th largest lane maximum of the group (-inf when fewer than k
  // lanes hold entries)
  float cp = -CUDART_INF_F;
  {
    float mv = lm;
    for (int r = 0; r < k; ++r) {
      float wz = mv;
#pragma unroll
      for (int o = G / 2; o > 0; o >>= 1) wz = fmaxf(wz, __shfl_xor_sync(0xffffffffu, wz, o));
      const uint32_t holders = group_bits(__ballot_sync(0xffffffffu, mv == wz));
      if (gl == __ffs(holders) - 1) mv = -CUDART_INF_F;
      cp = wz;
    }
  }
  // compact the entries that can reach the top k
  const float cut = cp - 2.f * eps;
  int m = 0;
#pragma unroll
  for (int x = 0; x < kPerLane; ++x) {
    const bool p = jl[x] >= 0 && c[x] >= cut;
    const uint32_t bal = group_bits(__ballot_sync(0xffffffffu, p));
    if (p) sj[slot][m + __popc(bal & lt)] = jl[x];
    m += __popc(bal);
  }
  __syncwarp();
  // fp32 logits: four lanes per entry, a quarter of the rotary pairs each;
  // both groups run the loop as often as the longer of the two needs
  int m_warp = m;
#pragma unroll
  for (int o = G; o < 32; o <<= 1) m_warp = max(m_warp, __shfl_xor_sync(0xffffffffu, m_warp, o));
  const __nv_bfloat16* kbase = reinterpret_cast<const __nv_bfloat16*>(a.K) + b * a.k_sb + g * a.k_sh;
  const int quarter = gl & 3;
  for (int e0 = 0; e0 < m_warp; e0 += G / 4) {
    const int e = e0 + (gl >> 2);
    float acc = 0.f;
    int j = -1;
    if (e < m) {
      j = sj[slot][e];
      // the pair's operands: capped (R(L) q, raw key) or rotated (R(i) q, R(j) k)
      bool cap = capped_all;
      const float* qv = sq[slot];
      if constexpr (kDual) {
        cap = i - j > a.L;
        if (cap) qv = sqc[slot];
      }
      const __nv_bfloat16* kp = kbase + (int64_t)j * a.k_st;
      float A0 = 0.f, A1 = 0.f;
#pragma unroll
      for (int c0 = quarter * QP; c0 < quarter * QP + QP; c0 += 8) {
        float k0[8], k1[8];
        const uint4 lo = *reinterpret_cast<const uint4*>(kp + c0);
        const uint4 hi = *reinterpret_cast<const uint4*>(kp + c0 + half);
        const __nv_bfloat162* l2 = reinterpret_cast<const __nv_bfloat162*>(&lo);
        const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&hi);
#pragma unroll
        for (int y = 0; y < 4; ++y) {
          const float2 p = __bfloat1622float2(l2[y]), r = __bfloat1622float2(h2[y]);
          k0[2 * y] = p.x;
          k0[2 * y + 1] = p.y;
          k1[2 * y] = r.x;
          k1[2 * y + 1] = r.y;
        }
        if (!cap && a.tab) {
          const float4* t = reinterpret_cast<const float4*>(a.tab + (int64_t)j * half + c0);
#pragma unroll
          for (int y = 0; y < 4; ++y) {
            const float4 cs = t[y];
            const float a0 = k0[2 * y], a1 = k0[2 * y + 1], r0 = k1[2 * y], r1 = k1[2 * y + 1];
            k0[2 * y] = a0 * cs.x - r0 * cs.y;
            k1[2 * y] = r0 * cs.x + a0 * cs.y;
            k0[2 * y + 1] = a1 * cs.z - r1 * cs.w;
            k1[2 * y + 1] = r1 * cs.z + a1 * cs.w;
          }
        }
#pragma unroll
        for (int y = 0; y < 8; y += 2) {
          fma2(A0, A1, qv[c0 + y], qv[c0 + y + 1], k0[y], k0[y + 1], A0, A1);
          fma2(A0, A1, qv[half + c0 + y], qv[half + c0 + y + 1], k1[y], k1[y + 1], A0, A1);
        }
      }
      acc = A0 + A1;
    }
    acc += __shfl_xor_sync(0xffffffffu, acc, 1);
    acc += __shfl_xor_sync(0xffffffffu, acc, 2);
    if (e < m && quarter == 0) se[slot][e] = make_float2(acc, __int_as_float(j));
  }
  __syncwarp();
  // rank by counting: entry e precedes entry f when z_e > z_f, or equal with j_e < j_f
  float zk = -CUDART_INF_F;
  for (int e = gl; e < m; e += G) {
    const float2 me = se[slot][e];
    const int mj = __float_as_int(me.y);
    int rank = 0;
    for (int f = 0; f < m; ++f) {
      const float2 o = se[slot][f];
      const int oj = __float_as_int(o.y);
      rank += (o.x > me.x || (o.x == me.x && oj < mj)) ? 1 : 0;
    }
    if (rank < k && live) {
      a.idx[row * k + rank] = mj;
      a.z[row * k + rank] = me.x;
    }
    if (rank == k - 1) zk = me.x;
  }
  if (live)
    for (int r = m + gl; r < k; r += G) {  // fewer than k entries: pad
      a.idx[row * k + r] = -1;
      a.z[row * k + r] = -CUDART_INF_F;
    }
#pragma unroll
  for (int o = G / 2; o > 0; o >>= 1) zk = fmaxf(zk, __shfl_xor_sync(0xffffffffu, zk, o));
  const bool certified = cnt <= kCandCap && (tau == -CUDART_INF_F || zk > tau + eps);
  if (live && !certified && gl == 0) {
    const int pos = atomicAdd(a.status + 2, 1);
    a.fallback_rows[pos] = (int32_t)row;
  }
}

// ---------------------------------------------------------------------------
// pass 3: exact fp32 scan of all candidates of a row (block per row)
// ---------------------------------------------------------------------------
constexpr int kExactThreads = 512;
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
    if constexpr (std::is_same<Tin, __nv_bfloat16>::value) {
      // two keys per thread in flight, 16-byte loads
      for (int j = a.n_start + threadIdx.x; j < jend; j += 2 * blockDim.x) {
        const int j2 = j + blockDim.x;
        const bool ok1 = !(flags && flags[j]);
        const bool ok2 = j2 < jend && !(flags && flags[j2]);
        const bool cap1 = a.L > 0 && (i - j) > a.L, cap2 = a.L > 0 && (i - j2) > a.L;
        float z1 = -CUDART_INF_F, z2 = -CUDART_INF_F;
        if (ok1) z1 = exact_logit_bf16<32 * PP>(kb + (int64_t)j * a.k_st, s_q[cap1 ? 1 : 0], cap1, a.tab, j);
        if (ok2) z2 = exact_logit_bf16<32 * PP>(kb + (int64_t)j2 * a.k_st, s_q[cap2 ? 1 : 0], cap2, a.tab, j2);
        if (ok1 && (z1 > vals[kMaxK - 1] || (z1 == vals[kMaxK - 1] && j < idxs[kMaxK - 1])))
          list_insert<kMaxK>(z1, j, vals, idxs);
        if (ok2 && (z2 > vals[kMaxK - 1] || (z2 == vals[kMaxK - 1] && j2 < idxs[kMaxK - 1])))
          list_insert<kMaxK>(z2, j2, vals, idxs);
      }
    } else {
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
    }
    // k rounds of block-wide argmax over (z desc, j asc)
    block_topk_rounds<kMaxK>(a.topk, vals, idxs, red_z, red_j, [&](int r, float wz, int wj) {
      a.idx[row * a.topk + r] = wj;
      a.z[row * a.topk + r] = (wj >= 0) ? wz : -CUDART_INF_F;
    });
  }
}

template <int D, bool kDual>
cudaError_t launch_score(const TopkArgs& a, const TopkMaps& m, cudaStream_t st) {
  const size_t tile = (size_t)D * kTile * 2;
  // Q tiles, K ring, scan scratch, barriers; at least 116 KB: one CTA per SM, so the
  // 512-column TMEM allocation never waits
  const size_t bytes =
      std::max<size_t>(116 * 1024, 1024 + tile * (2 + kStagesK) + 512 * kScratchStride * 4 + 256 * 4 + 256);
  cudaError_t e =
      cudaFuncSetAttribute(topk_score_kernel<D, kDual>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e != cudaSuccess) return e;
  const int nQB = kDual ? a.nQT : (a.nQT + 1) / 2;
  topk_score_kernel<D, kDual>
      <<<(unsigned)(a.B * a.Hq * nQB), kThreads, bytes, st>>>(m.qsel, m.ksel, m.qsel2, m.ksel2, a, nQB);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_topk_score(const TopkArgs& a, const TopkMaps& m, cudaStream_t st) {
  if ((int64_t)a.B * a.Hq * a.T == 0) return cudaSuccess;
  const bool dual = a.L > 0 && a.window < a.L;
  if (a.d == 128) return dual ? launch_score<128, true>(a, m, st) : launch_score<128, false>(a, m, st);
  if (a.d == 64) return dual ? launch_score<64, true>(a, m, st) : launch_score<64, false>(a, m, st);
  return cudaErrorInvalidValue;
}

cudaError_t launch_topk_rerank(const TopkArgs& a, cudaStream_t st) {
  const int64_t rows = (int64_t)a.B * a.Hq * a.T;
  if (rows == 0) return cudaSuccess;
  const unsigned blocks = (unsigned)((rows + kRerankRows - 1) / kRerankRows);
  const bool dual = a.L > 0 && a.window < a.L;
  if (a.d == 128) {
    if (dual) topk_rerank_kernel<128, true><<<blocks, kRerankWarps * 32, 0, st>>>(a);
    else topk_rerank_kernel<128, false><<<blocks, kRerankWarps * 32, 0, st>>>(a);
  } else if (a.d == 64) {
    if (dual) topk_rerank_kernel<64, true><<<blocks, kRerankWarps * 32, 0, st>>>(a);
    else topk_rerank_kernel<64, false><<<blocks, kRerankWarps * 32, 0, st>>>(a);
  } else {
    return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
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
