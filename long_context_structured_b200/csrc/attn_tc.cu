// attn_tc.cu -- K5: prefill attention over the structured key set on the
// 5th-generation tensor cores (tcgen05, accumulators in tensor memory).
//
// What it computes (per query row i of head h):
//   O_i = sum_{j in A_i} softmax_j(s_ij) v_j,  LSE_i = ln sum_{j in A_i} exp(s_ij),
//   s_ij = z_ij / sqrt(d), with A_i split into disjoint parts:
//     band      keys j in [lo(i), i], lo(i) = max(i - w, n_start) ("LM-Infinite",
//               section 方法: the recent window; sinks are excluded here),
//     gathered  separator keys j < i - w from the compacted separator list
//               ("SepLLM", section 五.2), or the retrieved prefix of a long
//               head in segmented execution ("Training-Inference Consistent
//               Segmented Execution", section 整体框架),
//     side      sink keys j < n_start and top-k keys, whose fp32 logits were
//               computed elsewhere (prep pass / selector); merged in the
//               epilogue.
//
// One CTA = one 128-row query tile of one (batch, head).  Warp roles:
//   warps 0-3  softmax + epilogue; thread r owns row r = TMEM lane r
//   warp 4     TMA producer (one lane): Q once, then K/V tiles into a
//              2-stage ring
//   warp 5     TMEM allocator + MMA issuer (one lane)
// Per key tile: S = Q K^T (tcgen05, fp32 in TMEM, double-buffered), the
// softmax warps read S, apply the per-row column range on partial tiles,
// keep a running max with lazy rescaling (only when the max grows by more
// than 2^8), write P (bf16) into a 128-byte-swizzled smem tile, and the MMA
// warp accumulates O += P V into TMEM.  Every wait is bounded; a timeout is
// written to the workspace status word.
#include <cuda.h>
#include <cuda_bf16.h>
#include <math_constants.h>

#include "kernels.cuh"
#include "sm100.cuh"

namespace sattn {

namespace {

constexpr int kThreads = 192;
constexpr int kNS = 2;                   // K/V pipeline stages
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleThreshold = 8.0f;  // log2 units

enum Site {
  kSiteQ = 1, kSiteKFull, kSiteVFull, kSiteKVEmpty, kSiteSFull, kSiteSFree, kSitePFull, kSiteODone, kSiteDrain
};

struct Smem {
  uint8_t* q;
  uint8_t* q2;
  uint8_t* k[kNS];
  uint8_t* v[kNS];
  uint8_t* p;
  uint64_t* q_full;
  uint64_t* k_full;    // [kNS]
  uint64_t* v_full;    // [kNS]
  uint64_t* kv_empty;  // [kNS]
  uint64_t* s_full;    // [2]
  uint64_t* s_free;    // [2]
  uint64_t* p_full;
  uint64_t* o_done;
  uint64_t* drain;
  uint32_t* tmem_slot;
  int* abort_flag;
  int* early;
};

__device__ __forceinline__ bool mbar_wait_raw(uint64_t* bar, uint32_t parity) {
  uint32_t a = smem_u32(bar);
  uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(a, parity)) {
    if (globaltimer_ns() - t0 > 100000000ull) return false;  // 100 ms drain bound
  }
  return true;
}

struct TilePlan {
  int n_gather;     // gathered tiles (first in the order)
  int g_count;      // valid gathered rows
  int g_full;       // gathered rows valid for every row of the query tile
  int g_plane;      // 3rd tensor-map coordinate of the gathered arrays
  int band_lo;      // fixed lower bound of band keys
  int u_lo;         // first band key tile
  int n_band;
  int total;
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmQ2,
                   const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                   const __grid_constant__ CUtensorMap tmKg, const __grid_constant__ CUtensorMap tmVg,
                   const AttnArgs a) {
  constexpr uint32_t kTileBytes = D * kTile * 2;  // one 128-row bf16 tile of width D
  constexpr int kChunks = D / 64;                 // 64-wide (128-byte) column chunks
  constexpr uint32_t kChunkBytes = kTile * 128;   // 16 KB per chunk
  constexpr uint32_t kPBytes = kTile * kTile * 2;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Smem sm;
  {
    uint8_t* p = base;
    sm.q = p;
    p += kTileBytes;
    sm.q2 = p;
    if (a.q2) p += kTileBytes;
    for (int s = 0; s < kNS; ++s) {
      sm.k[s] = p;
      p += kTileBytes;
    }
    for (int s = 0; s < kNS; ++s) {
      sm.v[s] = p;
      p += kTileBytes;
    }
    sm.p = p;
    p += kPBytes;
    uint64_t* bars = reinterpret_cast<uint64_t*>(p);
    sm.q_full = bars;
    sm.k_full = bars + 1;
    sm.v_full = bars + 1 + kNS;
    sm.kv_empty = bars + 1 + 2 * kNS;
    sm.s_full = bars + 1 + 3 * kNS;
    sm.s_free = bars + 3 + 3 * kNS;
    sm.p_full = bars + 5 + 3 * kNS;
    sm.o_done = bars + 6 + 3 * kNS;
    sm.drain = bars + 7 + 3 * kNS;
    sm.tmem_slot = reinterpret_cast<uint32_t*>(bars + 8 + 3 * kNS);
    sm.abort_flag = reinterpret_cast<int*>(sm.tmem_slot + 1);
    sm.early = sm.abort_flag + 1;
  }

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x % a.nQT;
  const int bh = blockIdx.x / a.nQT;
  const int h = bh % a.Hq;
  const int b = bh / a.Hq;
  const int g = h / (a.Hq / a.Hkv);
  const int i0 = t * kTile;

  // ---- which key tiles this query tile visits --------------------------
  TilePlan tp;
  tp.g_count = 0;
  tp.g_full = 0;
  tp.g_plane = g;
  tp.band_lo = 0;
  int seg_s = 0;
  if (a.gather_mode == 1) {
    tp.g_full = a.ranges[(b * a.nQT + t) * 2 + 0];
    tp.g_count = a.ranges[(b * a.nQT + t) * 2 + 1];
  } else if (a.gather_mode == 2) {
    seg_s = i0 / a.seg_S;
    const int seg0 = seg_s * a.seg_S;
    const int slot = a.long_slot[h];
    if (slot >= 0) {
      tp.band_lo = seg0;
      if (seg_s > 0) {
        tp.g_count = tp.g_full = a.prefix_cnt[(b * a.n_long + slot) * a.seg_N + seg_s];
        tp.g_plane = slot * a.seg_N + seg_s;
      }
    } else {
      tp.band_lo = seg_s > 0 ? max(0, seg0 - a.seg_M) : 0;
    }
  }
  tp.n_gather = (tp.g_count + kTile - 1) / kTile;
  {
    const int i_last = min(a.T - 1, i0 + kTile - 1);
    int j_lo = max(max(tp.band_lo, 0), max(i0 - a.w_eff, a.ns_band));
    if (j_lo > i_last) {
      tp.u_lo = 0;
      tp.n_band = 0;
    } else {
      tp.u_lo = j_lo / kTile;
      tp.n_band = i_last / kTile - tp.u_lo + 1;
    }
  }
  tp.total = tp.n_gather + tp.n_band;

  if (threadIdx.x == 0) {
    *sm.early = status_failed(a.status) ? 1 : 0;
    *sm.abort_flag = 0;
    mbar_init(sm.q_full, 1);
    for (int s = 0; s < kNS; ++s) {
      mbar_init(sm.k_full + s, 1);
      mbar_init(sm.v_full + s, 1);
      mbar_init(sm.kv_empty + s, 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(sm.s_full + s, 1);
      mbar_init(sm.s_free + s, 128);
    }
    mbar_init(sm.p_full, 128);
    mbar_init(sm.o_done, 1);
    mbar_init(sm.drain, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (*sm.early) return;
  if (warp == 5) {
    tmem_alloc(sm.tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *sm.tmem_slot;
  const uint32_t tO = tmem + 256;
  volatile int* abort_flag = sm.abort_flag;

  if (warp == 4) {
    // ===================== TMA producer =====================
    if (lane == 0 && tp.total > 0) {
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      const uint32_t qbytes = kTileBytes * (a.q2 ? 2u : 1u);
      mbar_expect_tx(sm.q_full, qbytes);
      for (int c = 0; c < kChunks; ++c) tma_load_4d(sm.q + c * kChunkBytes, &tmQ, sm.q_full, c * 64, i0, h, b);
      if (a.q2)
        for (int c = 0; c < kChunks; ++c) tma_load_4d(sm.q2 + c * kChunkBytes, &tmQ2, sm.q_full, c * 64, i0, h, b);
      int issued = 0;
      bool ok = true;
      for (int it = 0; it < tp.total && ok; ++it) {
        const int st = it % kNS;
        if (it >= kNS) ok = mbar_wait(sm.kv_empty + st, ((it / kNS) - 1) & 1, abort_flag, a.status, kSiteKVEmpty);
        if (!ok) break;
        const CUtensorMap* mk;
        const CUtensorMap* mv;
        int row, c2;
        if (it < tp.n_gather) {
          mk = &tmKg;
          mv = &tmVg;
          row = it * kTile;
          c2 = tp.g_plane;
        } else {
          mk = &tmK;
          mv = &tmV;
          row = (tp.u_lo + it - tp.n_gather) * kTile;
          c2 = g;
        }
        mbar_expect_tx(sm.k_full + st, kTileBytes);
        for (int c = 0; c < kChunks; ++c) tma_load_4d((sm.k[0] + st * kTileBytes) + c * kChunkBytes, mk, sm.k_full + st, c * 64, row, c2, b);
        mbar_expect_tx(sm.v_full + st, kTileBytes);
        for (int c = 0; c < kChunks; ++c) tma_load_4d((sm.v[0] + st * kTileBytes) + c * kChunkBytes, mv, sm.v_full + st, c * 64, row, c2, b);
        ++issued;
      }
      if (!ok) {
        // let loads already in flight land before the CTA retires
        mbar_wait_raw(sm.q_full, 0);
        for (int it = max(0, issued - kNS); it < issued; ++it) {
          mbar_wait_raw(sm.k_full + it % kNS, (it / kNS) & 1);
          mbar_wait_raw(sm.v_full + it % kNS, (it / kNS) & 1);
        }
      }
    }
  } else if (warp == 5) {
    // ===================== MMA issuer =====================
    if (lane == 0 && tp.total > 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, 128, false);
      constexpr uint32_t idesc_o = idesc_bf16_f32(128, D, true);
      const uint32_t q_addr = smem_u32(sm.q), q2_addr = smem_u32(sm.q2), p_addr = smem_u32(sm.p);
      bool ok = mbar_wait(sm.q_full, 0, abort_flag, a.status, kSiteQ);
      auto issue_pv = [&](int jt) -> bool {
        const int st = jt % kNS;
        if (!mbar_wait(sm.p_full, jt & 1, abort_flag, a.status, kSitePFull)) return false;
        if (!mbar_wait(sm.v_full + st, (jt / kNS) & 1, abort_flag, a.status, kSiteVFull)) return false;
        tc_fence_after();
        const uint32_t v_addr = smem_u32((sm.v[0] + st * kTileBytes));
#pragma unroll
        for (int kk = 0; kk < kTile / 16; ++kk) {
          const uint64_t ad = smem_desc_sw128(p_addr + (kk >> 2) * kChunkBytes + (kk & 3) * 32, 16, 1024);
          const uint64_t bd = smem_desc_sw128(v_addr + kk * 16 * 128, kChunkBytes, 1024);
          tc_mma_ss(tO, ad, bd, idesc_o, (jt > 0 || kk > 0) ? 1u : 0u);
        }
        tc_commit(sm.kv_empty + st);
        tc_commit(sm.o_done);
        return true;
      };
      for (int it = 0; it < tp.total && ok; ++it) {
        const int st = it % kNS;
        const int sb = it & 1;
        ok = mbar_wait(sm.k_full + st, (it / kNS) & 1, abort_flag, a.status, kSiteKFull);
        if (ok && it >= 2) ok = mbar_wait(sm.s_free + sb, ((it >> 1) - 1) & 1, abort_flag, a.status, kSiteSFree);
        if (!ok) break;
        tc_fence_after();
        const uint32_t a_addr = (it < tp.n_gather && a.q2) ? q2_addr : q_addr;
        const uint32_t k_addr = smem_u32((sm.k[0] + st * kTileBytes));
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * kChunkBytes + (kk & 3) * 32;
          const uint64_t ad = smem_desc_sw128(a_addr + off, 16, 1024);
          const uint64_t bd = smem_desc_sw128(k_addr + off, 16, 1024);
          tc_mma_ss((tmem + sb * 128u), ad, bd, idesc_s, kk > 0 ? 1u : 0u);
        }
        tc_commit(sm.s_full + sb);
        if (it >= 1) ok = issue_pv(it - 1);
      }
      if (ok) issue_pv(tp.total - 1);
      // every MMA issued by this thread has finished before TMEM is released
      tc_commit(sm.drain);
      mbar_wait_raw(sm.drain, 0);
    }
    __syncwarp();
  } else {
    // ===================== softmax + epilogue (warps 0-3) =====================
    const int r = threadIdx.x;  // row within the tile == TMEM lane
    const int i = i0 + r;
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    const float sl2 = a.scale_log2;
    float m_used = -CUDART_INF_F;  // running max in log2 units (lazy)
    float l_sum = 0.f;
    bool ok = true;
    float sv[128];

    for (int it = 0; it < tp.total; ++it) {
      const int sb = it & 1;
      ok = ok && mbar_wait(sm.s_full + sb, (it >> 1) & 1, abort_flag, a.status, kSiteSFull);
      // tcgen05.ld is warp-collective: all lanes take part even after a failure
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32((tmem + sb * 128u) + lane_off + c * 32, sv + c * 32);
      tc_wait_ld();
      tc_fence_before();
      if (ok) mbar_arrive(sm.s_free + sb);

      // ---- per-row column range [c_lo, c_hi] on partial tiles ----
      int c_lo = 0, c_hi = kTile - 1;
      if (it < tp.n_gather) {
        const int r0 = it * kTile;
        if (r0 + kTile > tp.g_full) {
          int lim = min(kTile, tp.g_count - r0);  // rows present
          if (a.gather_mode == 1) {
            // separators kept iff pos < i - w; positions ascend
            const int* pos = a.sep_pos + (size_t)b * a.T + r0;
            const int thr = i - a.window;
            int lo = 0, hi = lim;  // count of pos[x] < thr among the first lim
            while (lo < hi) {
              const int mid = (lo + hi) >> 1;
              if (__ldg(pos + mid) < thr) lo = mid + 1; else hi = mid;
            }
            lim = lo;
          }
          c_hi = lim - 1;
        }
      } else {
        const int j0 = (tp.u_lo + it - tp.n_gather) * kTile;
        const int lo_fix = max(tp.band_lo, a.ns_band);
        const bool full = (j0 + kTile - 1 <= i0) && (j0 >= max(lo_fix, i0 + kTile - 1 - a.w_eff));
        if (!full) {
          c_lo = max(lo_fix, i - a.w_eff) - j0;
          c_hi = i - j0;
        }
      }
      // row max with 8 independent partial maxima (short dependency chains)
      if (c_lo > 0 || c_hi < kTile - 1) {
#pragma unroll
        for (int c = 0; c < kTile; ++c)
          if (c < c_lo || c > c_hi) sv[c] = -CUDART_INF_F;
      }
      float mx;
      {
        float pm[8];
#pragma unroll
        for (int x = 0; x < 8; ++x) pm[x] = sv[x];
#pragma unroll
        for (int c = 8; c < kTile; ++c) pm[c & 7] = fmaxf(pm[c & 7], sv[c]);
        mx = fmaxf(fmaxf(fmaxf(pm[0], pm[1]), fmaxf(pm[2], pm[3])), fmaxf(fmaxf(pm[4], pm[5]), fmaxf(pm[6], pm[7])));
      }
      const float m_tile = mx * sl2;
      const float m_new = fmaxf(m_used, m_tile);
      const bool grow = m_new > m_used + kRescaleThreshold;
      float alpha = 1.f;
      bool rescale_o = false;
      if (grow) {
        alpha = (m_used == -CUDART_INF_F) ? 0.f : ex2_approx(m_used - m_new);
        rescale_o = (it > 0) && (m_used != -CUDART_INF_F);
        l_sum *= alpha;
        m_used = m_new;
      }
      // P = 2^(s*log2e/sqrt(d) - m), packed to bf16 pairs at once; 8 partial sums
      uint32_t pk[kTile / 2];
      {
        float ps[8];
#pragma unroll
        for (int x = 0; x < 8; ++x) ps[x] = 0.f;
        const float neg_m = (m_used == -CUDART_INF_F) ? 0.f : -m_used;
        const bool none = (m_used == -CUDART_INF_F);
#pragma unroll
        for (int c = 0; c < kTile; c += 2) {
          float p0 = ex2_approx(fmaf(sv[c], sl2, neg_m));
          float p1 = ex2_approx(fmaf(sv[c + 1], sl2, neg_m));
          if (none) p0 = p1 = 0.f;
          ps[(c >> 1) & 7] += p0 + p1;
          pk[c >> 1] = pack_bf16x2(p0, p1);
        }
        l_sum += ((ps[0] + ps[1]) + (ps[2] + ps[3])) + ((ps[4] + ps[5]) + (ps[6] + ps[7]));
      }

      // PV of the previous tile must be done: P buffer free and O stable
      if (it > 0) {
        ok = ok && mbar_wait(sm.o_done, (it - 1) & 1, abort_flag, a.status, kSiteODone);
        tc_fence_after();
      }
      if (__any_sync(0xffffffffu, rescale_o)) {
        const float f = rescale_o ? alpha : 1.f;
        float ov[32];
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          tmem_ld32(tO + lane_off + c * 32, ov);
          tc_wait_ld();
#pragma unroll
          for (int x = 0; x < 32; ++x) ov[x] *= f;
          tmem_st32(tO + lane_off + c * 32, ov);
        }
        tc_wait_st();
      }
      // P (bf16) -> swizzled smem, two 64-key chunks
#pragma unroll
      for (int gq = 0; gq < 16; ++gq) {
        const int kc = gq >> 3, gg = gq & 7;
        const uint4 val = make_uint4(pk[gq * 4 + 0], pk[gq * 4 + 1], pk[gq * 4 + 2], pk[gq * 4 + 3]);
        *reinterpret_cast<uint4*>(sm.p + kc * kChunkBytes + sw128_offset(r, gg)) = val;
      }
      fence_proxy_async_smem();
      tc_fence_before();
      if (ok) mbar_arrive(sm.p_full);
    }

    // ---- epilogue: wait for the last PV, merge side keys, normalise ----
    if (tp.total > 0) {
      ok = ok && mbar_wait(sm.o_done, (tp.total - 1) & 1, abort_flag, a.status, kSiteODone);
      tc_fence_after();
    }
    const bool row_ok = i < a.T;
    const int ir = row_ok ? i : a.T - 1;
    const size_t row_id = ((size_t)b * a.Hq + h) * a.T + ir;
    const int n_sink = min(a.n_sink, ir + 1);
    const float* sz = a.sink_z ? a.sink_z + row_id * a.n_sink : nullptr;
    const int32_t* tki = a.tk_idx ? a.tk_idx + row_id * a.topk : nullptr;
    const float* tkz = a.tk_z ? a.tk_z + row_id * a.topk : nullptr;
    float m_fin = m_used;
    for (int j = 0; j < n_sink; ++j) m_fin = fmaxf(m_fin, sz[j] * sl2);
    for (int x = 0; x < a.topk; ++x)
      if (tki[x] >= 0 && tki[x] < a.T) m_fin = fmaxf(m_fin, tkz[x] * sl2);
    const float alpha = (m_used == -CUDART_INF_F) ? 0.f : ex2_approx(m_used - m_fin);
    float l_fin = l_sum * alpha;
    for (int j = 0; j < n_sink; ++j) l_fin += ex2_approx(sz[j] * sl2 - m_fin);
    for (int x = 0; x < a.topk; ++x)
      if (tki[x] >= 0 && tki[x] < a.T) l_fin += ex2_approx(tkz[x] * sl2 - m_fin);
    const float inv_l = (l_fin > 0.f) ? 1.f / l_fin : 0.f;
    const __nv_bfloat16* vbase = a.V + (size_t)b * a.v_sb + (size_t)g * a.v_sh;
    __nv_bfloat16* orow = a.O + (size_t)b * a.o_sb + (size_t)h * a.o_sh + (size_t)ir * a.o_st;
#pragma unroll 1
    for (int c = 0; c < D / 32; ++c) {
      float ov[32];
      if (tp.total > 0) {
        tmem_ld32(tO + lane_off + c * 32, ov);
        tc_wait_ld();
#pragma unroll
        for (int x = 0; x < 32; ++x) ov[x] *= alpha;
      } else {
#pragma unroll
        for (int x = 0; x < 32; ++x) ov[x] = 0.f;
      }
      for (int j = 0; j < n_sink; ++j) {
        const float pk = ex2_approx(sz[j] * sl2 - m_fin);
        const __nv_bfloat16* vr = vbase + (size_t)j * a.v_st + c * 32;
#pragma unroll
        for (int x = 0; x < 32; x += 2) {
          const float2 vv = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(vr + x));
          ov[x] = fmaf(pk, vv.x, ov[x]);
          ov[x + 1] = fmaf(pk, vv.y, ov[x + 1]);
        }
      }
      for (int y = 0; y < a.topk; ++y) {
        const int j = tki[y];
        if (j < 0 || j >= a.T) continue;
        const float pk = ex2_approx(tkz[y] * sl2 - m_fin);
        const __nv_bfloat16* vr = vbase + (size_t)j * a.v_st + c * 32;
#pragma unroll
        for (int x = 0; x < 32; x += 2) {
          const float2 vv = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(vr + x));
          ov[x] = fmaf(pk, vv.x, ov[x]);
          ov[x + 1] = fmaf(pk, vv.y, ov[x + 1]);
        }
      }
      if (row_ok) {
        uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          uint4 val;
          val.x = pack_bf16x2(ov[q4 * 8 + 0] * inv_l, ov[q4 * 8 + 1] * inv_l);
          val.y = pack_bf16x2(ov[q4 * 8 + 2] * inv_l, ov[q4 * 8 + 3] * inv_l);
          val.z = pack_bf16x2(ov[q4 * 8 + 4] * inv_l, ov[q4 * 8 + 5] * inv_l);
          val.w = pack_bf16x2(ov[q4 * 8 + 6] * inv_l, ov[q4 * 8 + 7] * inv_l);
          dst[q4] = val;
        }
      }
    }
    if (row_ok) {
      a.lse[row_id] = (l_fin > 0.f) ? (m_fin + __log2f(l_fin)) * 0.69314718055994531f : -CUDART_INF_F;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <int D>
cudaError_t launch_d(const AttnArgs& a, const AttnMaps& m, cudaStream_t st) {
  const size_t tile = (size_t)D * kTile * 2;
  // at least 116 KB: one CTA per SM, so the 512-column TMEM allocation never waits
  const size_t bytes = std::max<size_t>(116 * 1024, 1024 + tile * (1 + (a.q2 ? 1 : 0) + 2 * kNS) + (size_t)kTile * kTile * 2 + 256);
  cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e != cudaSuccess) return e;
  const unsigned grid = (unsigned)a.B * a.Hq * a.nQT;
  attn_tc_kernel<D><<<grid, kThreads, bytes, st>>>(m.q, m.q2, m.k, m.v, m.kg, m.vg, a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_tc(const AttnArgs& a, const AttnMaps& m, cudaStream_t st) {
  if (a.B * a.Hq * a.nQT == 0) return cudaSuccess;
  if (a.d == 128) return launch_d<128>(a, m, st);
  if (a.d == 64) return launch_d<64>(a, m, st);
  return cudaErrorInvalidValue;
}

}  // namespace sattn
