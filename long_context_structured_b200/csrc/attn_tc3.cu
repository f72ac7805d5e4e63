// attn_tc3.cu -- K5, one 128-row query tile per CTA with the score tile
// triple-buffered in tensor memory: the prefill attention kernel for capped
// separator tiles and for segment lengths that are not a multiple of 256.
//
// Mathematics (same as attn_tc2.cu): the kept keys of a query row are the
// band keys (the recent window of LM-Infinite's Lambda-shaped mask, section
// 方法; the starting span is handled as fp32 side keys, so the band here is
// i - w_eff <= j <= i, or the segment's band in segmented execution) plus
// gathered keys (SepLLM's separators, section 五.2; or the retrieved prefix of
// segmented execution, section 整体框架), plus fp32 side keys (sinks, top-k
// middle keys) merged in the epilogue.  Softmax is the online
// (running-reference) form; P is bf16, accumulation fp32.
//
// Schedule (one CTA, 384 threads):
//   warps 0-7  softmax + epilogue.  Query row 32(w%4) + 16(w/4) + (lane%16)
//              is shared by lanes l and l^16 of warp w, each owning half of
//              the row's 128 key columns (TMEM 16x32bx2 accesses), so row
//              reductions are one shuffle and two softmax warps share each
//              SM sub-partition (one warp alone cannot keep the exponential
//              unit busy);
//   warp 8     TMA producer: Q (and Qc, the capped-query tile, for capped
//              separator tiles), then the K ring;
//   warp 9     MMA issuer (whole warp in lockstep, an elected lane issues)
//              and TMEM owner;
//   warp 10    TMA producer: the V ring.
// TMEM: S buffers at columns 0, 128, 256 | O at 384.  Key tile j's score
// S(j) goes to buffer j % 3, and the issuer runs two tiles ahead:
//     S(0), S(1), S(2), PV(0), S(3), PV(1), S(4), ...
// so the softmax finds S(j+1) ready when it finishes P(j) and never waits
// for its own PV.  P(j) (bf16) is written over the first 64 columns of its S
// buffer and read from there by PV(j).  Ordering facts used: one thread's
// MMAs execute in issue order, so S(j+3) cannot overwrite P(j) before PV(j)
// read it; a commit arrives only after every earlier MMA of the issuing
// thread completed.
//
// Softmax without a per-tile row maximum: a tile's P is taken against the
// row's running reference m (log2 units), which only the row's first
// non-empty tile sets from its maximum.  bf16 P and fp32 sums keep their
// relative precision at any magnitude, so the result is the same softmax as
// long as nothing overflows; a row whose tile sum exceeds 2^kSumAccept
// (including +inf) redoes the tile against its true maximum, and a row whose
// accepted sum exceeds 2^kSumRebase moves m up by a power of two before its
// next tile (an exact rescale of O and l).  Both rescale O, which needs the
// previous PV to be complete: those rare paths wait for it.
#include <cuda.h>
#include <cuda_bf16.h>
#include <math_constants.h>

#include "attn_common.cuh"
#include "kernels.cuh"
#include "sm100.cuh"

namespace sattn {

namespace {

using attn::exp2_neg_int;
using attn::kSumAccept;
using attn::kSumRebase;
using attn::make_plan;
using attn::Plan;

constexpr int kThreads = 384;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemO = 384;  // O columns (S buffers at 0, 128, 256)

// P = 2^(s*sl2 + neg_m) for this thread's half row (64 keys), packed to
// bf16 and stored to TMEM: the pair owning the row writes P columns 0-31
// (keys 0-63) and 32-63 (keys 64-127) over its S buffer.  Returns the fp32
// sum of the half row's P.  Masked entries hold -inf and give exactly 0.
__device__ __forceinline__ float emit_p(const float (&sv)[64], float sl2, float neg_m, uint32_t taddr) {
  float ps[8];
#pragma unroll
  for (int y = 0; y < 8; ++y) ps[y] = 0.f;
  uint32_t pk[32];
#pragma unroll
  for (int c = 0; c < 64; c += 2) {
    float a0, a1;
    fma2(a0, a1, sv[c], sv[c + 1], sl2, sl2, neg_m, neg_m);
    const float p0 = ex2_approx(a0);
    const float p1 = ex2_approx(a1);
    add2(ps[(c >> 1) & 3], ps[4 + ((c >> 1) & 3)], p0, p1);
    pk[c >> 1] = pack_bf16x2(p0, p1);
  }
  tc::st16x2<32>(taddr, pk);
  return ((ps[0] + ps[1]) + (ps[2] + ps[3])) + ((ps[4] + ps[5]) + (ps[6] + ps[7]));
}

// maximum over the whole row: this half's 64 entries (8 independent 2-input
// chains), then the partner lane's half
__device__ __forceinline__ float row_max(const float (&sv)[64]) {
  float pm[8];
#pragma unroll
  for (int y = 0; y < 8; ++y) pm[y] = sv[y];
#pragma unroll
  for (int c = 8; c < 64; ++c) pm[c & 7] = fmaxf(pm[c & 7], sv[c]);
#pragma unroll
  for (int w = 4; w > 0; w >>= 1)
#pragma unroll
    for (int y = 0; y < w; ++y) pm[y] = fmaxf(pm[y], pm[y + w]);
  return fmaxf(pm[0], __shfl_xor_sync(0xffffffffu, pm[0], 16));
}

// this half row of O *= f (warp-collective: every lane takes part, f = 1
// leaves a row as is); the half row is D/2 columns from taddr (+ D/2 for
// lanes 16-31)
template <int D>
__device__ __forceinline__ void scale_o(uint32_t taddr, float f) {
#pragma unroll 1
  for (int c = 0; c < D / 2; c += 32) {
    float ov[32];
    tc::ld16x2<D / 2>(taddr + c, ov);
    tc_wait_ld();
#pragma unroll
    for (int y = 0; y < 32; ++y) ov[y] *= f;
    tc::st16x2<D / 2>(taddr + c, reinterpret_cast<const uint32_t*>(ov));
  }
}

template <int D, bool Q2>
struct Cfg {
  static constexpr uint32_t kTileBytes = D * kTile * 2;
  static constexpr int kKS = 3;           // K stages
  static constexpr int kVS = Q2 ? 2 : 3;  // V stages (the capped-query tile takes one stage's room)
  static constexpr int kQTiles = Q2 ? 2 : 1;
  static constexpr size_t kSmem = 1024 + (size_t)kTileBytes * (kQTiles + kKS + kVS) + 256;
};

template <int D, bool Q2, bool kAlibi>
__global__ void __launch_bounds__(kThreads, 1)
    attn_tc3_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmQ2,
                    const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                    const __grid_constant__ CUtensorMap tmKg, const __grid_constant__ CUtensorMap tmVg,
                    const AttnArgs a) {
  using C = Cfg<D, Q2>;
  constexpr uint32_t kTileBytes = C::kTileBytes;
  constexpr int kKS = C::kKS, kVS = C::kVS;
  constexpr int kChunks = D / 64;
  constexpr uint32_t kChunkBytes = kTile * 128;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = base;                            // Q | Qc (Q2 only)
  uint8_t* sK = base + C::kQTiles * kTileBytes;  // kKS stages
  uint8_t* sV = sK + kKS * kTileBytes;           // kVS stages
  uint64_t* bars = reinterpret_cast<uint64_t*>(sV + kVS * kTileBytes);
  uint64_t* q_full = bars;
  uint64_t* k_full = bars + 1;
  uint64_t* k_empty = k_full + kKS;
  uint64_t* v_full = k_empty + kKS;
  uint64_t* v_empty = v_full + kVS;
  uint64_t* s_full = v_empty + kVS;  // [3] one per S buffer
  uint64_t* p_full = s_full + 3;     // [3]
  uint64_t* o_done = p_full + 3;     // [2] PV(j) completes a phase of o_done[j & 1]
  uint64_t* o_final = o_done + 2;    // the last PV
  uint64_t* drain = o_final + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  int* abort_i = reinterpret_cast<int*>(tmem_slot + 1);
  int* early = abort_i + 1;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x % a.nQT;         // query tile of the Q / O tensors
  const int tg = t + a.q_pos0 / kTile;      // its position / kTile
  const int bh = blockIdx.x / a.nQT;
  const int h = bh % a.Hq;
  const int b = bh / a.Hq;
  const int g = h / (a.Hq / a.Hkv);
  const Plan pl = make_plan(a, b, h, tg);
  const int n = pl.n_gather + pl.n_band;  // key tiles of this query tile
  const int g_plane = attn::prefix_plane(a, h, g, tg);

  if (threadIdx.x == 0) {
    *early = status_failed(a.status) ? 1 : 0;
    *abort_i = 0;
    mbar_init(q_full, 1);
    for (int s = 0; s < kKS; ++s) {
      mbar_init(k_full + s, 1);
      mbar_init(k_empty + s, 1);
    }
    for (int s = 0; s < kVS; ++s) {
      mbar_init(v_full + s, 1);
      mbar_init(v_empty + s, 1);
    }
    for (int x = 0; x < 3; ++x) {
      mbar_init(s_full + x, 1);
      mbar_init(p_full + x, 256);
    }
    mbar_init(o_done + 0, 1);
    mbar_init(o_done + 1, 1);
    mbar_init(o_final, 1);
    mbar_init(drain, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (*early) return;
  if (warp == 9) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  volatile int* abort_flag = abort_i;

  if (warp == 8 || warp == 10) {
    // ===================== TMA producers: warp 8 Q and K, warp 10 V =====================
    const bool kstream = (warp == 8);
    if (lane == 0 && n > 0) {
      if (kstream) {
        const int i0 = t * kTile;
        const bool want_q2 = Q2 && pl.n_gather > 0;
        mbar_expect_tx(q_full, (want_q2 ? 2 : 1) * kTileBytes);
        for (int c = 0; c < kChunks; ++c) tma_load_4d(sQ + c * kChunkBytes, &tmQ, q_full, c * 64, i0, h, b);
        if (want_q2)
          for (int c = 0; c < kChunks; ++c)
            tma_load_4d(sQ + kTileBytes + c * kChunkBytes, &tmQ2, q_full, c * 64, i0, h, b);
      }
      const int NS = kstream ? kKS : kVS;
      uint8_t* ring = kstream ? sK : sV;
      uint64_t* full = kstream ? k_full : v_full;
      uint64_t* empty = kstream ? k_empty : v_empty;
      int issued = 0;
      bool ok = true;
      for (int j = 0; j < n && ok; ++j) {
        const bool gat = j < pl.n_gather;
        const int row = gat ? j * kTile : (pl.u_lo + j - pl.n_gather) * kTile;
        const int c2 = gat ? g_plane : g;
        const CUtensorMap* mp = kstream ? (gat ? &tmKg : &tmK) : (gat ? &tmVg : &tmV);
        const int st = j % NS;
        if (j >= NS) ok = mbar_wait(empty + st, ((j / NS) - 1) & 1, abort_flag, a.status, kstream ? 31 : 32);
        if (!ok) break;
        mbar_expect_tx(full + st, kTileBytes);
        for (int c = 0; c < kChunks; ++c)
          tma_load_4d(ring + st * kTileBytes + c * kChunkBytes, mp, full + st, c * 64, row, c2, b);
        ++issued;
      }
      if (!ok) {
        // let the loads in flight land before the CTA's shared memory goes away
        if (kstream) tc::wait_raw(q_full, 0);
        for (int j = max(0, issued - NS); j < issued; ++j) tc::wait_raw(full + j % NS, (j / NS) & 1);
      }
    }
  } else if (warp == 9) {
    // ===================== MMA issuer =====================
    // S(0), S(1), S(2), PV(0), S(3), PV(1), ...: S(j) is issued as soon as K(j)
    // is in and PV(j-3) (the last reader of its buffer) has been issued.
    if (n > 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, 128, false);
      constexpr uint32_t idesc_o = idesc_bf16_f32(128, D, true);
      // descriptors of stage / tile bases; the start-address field is addr >> 4
      // in the low 14 bits, so adding (offset >> 4) moves a descriptor within
      // shared memory (below 256 KB, the field cannot carry out)
      const uint64_t dq = smem_desc_sw128(smem_u32(sQ), 16, 1024);
      const uint64_t dk = smem_desc_sw128(smem_u32(sK), 16, 1024);
      const uint64_t dv = smem_desc_sw128(smem_u32(sV), kChunkBytes, 1024);
      auto wait_all = [&](uint64_t* bar, uint32_t parity, int site) -> bool {
        const bool r = mbar_wait(bar, parity, abort_flag, a.status, site);
        return __all_sync(0xffffffffu, r);
      };
      bool ok = wait_all(q_full, 0, 33);
      for (int j = 0; j <= n + 1 && ok; ++j) {
        if (j < n) {
          const int ks = j % kKS;
          ok = wait_all(k_full + ks, (j / kKS) & 1, 40);
          if (!ok) break;
          tc_fence_after();
          const uint64_t ba = dq + (uint64_t)(((Q2 && j < pl.n_gather) ? kTileBytes : 0u) >> 4);
          const uint64_t bk = dk + (uint64_t)((ks * kTileBytes) >> 4);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint64_t off = (uint64_t)(((kk >> 2) * kChunkBytes + (kk & 3) * 32) >> 4);
            tc::mma_ss(tmem + (j % 3) * 128, ba + off, bk + off, idesc_s, kk > 0 ? 1u : 0u);
          }
          tc::commit(s_full + (j % 3));
          tc::commit(k_empty + ks);
        }
        if (j >= 2) {
          const int jj = j - 2;
          const int vs = jj % kVS;
          ok = wait_all(p_full + (jj % 3), (jj / 3) & 1, 34);
          if (ok) ok = wait_all(v_full + vs, (jj / kVS) & 1, 36);
          if (!ok) break;
          tc_fence_after();
          const uint64_t bv = dv + (uint64_t)((vs * kTileBytes) >> 4);
#pragma unroll
          for (int kk = 0; kk < kTile / 16; ++kk)
            tc::mma_ts(tmem + kTmemO, tmem + (jj % 3) * 128 + kk * 8, bv + (uint64_t)((kk * 16 * 128) >> 4),
                         idesc_o, (jj > 0 || kk > 0) ? 1u : 0u);
          tc::commit(o_done + (jj & 1));
          tc::commit(v_empty + vs);
          if (jj == n - 1) tc::commit(o_final);
        }
      }
      tc::commit(drain);
      tc::wait_raw(drain, 0);
    }
    __syncwarp();
  } else if (warp < 8) {
    // ===================== softmax + epilogue (warps 0-7) =====================
    const int rr = 32 * (warp & 3) + 16 * (warp >> 2) + (lane & 15);  // row of the query tile
    const int hc = lane >> 4;                                           // which half of the row's columns
    const int i0 = tg * kTile;
    const int i = i0 + rr;
    const uint32_t lane_off = (uint32_t)(32 * (warp & 3) + 16 * (warp >> 2)) << 16;
    const uint32_t tO = tmem + kTmemO + lane_off;
    const float sl2 = a.scale_log2;
    float m_used = -CUDART_INF_F;  // running reference (log2 units) P is taken against
    float l_sum = 0.f;             // the row's sum (both lanes of the pair hold it)
    int rebase = 0;                // pending: m_used += rebase, O and l_sum *= 2^-rebase
    bool ok = true;
    // O is complete up to PV(j-1) once that PV's phase of o_done[(j-1) & 1]
    // passed.  At key tile j PV(j-3) has finished (it was issued before S(j))
    // and PV(j+1) cannot start (it needs P(j+1)), so that barrier is at most
    // one phase short of the wanted one and a parity wait is exact.
    auto o_stable = [&](int j) {
      if (j >= 1) ok = ok && mbar_wait(o_done + ((j - 1) & 1), ((j - 1) >> 1) & 1, abort_flag, a.status, 45);
    };
    for (int j = 0; j < n; ++j) {
      const int buf = j % 3;
      const uint32_t tS = tmem + buf * 128 + lane_off;
      ok = ok && mbar_wait(s_full + buf, (j / 3) & 1, abort_flag, a.status, 41);
      tc_fence_after();
      // kept columns [c_lo, c_hi] of the row's 128 (band or gathered tile)
      int c_lo = 0, c_hi = kTile - 1;
      if (j < pl.n_gather) {
        const int r0 = j * kTile;
        if (r0 + kTile > pl.g_full) {
          int lim = min(kTile, pl.g_count - r0);
          if (a.gather_mode == 1) {
            // gathered separators kept by row i: pos < i - window (window = L
            // when the band keeps the nearer ones); a prefix count
            const int thr = i - a.window;
            const int cnt = thr > 0 ? sep_before(a.sep_words, a.T, b, thr) : 0;
            lim = max(0, min(lim, cnt - r0));
          }
          c_hi = lim - 1;
        }
      }
      uint64_t xm = 0;  // separators kept beyond the window (this lane's 64 columns)
      if (j >= pl.n_gather) {
        const int j0 = (pl.u_lo + j - pl.n_gather) * kTile;
        const int lo_fix = max(pl.band_lo, a.ns_band);
        const bool full = (j0 + kTile - 1 <= i0) && (j0 >= max(lo_fix, i0 + kTile - 1 - a.w_eff)) &&
                          (i0 + kTile <= a.T);
        if (!full) {
          c_lo = max(lo_fix, i - a.w_eff) - j0;
          c_hi = i - j0;
        }
        if (a.w_sepband > a.w_eff)  // window below the cap: uncapped separators i - L <= j < i - w
          xm = sep_bits64(a.sep_words, a.T, b, j0 + 64 * hc, max(lo_fix, i - a.w_sepband), i - a.w_eff - 1);
      }
      // this lane's columns are 64*hc + [0, 64)
      c_lo -= 64 * hc;
      c_hi -= 64 * hc;
      const bool partial = (c_lo > 0 || c_hi < 63);
      float sv[64];
      tc::ld16x2<64>(tS, sv);
      tc::ld16x2<64>(tS + 32, sv + 32);
      tc_wait_ld();
      if (partial) {
#pragma unroll
        for (int c = 0; c < 64; ++c)
          if ((c < c_lo || c > c_hi) && !((xm >> c) & 1ull)) sv[c] = -CUDART_INF_F;  // exp2(-inf) = 0 below
      }
      if constexpr (kAlibi) {
        // ALiBi bias in units of q.k: band keys -m (i - j) (inside the window,
        // below the cap); gathered separators lie beyond w = L: -m L
        const float sq = alibi_slope_qk(h, a.Hq, a.d);
        if (j < pl.n_gather) {
          const float cb = sq * (float)a.alibi_cap;
#pragma unroll
          for (int c = 0; c < 64; ++c) sv[c] -= cb;
        } else {
          const float base = -sq * (float)(i - (pl.u_lo + j - pl.n_gather) * kTile - 64 * hc);
#pragma unroll
          for (int c = 0; c < 64; ++c) sv[c] += fmaf((float)c, sq, base);
        }
      }
      if (__any_sync(0xffffffffu, rebase != 0)) {
        o_stable(j);
        scale_o<D>(tO, exp2_neg_int(rebase));
        if (rebase != 0) {
          m_used += (float)rebase;
          l_sum *= exp2_neg_int(rebase);
          rebase = 0;
        }
      }
      // a row whose every P so far was 0 (m_used = -inf) has O = 0 and l = 0:
      // it takes its reference from this tile's maximum with nothing to rescale
      if (__any_sync(0xffffffffu, m_used == -CUDART_INF_F)) {
        const float mx = row_max(sv);
        if (m_used == -CUDART_INF_F) m_used = mx * sl2;  // stays -inf if all masked
      }
      // with a zero offset each exp2(-inf) of an all-masked row is exactly 0
      float l_half = emit_p(sv, sl2, (m_used == -CUDART_INF_F) ? 0.f : -m_used, tS);
      float l_tile = l_half + __shfl_xor_sync(0xffffffffu, l_half, 16);
      const bool over = !(l_tile <= kSumAccept);
      if (__any_sync(0xffffffffu, over)) {
        // some row outgrew its reference: move it to the tile's true maximum
        tc_wait_st();
        o_stable(j);
        const float mx = row_max(sv);
        float alpha = 1.f;
        if (over) {
          const float m_new = fmaxf(m_used, mx * sl2);
          alpha = ex2_approx(m_used - m_new);
          l_sum *= alpha;
          m_used = m_new;
        }
        scale_o<D>(tO, alpha);
        l_half = emit_p(sv, sl2, (m_used == -CUDART_INF_F) ? 0.f : -m_used, tS);
        l_tile = l_half + __shfl_xor_sync(0xffffffffu, l_half, 16);
      }
      l_sum += l_tile;
      if (l_tile > kSumRebase) rebase = ((__float_as_int(l_tile) >> 23) & 0xff) - 126;  // 2^rebase > l_tile
      tc_wait_st();
      tc_fence_before();
      if (ok) mbar_arrive(p_full + buf);
    }

    // ---- epilogue: this lane writes O columns hc*D/2 + [0, D/2) of its row ----
    if (n > 0) {
      ok = ok && mbar_wait(o_final, 0, abort_flag, a.status, 43);
      tc_fence_after();
    }
    float o_rebase = 1.f;
    if (rebase != 0) {
      m_used += (float)rebase;
      l_sum *= exp2_neg_int(rebase);
      o_rebase = exp2_neg_int(rebase);
    }
    const bool row_ok = (i < a.T);
    const int ir = row_ok ? i : a.T - 1;
    const int il = ir - a.q_pos0;  // row of the O / LSE tensors
    const size_t row_id = ((size_t)b * a.Hq + h) * attn::q_rows(a) + il;
    const int n_sink = min(a.n_sink, ir + 1);
    const float* sz = a.sink_z ? a.sink_z + row_id * a.n_sink : nullptr;
    const int32_t* tki = a.tk_idx ? a.tk_idx + row_id * a.topk : nullptr;
    const float* tkz = a.tk_z ? a.tk_z + row_id * a.topk : nullptr;
    // top-k keys are middle keys beyond the cap: ALiBi gives them -m L (sink
    // logits carry their bias from the prep pass)
    const float tkb = kAlibi ? alibi_slope_qk(h, a.Hq, a.d) * (float)a.alibi_cap : 0.f;
    float m_fin = m_used;
    for (int jj = 0; jj < n_sink; ++jj) m_fin = fmaxf(m_fin, sz[jj] * sl2);
    for (int y = 0; y < a.topk; ++y)
      if (tki[y] >= 0 && tki[y] < a.T) m_fin = fmaxf(m_fin, (tkz[y] - tkb) * sl2);
    const float alpha = (m_used == -CUDART_INF_F) ? 0.f : ex2_approx(m_used - m_fin);
    float l_fin = l_sum * alpha;
    for (int jj = 0; jj < n_sink; ++jj) l_fin += ex2_approx(sz[jj] * sl2 - m_fin);
    for (int y = 0; y < a.topk; ++y)
      if (tki[y] >= 0 && tki[y] < a.T) l_fin += ex2_approx((tkz[y] - tkb) * sl2 - m_fin);
    const float inv_l = (l_fin > 0.f) ? 1.f / l_fin : 0.f;
    const int col0 = hc * (D / 2);
    const __nv_bfloat16* vbase = a.V + (size_t)b * a.v_sb + (size_t)g * a.v_sh + col0;
    __nv_bfloat16* orow = a.O + (size_t)b * a.o_sb + (size_t)h * a.o_sh + (size_t)il * a.o_st + col0;
#pragma unroll 1
    for (int c = 0; c < D / 2; c += 32) {
      float ov[32];
      if (n > 0) {
        tc::ld16x2<D / 2>(tO + c, ov);
        tc_wait_ld();
#pragma unroll
        for (int y = 0; y < 32; ++y) ov[y] *= alpha * o_rebase;
      } else {
#pragma unroll
        for (int y = 0; y < 32; ++y) ov[y] = 0.f;
      }
      for (int jj = 0; jj < n_sink; ++jj) {
        const float pkv = ex2_approx(sz[jj] * sl2 - m_fin);
        const __nv_bfloat16* vr = vbase + (size_t)jj * a.v_st + c;
#pragma unroll
        for (int y = 0; y < 32; y += 2) {
          const float2 vv = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(vr + y));
          ov[y] = fmaf(pkv, vv.x, ov[y]);
          ov[y + 1] = fmaf(pkv, vv.y, ov[y + 1]);
        }
      }
      for (int t2 = 0; t2 < a.topk; ++t2) {
        const int jk = tki[t2];
        if (jk < 0 || jk >= a.T) continue;
        const float pkv = ex2_approx((tkz[t2] - tkb) * sl2 - m_fin);
        const __nv_bfloat16* vr = vbase + (size_t)jk * a.v_st + c;
#pragma unroll
        for (int y = 0; y < 32; y += 2) {
          const float2 vv = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(vr + y));
          ov[y] = fmaf(pkv, vv.x, ov[y]);
          ov[y + 1] = fmaf(pkv, vv.y, ov[y + 1]);
        }
      }
      if (row_ok) {
        uint4* dst = reinterpret_cast<uint4*>(orow + c);
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
    if (row_ok && hc == 0)
      a.lse[row_id] = (l_fin > 0.f) ? (m_fin + __log2f(l_fin)) * 0.69314718055994531f : -CUDART_INF_F;
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ALiBi is a template parameter, so the kernels without it carry no code for it
template <int D, bool Q2, bool kAlibi>
cudaError_t launch_d(const AttnArgs& a, const AttnMaps& m, cudaStream_t st) {
  const size_t bytes = Cfg<D, Q2>::kSmem;
  cudaError_t e =
      cudaFuncSetAttribute(attn_tc3_kernel<D, Q2, kAlibi>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e != cudaSuccess) return e;
  const unsigned grid = (unsigned)a.B * a.Hq * a.nQT;
  attn_tc3_kernel<D, Q2, kAlibi><<<grid, kThreads, bytes, st>>>(m.q, m.q2, m.k, m.v, m.kg, m.vg, a);
  return cudaGetLastError();
}

template <int D, bool Q2>
cudaError_t launch_q(const AttnArgs& a, const AttnMaps& m, cudaStream_t st) {
  return a.alibi ? launch_d<D, Q2, true>(a, m, st) : launch_d<D, Q2, false>(a, m, st);
}

}  // namespace

cudaError_t launch_attn_tc3(const AttnArgs& a, const AttnMaps& m, cudaStream_t st) {
  if (a.B * a.Hq * a.nQT == 0) return cudaSuccess;
  if (a.d == 128) return a.q2 ? launch_q<128, true>(a, m, st) : launch_q<128, false>(a, m, st);
  if (a.d == 64) return a.q2 ? launch_q<64, true>(a, m, st) : launch_q<64, false>(a, m, st);
  return cudaErrorInvalidValue;
}

}  // namespace sattn
