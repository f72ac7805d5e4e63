// bwd_tc.cu -- the tensor-core parts of the bf16 backward pass ("SepLLM",
// section 6.2: training runs the forward and the backward pass through the
// masked product).  With P = exp(s - LSE) recomputed from the forward's
// LSE, dP = dO V^T, D_i = dO_i . O_i and dS = P (dP - D):
//
//   bwd_dq_kernel   one 128-row query tile per CTA: over its band and
//                   gathered key tiles S = Q K^T and dP = dO V^T go to TMEM,
//                   eight warps turn them into dS (bf16, written back over S),
//                   and dQ += dS K accumulates in TMEM (K read as an MN-major
//                   operand from the same shared-memory tile S used).  The
//                   epilogue rotates the row back (R(i)^T; R(L)^T in the
//                   capped-separator pass, whose keys are raw: "LM-Infinite",
//                   section 方法), scales by 1/sqrt(d) and adds the fp32 side
//                   terms (sinks, capped separators).
//   bwd_dkv_kernel  one 128-key tile per CTA (a band tile over positions or a
//                   tile of compacted separators, "SepLLM" section 五.2): over
//                   the query tiles of every query head of its group that
//                   keep its keys, S^T = K Q^T and dP^T = V dO^T go to TMEM,
//                   the warps write P^T and dS^T back over them, and
//                   dV += P^T dO, dK += dS^T Q accumulate in TMEM.
//
// Both kernels: 384 threads; warps 0-7 compute (a row shared by lanes l and
// l^16, each holding 64 columns), warp 8 TMA producer, warp 9 MMA issuer
// and TMEM owner, warp 10 second producer (dq kernel: the V ring).  Every
// barrier wait is bounded; a timeout sets the status word and the CTA
// drains its copies and products before releasing TMEM.
#include <cuda.h>
#include <cuda_bf16.h>
#include <math_constants.h>

#include "kernels.cuh"
#include "tc_ops.cuh"

namespace sattn {

namespace {

constexpr int kThreads = 384;
constexpr uint32_t kTmemCols = 512;

__device__ __forceinline__ float2 tab_at(const float2* tab, int64_t pos, int half, int c) {
  return tab ? tab[pos * half + c] : make_float2(1.f, 0.f);
}

// Rotate this lane's 32 accumulator columns back (R(pos)^T) with the
// partner lane's: lane hc = 0 holds columns cc + y of the first half (x0 of
// pair cc + y), lane hc = 1 the same pairs' second components (x1).
__device__ __forceinline__ void rotate_back(float (&v)[32], const float2* tab, int64_t pos, int half, int cc,
                                            int hc) {
#pragma unroll
  for (int y = 0; y < 32; ++y) {
    const float other = __shfl_xor_sync(0xffffffffu, v[y], 16);
    const float2 cs = tab_at(tab, pos, half, cc + y);
    v[y] = hc == 0 ? fmaf(v[y], cs.x, other * cs.y) : fmaf(v[y], cs.x, -other * cs.y);
  }
}

__device__ __forceinline__ void pack_store64(uint32_t taddr, const float (&x)[64]) {
  uint32_t pk[32];
#pragma unroll
  for (int c = 0; c < 64; c += 2) pk[c >> 1] = pack_bf16x2(x[c], x[c + 1]);
  tc::st16x2<32>(taddr, pk);
}

// ===========================================================================
// dQ kernel
// ===========================================================================

struct QPlan {
  int g_count, g_full, n_gather, u_lo, n_band;
};

__device__ __forceinline__ QPlan make_qplan(const BwdArgs& a, int b, int t) {
  QPlan p{};
  const int i0 = t * kTile;
  const int rows = min(kTile, a.T - i0);
  if (a.gather && (a.dq_mode == 1 || !a.capped_sep)) {
    p.g_full = a.ranges[(b * a.nQT + t) * 2 + 0];
    p.g_count = a.ranges[(b * a.nQT + t) * 2 + 1];
    p.n_gather = (p.g_count + kTile - 1) / kTile;
  }
  if (a.dq_mode == 0) {
    const int i_last = i0 + rows - 1;
    const int j_lo = max(i0 - max(a.window, a.w_sepband), a.n_start);
    if (j_lo <= i_last) {
      p.u_lo = j_lo / kTile;
      p.n_band = i_last / kTile - p.u_lo + 1;
    }
  }
  return p;
}

constexpr int kFoldStage = 16;  // sink key rows staged at a time in the dq epilogue

template <int D>
struct QCfg {
  static constexpr uint32_t kTileBytes = D * kTile * 2;
  static constexpr int kKS = 3, kVS = 2;
  static constexpr size_t kSmem = 1024 + (size_t)kTileBytes * (2 + kKS + kVS) + 256;
};

template <int D, bool kAlibi>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_dq_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmDO,
                  const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                  const __grid_constant__ CUtensorMap tmKg, const __grid_constant__ CUtensorMap tmVg,
                  const BwdArgs a) {
  using C = QCfg<D>;
  constexpr uint32_t kTileBytes = C::kTileBytes;
  constexpr int kKS = C::kKS, kVS = C::kVS;
  constexpr int kChunks = D / 64;
  constexpr uint32_t kChunkBytes = kTile * 128;
  constexpr uint32_t kTmemDP = 256, kTmemDQ = 384;  // S buffers at 0 and 128

  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = base;
  uint8_t* sDO = sQ + kTileBytes;
  uint8_t* sK = sDO + kTileBytes;
  uint8_t* sV = sK + kKS * kTileBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sV + kVS * kTileBytes);
  uint64_t* q_full = bars;
  uint64_t* k_full = q_full + 1;
  uint64_t* k_empty = k_full + kKS;
  uint64_t* v_full = k_empty + kKS;
  uint64_t* v_empty = v_full + kVS;
  uint64_t* s_full = v_empty + kVS;  // [2]
  uint64_t* dp_full = s_full + 2;
  uint64_t* ds_full = dp_full + 1;   // [2], 256 arrivals
  uint64_t* dq_done = ds_full + 2;
  uint64_t* drain = dq_done + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  int* abort_i = reinterpret_cast<int*>(tmem_slot + 1);
  int* early = abort_i + 1;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x % a.nQT;
  const int bh = blockIdx.x / a.nQT;
  const int h = bh % a.Hq;
  const int b = bh / a.Hq;
  const int g = h / (a.Hq / a.Hkv);
  const QPlan pl = make_qplan(a, b, t);
  const int n = pl.n_gather + pl.n_band;

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
    for (int x = 0; x < 2; ++x) {
      mbar_init(s_full + x, 1);
      mbar_init(ds_full + x, 256);
    }
    mbar_init(dp_full, 1);
    mbar_init(dq_done, 1);
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
    // ===================== producers: warp 8 Q, dO and K; warp 10 V =====================
    const bool kstream = (warp == 8);
    if (lane == 0 && n > 0) {
      if (kstream) {
        const int i0 = t * kTile;
        mbar_expect_tx(q_full, 2 * kTileBytes);
        for (int c = 0; c < kChunks; ++c) {
          tma_load_4d(sQ + c * kChunkBytes, &tmQ, q_full, c * 64, i0, h, b);
          tma_load_4d(sDO + c * kChunkBytes, &tmDO, q_full, c * 64, i0, h, b);
        }
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
        const CUtensorMap* mp = kstream ? (gat ? &tmKg : &tmK) : (gat ? &tmVg : &tmV);
        const int st = j % NS;
        if (j >= NS) ok = mbar_wait(empty + st, ((j / NS) - 1) & 1, abort_flag, a.status, kstream ? 61 : 62);
        if (!ok) break;
        mbar_expect_tx(full + st, kTileBytes);
        for (int c = 0; c < kChunks; ++c)
          tma_load_4d(ring + st * kTileBytes + c * kChunkBytes, mp, full + st, c * 64, row, g, b);
        ++issued;
      }
      if (!ok) {
        if (kstream) tc::wait_raw(q_full, 0);
        for (int j = max(0, issued - NS); j < issued; ++j) tc::wait_raw(full + j % NS, (j / NS) & 1);
      }
    }
  } else if (warp == 9) {
    // ===================== MMA issuer =====================
    // S(0), dP(0), S(1), then per tile j: dQ(j), dP(j+1), S(j+2).
    if (n > 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, 128, false);
      constexpr uint32_t idesc_q = idesc_bf16_f32(128, D, true);
      const uint64_t dq_ = smem_desc_sw128(smem_u32(sQ), 16, 1024);
      const uint64_t ddo = smem_desc_sw128(smem_u32(sDO), 16, 1024);
      const uint64_t dk = smem_desc_sw128(smem_u32(sK), 16, 1024);
      const uint64_t dkm = smem_desc_sw128(smem_u32(sK), kChunkBytes, 1024);  // K as an MN-major operand
      const uint64_t dv = smem_desc_sw128(smem_u32(sV), 16, 1024);
      auto wait_all = [&](uint64_t* bar, uint32_t parity, int site) -> bool {
        const bool r = mbar_wait(bar, parity, abort_flag, a.status, site);
        return __all_sync(0xffffffffu, r);
      };
      auto koff = [&](int kk) -> uint64_t { return (uint64_t)(((kk >> 2) * kChunkBytes + (kk & 3) * 32) >> 4); };
      auto issue_s = [&](int j) -> bool {
        const int ks = j % kKS;
        if (!wait_all(k_full + ks, (j / kKS) & 1, 63)) return false;
        tc_fence_after();
        const uint64_t bk = dk + (uint64_t)((ks * kTileBytes) >> 4);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          tc::mma_ss(tmem + (j & 1) * 128, dq_ + koff(kk), bk + koff(kk), idesc_s, kk > 0 ? 1u : 0u);
        tc::commit(s_full + (j & 1));
        return true;
      };
      auto issue_dp = [&](int j) -> bool {
        const int vs = j % kVS;
        if (!wait_all(v_full + vs, (j / kVS) & 1, 64)) return false;
        tc_fence_after();
        const uint64_t bv = dv + (uint64_t)((vs * kTileBytes) >> 4);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          tc::mma_ss(tmem + kTmemDP, ddo + koff(kk), bv + koff(kk), idesc_s, kk > 0 ? 1u : 0u);
        tc::commit(dp_full);
        tc::commit(v_empty + vs);
        return true;
      };
      auto issue_dq = [&](int j) -> bool {
        if (!wait_all(ds_full + (j & 1), (j >> 1) & 1, 65)) return false;
        tc_fence_after();
        const int ks = j % kKS;
        const uint64_t bk = dkm + (uint64_t)((ks * kTileBytes) >> 4);
#pragma unroll
        for (int kk = 0; kk < kTile / 16; ++kk)
          tc::mma_ts(tmem + kTmemDQ, tmem + (j & 1) * 128 + kk * 8, bk + (uint64_t)((kk * 16 * 128) >> 4), idesc_q,
                     (j > 0 || kk > 0) ? 1u : 0u);
        tc::commit(k_empty + ks);
        return true;
      };
      bool ok = wait_all(q_full, 0, 60);
      ok = ok && issue_s(0) && issue_dp(0);
      if (n > 1) ok = ok && issue_s(1);
      for (int j = 0; j < n && ok; ++j) {
        ok = issue_dq(j);
        if (ok && j + 1 < n) ok = issue_dp(j + 1);
        if (ok && j + 2 < n) ok = issue_s(j + 2);
      }
      if (ok) tc::commit(dq_done);
      tc::commit(drain);
      tc::wait_raw(drain, 0);
    }
    __syncwarp();
  } else if (warp < 8) {
    // ===================== dS + epilogue (warps 0-7) =====================
    const int rr = tc::pair_row(warp, lane);
    const int hc = lane >> 4;
    const int i0 = t * kTile;
    const int i = i0 + rr;
    const uint32_t lane_off = tc::pair_lane_off(warp);
    const float sl2 = a.scale_log2;
    const int64_t prow = (int64_t)bh * a.Tpad + i;
    const float Drow = a.Dsum[prow], nl2 = a.nlse2[prow];
    bool ok = true;
    for (int j = 0; j < n; ++j) {
      const uint32_t tS = tmem + (j & 1) * 128 + lane_off;
      ok = ok && mbar_wait(s_full + (j & 1), (j >> 1) & 1, abort_flag, a.status, 66);
      tc_fence_after();
      int c_lo = 0, c_hi = kTile - 1;
      if (j < pl.n_gather) {
        const int r0 = j * kTile;
        if (r0 + kTile > pl.g_full) {
          int lim = min(kTile, pl.g_count - r0);
          const int thr = i - a.sep_split;  // compacted separators kept by row i: pos < i - split
          const int cnt = thr > 0 ? sep_before(a.sep_words, a.T, b, thr) : 0;
          lim = max(0, min(lim, cnt - r0));
          c_hi = lim - 1;
        }
      }
      uint64_t xm = 0;  // uncapped separators beyond the window (this lane's 64 columns)
      if (j >= pl.n_gather) {
        const int j0 = (pl.u_lo + j - pl.n_gather) * kTile;
        c_lo = max(a.n_start, i - a.window) - j0;
        c_hi = i - j0;
        if (a.w_sepband > a.window)
          xm = sep_bits64(a.sep_words, a.T, b, j0 + 64 * hc, max(a.n_start, i - a.w_sepband), i - a.window - 1);
      }
      c_lo -= 64 * hc;
      c_hi -= 64 * hc;
      float sv[64];
      tc::ld16x2<64>(tS, sv);
      tc::ld16x2<64>(tS + 32, sv + 32);
      tc_wait_ld();
      if constexpr (kAlibi) {
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
#pragma unroll
      for (int c = 0; c < 64; ++c)
        sv[c] = ((c < c_lo || c > c_hi) && !((xm >> c) & 1ull)) ? 0.f : ex2_approx(fmaf(sv[c], sl2, nl2));
      ok = ok && mbar_wait(dp_full, j & 1, abort_flag, a.status, 67);
      tc_fence_after();
      float dp[64];
      tc::ld16x2<64>(tmem + kTmemDP + lane_off, dp);
      tc::ld16x2<64>(tmem + kTmemDP + lane_off + 32, dp + 32);
      tc_wait_ld();
#pragma unroll
      for (int c = 0; c < 64; ++c) sv[c] *= dp[c] - Drow;
      pack_store64(tS, sv);
      tc_wait_st();
      tc_fence_before();
      if (ok) mbar_arrive(ds_full + (j & 1));
    }

    // ---- epilogue: this lane's columns hc * D/2 + [0, D/2) of row i ----
    if (n > 0) {
      ok = ok && mbar_wait(dq_done, 0, abort_flag, a.status, 68);
      tc_fence_after();
    }
    const int half = D / 2;
    const float scale = rsqrtf((float)D);
    const int64_t pos = a.dq_mode == 1 ? a.L : i;
    const bool row_ok = i < a.T;
    const int64_t grow = (int64_t)bh * a.T + (row_ok ? i : a.T - 1);
#pragma unroll 1
    for (int cc = 0; cc < half; cc += 32) {
      float v[32];
      if (n > 0) {
        tc::ld16x2<D / 2>(tmem + kTmemDQ + lane_off + cc, v);
        tc_wait_ld();
      } else {
#pragma unroll
        for (int y = 0; y < 32; ++y) v[y] = 0.f;
      }
      if (a.fold_sinks) {
        // the sink pairs (fp32 side keys; P and dS from the row pass): the
        // uncapped sum of dS R(j) k_j joins v before the rotation back by
        // R(i)^T, the capped sum of dS k_j is rotated back by R(L)^T.  The
        // sink keys (rotated and raw, fp32) are staged in the K ring, free
        // once the last MMA has completed; a lane reads the component (hc)
        // of the pairs it holds.
        float* s_kr = reinterpret_cast<float*>(sK);  // [kFoldStage][D] R(j) k_j
        float* s_kw = s_kr + kFoldStage * D;          // [kFoldStage][D] k_j
        float vc[32];
#pragma unroll
        for (int y = 0; y < 32; ++y) vc[y] = 0.f;
        const int ns = row_ok ? min(a.n_sink, i + 1) : 0;
        const float* dsr = a.sink_ds + grow * a.n_sink;
        const bool restage = a.n_sink > kFoldStage || cc == 0;  // one stage serves both chunks
        for (int js = 0; js < a.n_sink; js += kFoldStage) {
          const int nst = min(kFoldStage, a.n_sink - js);
          if (restage) {
            asm volatile("bar.sync 1, 256;" ::: "memory");  // the epilogue warps: the stage is free
            for (int x = threadIdx.x; x < nst * half; x += 256) {
              const int jj = x / half, p = x - jj * half, j = js + jj;
              const __nv_bfloat16* kp = a.K + (int64_t)b * a.k_sb + (int64_t)g * a.k_sh + (int64_t)j * a.k_st;
              const float k0 = __bfloat162float(kp[p]), k1 = __bfloat162float(kp[p + half]);
              const float2 cs = tab_at(a.tab, j, half, p);
              s_kr[jj * D + p] = k0 * cs.x - k1 * cs.y;
              s_kr[jj * D + p + half] = k1 * cs.x + k0 * cs.y;
              s_kw[jj * D + p] = k0;
              s_kw[jj * D + p + half] = k1;
            }
            asm volatile("bar.sync 1, 256;" ::: "memory");
          }
          for (int jj = 0; jj < nst && js + jj < ns; ++jj) {
            const int j = js + jj;
            const float ds = dsr[j];
            const bool capped = a.L > 0 && i - j > a.L;
            const float* src = (capped ? s_kw : s_kr) + jj * D + hc * half + cc;
#pragma unroll
            for (int y = 0; y < 32; ++y) {
              if (capped) vc[y] = fmaf(ds, src[y], vc[y]);
              else v[y] = fmaf(ds, src[y], v[y]);
            }
          }
        }
        rotate_back(v, a.tab, pos, half, cc, hc);
        if (a.L > 0) {
          rotate_back(vc, a.tab, a.L, half, cc, hc);
#pragma unroll
          for (int y = 0; y < 32; ++y) v[y] += vc[y];
        }
      } else {
        rotate_back(v, a.tab, pos, half, cc, hc);
      }
      const int col = hc * half + cc;
      float* side = a.dq_side + grow * D + col;
      if (a.side_valid && row_ok) {
#pragma unroll
        for (int y = 0; y < 32; y += 4) {
          const float4 s4 = *reinterpret_cast<const float4*>(side + y);
          v[y] = fmaf(v[y], scale, s4.x);
          v[y + 1] = fmaf(v[y + 1], scale, s4.y);
          v[y + 2] = fmaf(v[y + 2], scale, s4.z);
          v[y + 3] = fmaf(v[y + 3], scale, s4.w);
        }
      } else {
#pragma unroll
        for (int y = 0; y < 32; ++y) v[y] *= scale;
      }
      if (!row_ok) continue;
      if (a.dq_mode == 1) {
#pragma unroll
        for (int y = 0; y < 32; y += 4) *reinterpret_cast<float4*>(side + y) = make_float4(v[y], v[y + 1], v[y + 2], v[y + 3]);
      } else {
        __nv_bfloat16* dst = a.dQ + (int64_t)b * a.q_sb + (int64_t)h * a.q_sh + (int64_t)i * a.q_st + col;
#pragma unroll
        for (int y = 0; y < 32; y += 8) {
          uint4 u;
          u.x = pack_bf16x2(v[y], v[y + 1]);
          u.y = pack_bf16x2(v[y + 2], v[y + 3]);
          u.z = pack_bf16x2(v[y + 4], v[y + 5]);
          u.w = pack_bf16x2(v[y + 6], v[y + 7]);
          *reinterpret_cast<uint4*>(dst + y) = u;
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ===========================================================================
// dK / dV kernel
// ===========================================================================

template <int D>
struct KVCfg {
  static constexpr uint32_t kTileBytes = D * kTile * 2;
  static constexpr uint32_t kStatBytes = 2 * kTile * 4;  // -lse2 and D of a query tile
  static constexpr size_t kSmem = 1024 + (size_t)kTileBytes * 6 + 2 * kStatBytes + 256;
};

// The query tiles a key tile's CTA visits, for each query head of its group:
// [t_lo, t_hi].  Band tile u: its keys are kept by rows j <= i <= j + w;
// separator tile r: by rows i > j + w.
struct KVPlan {
  bool sep;          // a tile of compacted separators
  int tile;          // band tile u, or separator tile r
  int t_lo, n_t;     // query tiles per head
  int n;             // steps = heads of the group x n_t
};

__device__ __forceinline__ KVPlan make_kvplan(const BwdArgs& a, int b, int tile_id) {
  KVPlan p{};
  p.sep = tile_id >= a.nQT;
  p.tile = p.sep ? tile_id - a.nQT : tile_id;
  const int rep = a.Hq / a.Hkv;
  if (!p.sep) {
    const int j_lo = max(p.tile * kTile, a.n_start);
    const int j_hi = min(p.tile * kTile + kTile, a.T) - 1;
    if (j_lo > j_hi) return p;
    p.t_lo = j_lo / kTile;
    const int t_hi = min(a.nQT - 1, (j_hi + max(a.window, a.w_sepband)) / kTile);
    p.n_t = t_hi - p.t_lo + 1;
  } else {
    const int cnt = a.sep_count[b];
    if (p.tile * kTile >= cnt) return p;
    const int j_first = a.sep_pos[(size_t)b * a.T + p.tile * kTile];
    const int i_first = j_first + a.sep_split + 1;
    if (i_first >= a.T) return p;
    p.t_lo = i_first / kTile;
    p.n_t = a.nQT - p.t_lo;
  }
  p.n = rep * p.n_t;
  return p;
}

template <int D, bool kAlibi>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_dkv_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmQc,
                   const __grid_constant__ CUtensorMap tmDO,
                   const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                   const __grid_constant__ CUtensorMap tmKg, const __grid_constant__ CUtensorMap tmVg,
                   const BwdArgs a) {
  using C = KVCfg<D>;
  constexpr uint32_t kTileBytes = C::kTileBytes;
  constexpr uint32_t kStatBytes = C::kStatBytes;
  constexpr int kChunks = D / 64;
  constexpr uint32_t kChunkBytes = kTile * 128;
  constexpr uint32_t kTmemDP = 128, kTmemDV = 256, kTmemDK = 384;  // S^T at 0

  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sK = base;
  uint8_t* sV = sK + kTileBytes;
  uint8_t* sQ = sV + kTileBytes;          // 2 stages
  uint8_t* sDO = sQ + 2 * kTileBytes;     // 2 stages
  float* sStat = reinterpret_cast<float*>(sDO + 2 * kTileBytes);  // 2 stages of [-lse2 (128) | D (128)]
  uint64_t* bars = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(sStat) + 2 * kStatBytes);
  uint64_t* kv_full = bars;
  uint64_t* q_full = kv_full + 1;  // [2]
  uint64_t* q_empty = q_full + 2;  // [2]
  uint64_t* s_full = q_empty + 2;
  uint64_t* dp_full = s_full + 1;
  uint64_t* p_full = dp_full + 1;   // 256 arrivals
  uint64_t* ds_full = p_full + 1;   // 256 arrivals
  uint64_t* kv_done = ds_full + 1;
  uint64_t* drain = kv_done + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  int* abort_i = reinterpret_cast<int*>(tmem_slot + 1);
  int* early = abort_i + 1;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int tiles = a.gather ? 2 * a.nQT : a.nQT;
  const int tile_id = blockIdx.x % tiles;
  const int bg = blockIdx.x / tiles;
  const int g = bg % a.Hkv;
  const int b = bg / a.Hkv;
  const KVPlan pl = make_kvplan(a, b, tile_id);
  if (pl.sep && pl.tile * kTile >= a.sep_count[b]) return;  // no such separator tile (uniform per CTA)
  const int n = pl.n;
  const int rep = a.Hq / a.Hkv;

  if (threadIdx.x == 0) {
    *early = status_failed(a.status) ? 1 : 0;
    *abort_i = 0;
    mbar_init(kv_full, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(q_full + s, 1);
      mbar_init(q_empty + s, 1);
    }
    mbar_init(s_full, 1);
    mbar_init(dp_full, 1);
    mbar_init(p_full, 256);
    mbar_init(ds_full, 256);
    mbar_init(kv_done, 1);
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

  if (warp == 8) {
    // ===================== producer: K, V once; Q, dO and row statistics per step =====================
    if (lane == 0 && n > 0) {
      const int row = pl.tile * kTile;
      // capped separators pair R(L) q_i with the raw keys; band tiles R(i) q_i with R(j) k_j
      const CUtensorMap* qmap = (pl.sep && a.capped_sep) ? &tmQc : &tmQ;
      mbar_expect_tx(kv_full, 2 * kTileBytes);
      for (int c = 0; c < kChunks; ++c) {
        tma_load_4d(sK + c * kChunkBytes, pl.sep ? &tmKg : &tmK, kv_full, c * 64, row, g, b);
        tma_load_4d(sV + c * kChunkBytes, pl.sep ? &tmVg : &tmV, kv_full, c * 64, row, g, b);
      }
      int issued = 0;
      bool ok = true;
      for (int s = 0; s < n && ok; ++s) {
        const int h = g * rep + s / pl.n_t;
        const int t = pl.t_lo + s % pl.n_t;
        const int st = s & 1;
        if (s >= 2) ok = mbar_wait(q_empty + st, ((s >> 1) - 1) & 1, abort_flag, a.status, 71);
        if (!ok) break;
        mbar_expect_tx(q_full + st, 2 * kTileBytes + kStatBytes);
        for (int c = 0; c < kChunks; ++c) {
          tma_load_4d(sQ + st * kTileBytes + c * kChunkBytes, qmap, q_full + st, c * 64, t * kTile, h, b);
          tma_load_4d(sDO + st * kTileBytes + c * kChunkBytes, &tmDO, q_full + st, c * 64, t * kTile, h, b);
        }
        const int64_t srow = ((int64_t)b * a.Hq + h) * a.Tpad + (int64_t)t * kTile;
        tc::bulk_load(sStat + st * 2 * kTile, a.nlse2 + srow, kTile * 4, q_full + st);
        tc::bulk_load(sStat + st * 2 * kTile + kTile, a.Dsum + srow, kTile * 4, q_full + st);
        ++issued;
      }
      if (!ok) {
        tc::wait_raw(kv_full, 0);
        for (int s = max(0, issued - 2); s < issued; ++s) tc::wait_raw(q_full + (s & 1), (s >> 1) & 1);
      }
    }
  } else if (warp == 9) {
    // ===================== MMA issuer =====================
    // S(0), dP(0), then per step s: dV(s), S(s+1), dK(s), dP(s+1).
    if (n > 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, 128, false);
      constexpr uint32_t idesc_kv = idesc_bf16_f32(128, D, true);
      const uint64_t dk = smem_desc_sw128(smem_u32(sK), 16, 1024);
      const uint64_t dv = smem_desc_sw128(smem_u32(sV), 16, 1024);
      const uint64_t dq_ = smem_desc_sw128(smem_u32(sQ), 16, 1024);
      const uint64_t ddo = smem_desc_sw128(smem_u32(sDO), 16, 1024);
      const uint64_t dqm = smem_desc_sw128(smem_u32(sQ), kChunkBytes, 1024);   // Q as an MN-major operand
      const uint64_t ddom = smem_desc_sw128(smem_u32(sDO), kChunkBytes, 1024); // dO as an MN-major operand
      auto wait_all = [&](uint64_t* bar, uint32_t parity, int site) -> bool {
        const bool r = mbar_wait(bar, parity, abort_flag, a.status, site);
        return __all_sync(0xffffffffu, r);
      };
      auto koff = [&](int kk) -> uint64_t { return (uint64_t)(((kk >> 2) * kChunkBytes + (kk & 3) * 32) >> 4); };
      auto stage = [&](uint64_t d, int s) -> uint64_t { return d + (uint64_t)(((s & 1) * kTileBytes) >> 4); };
      auto issue_s = [&](int s) -> bool {
        if (!wait_all(q_full + (s & 1), (s >> 1) & 1, 72)) return false;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          tc::mma_ss(tmem, dk + koff(kk), stage(dq_, s) + koff(kk), idesc_s, kk > 0 ? 1u : 0u);
        tc::commit(s_full);
        return true;
      };
      auto issue_dp = [&](int s) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          tc::mma_ss(tmem + kTmemDP, dv + koff(kk), stage(ddo, s) + koff(kk), idesc_s, kk > 0 ? 1u : 0u);
        tc::commit(dp_full);
      };
      bool ok = wait_all(kv_full, 0, 70);
      ok = ok && issue_s(0);
      if (ok) issue_dp(0);
      for (int s = 0; s < n && ok; ++s) {
        ok = wait_all(p_full, s & 1, 73);
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < kTile / 16; ++kk)
          tc::mma_ts(tmem + kTmemDV, tmem + kk * 8, stage(ddom, s) + (uint64_t)((kk * 16 * 128) >> 4), idesc_kv,
                     (s > 0 || kk > 0) ? 1u : 0u);
        if (s + 1 < n) ok = issue_s(s + 1);
        if (!ok) break;
        ok = wait_all(ds_full, s & 1, 74);
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < kTile / 16; ++kk)
          tc::mma_ts(tmem + kTmemDK, tmem + kTmemDP + kk * 8, stage(dqm, s) + (uint64_t)((kk * 16 * 128) >> 4),
                     idesc_kv, (s > 0 || kk > 0) ? 1u : 0u);
        tc::commit(q_empty + (s & 1));
        if (s + 1 < n) issue_dp(s + 1);
      }
      if (ok) tc::commit(kv_done);
      tc::commit(drain);
      tc::wait_raw(drain, 0);
    }
    __syncwarp();
  } else if (warp < 8) {
    // ===================== P^T, dS^T + epilogue (warps 0-7) =====================
    const int rr = tc::pair_row(warp, lane);  // key row of the tile
    const int hc = lane >> 4;                 // query columns 64 hc + [0, 64)
    const uint32_t lane_off = tc::pair_lane_off(warp);
    const float sl2 = a.scale_log2;
    int j = -1;  // this row's key position (-1: no key)
    if (!pl.sep) {
      const int jj = pl.tile * kTile + rr;
      if (jj < a.T) j = jj;
    } else if (pl.tile * kTile + rr < a.sep_count[b]) {
      j = a.sep_pos[(size_t)b * a.T + pl.tile * kTile + rr];
    }
    const bool live = j >= 0 && (pl.sep || j >= a.n_start);  // band rows of sink keys take no part
    // a band key that is a separator kept by the band beyond the window
    bool key_sep = false;
    if (!pl.sep && live && a.w_sepband > a.window) {
      const uint2 wd = a.sep_words[(size_t)b * (a.T / 32 + 1) + (j >> 5)];
      key_sep = ((wd.y >> (j & 31)) & 1u) != 0;
    }
    bool ok = true;
    for (int s = 0; s < n; ++s) {
      const int h = g * rep + s / pl.n_t;
      const int t = pl.t_lo + s % pl.n_t;
      const int ic = t * kTile + 64 * hc;  // query position of this lane's column 0
      const float* nls = sStat + (s & 1) * 2 * kTile + 64 * hc;
      const float* dss = nls + kTile;
      ok = ok && mbar_wait(s_full, s & 1, abort_flag, a.status, 75);
      tc_fence_after();
      // kept columns [c_lo, c_hi]: band rows j <= i <= j + w (j + w_sepband
      // for a separator when the band also carries the uncapped ones);
      // compacted separators i > j + split
      int c_lo, c_hi;
      if (!live) {
        c_lo = 1;
        c_hi = 0;
      } else if (!pl.sep) {
        c_lo = j - ic;
        c_hi = j + (key_sep ? a.w_sepband : a.window) - ic;
      } else {
        c_lo = j + a.sep_split + 1 - ic;
        c_hi = 63;
      }
      c_hi = min(c_hi, a.T - 1 - ic);
      float sv[64];
      tc::ld16x2<64>(tmem + lane_off, sv);
      tc::ld16x2<64>(tmem + lane_off + 32, sv + 32);
      tc_wait_ld();
      if constexpr (kAlibi) {
        const float sq = alibi_slope_qk(h, a.Hq, a.d);
        if (pl.sep) {
          const float cb = sq * (float)a.alibi_cap;
#pragma unroll
          for (int c = 0; c < 64; ++c) sv[c] -= cb;
        } else {
          const float base = -sq * (float)(ic - j);
#pragma unroll
          for (int c = 0; c < 64; ++c) sv[c] += fmaf(-(float)c, sq, base);
        }
      }
#pragma unroll
      for (int c = 0; c < 64; ++c)
        sv[c] = (c < c_lo || c > c_hi) ? 0.f : ex2_approx(fmaf(sv[c], sl2, nls[c]));
      pack_store64(tmem + lane_off, sv);
      tc_wait_st();
      tc_fence_before();
      if (ok) mbar_arrive(p_full);
      ok = ok && mbar_wait(dp_full, s & 1, abort_flag, a.status, 76);
      tc_fence_after();
      float dp[64];
      tc::ld16x2<64>(tmem + kTmemDP + lane_off, dp);
      tc::ld16x2<64>(tmem + kTmemDP + lane_off + 32, dp + 32);
      tc_wait_ld();
#pragma unroll
      for (int c = 0; c < 64; ++c) sv[c] *= dp[c] - dss[c];
      pack_store64(tmem + kTmemDP + lane_off, sv);
      tc_wait_st();
      tc_fence_before();
      if (ok) mbar_arrive(ds_full);
    }

    // ---- epilogue: dK (rotated back by R(j)^T unless a capped separator), dV ----
    if (n > 0) {
      ok = ok && mbar_wait(kv_done, 0, abort_flag, a.status, 77);
      tc_fence_after();
    }
    const int half = D / 2;
    const float scale = rsqrtf((float)D);
    const int slot = pl.tile * kTile + rr;
    const int64_t krow = pl.sep ? ((int64_t)b * a.Hkv + g) * a.Tpad + slot : ((int64_t)b * a.Hkv + g) * a.T + j;
    float* dk_out = (pl.sep ? a.dk_sep : a.dk_band) + krow * D;
    float* dv_out = (pl.sep ? a.dv_sep : a.dv_band) + krow * D;
    const bool rotate = !(pl.sep && a.capped_sep);
#pragma unroll 1
    for (int cc = 0; cc < half; cc += 32) {
      float v[32], k[32];
      if (n > 0) {
        tc::ld16x2<D / 2>(tmem + kTmemDV + lane_off + cc, v);
        tc::ld16x2<D / 2>(tmem + kTmemDK + lane_off + cc, k);
        tc_wait_ld();
      } else {
#pragma unroll
        for (int y = 0; y < 32; ++y) v[y] = k[y] = 0.f;
      }
      if (rotate) rotate_back(k, a.tab, j < 0 ? 0 : j, half, cc, hc);
      if (j < 0) continue;
      const int col = hc * half + cc;
#pragma unroll
      for (int y = 0; y < 32; y += 4) {
        *reinterpret_cast<float4*>(dk_out + col + y) =
            make_float4(k[y] * scale, k[y + 1] * scale, k[y + 2] * scale, k[y + 3] * scale);
        *reinterpret_cast<float4*>(dv_out + col + y) = make_float4(v[y], v[y + 1], v[y + 2], v[y + 3]);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <int D, bool kAlibi>
cudaError_t launch_dq_d(const BwdArgs& a, const BwdMaps& m, cudaStream_t st) {
  // at least 116 KB, so that one CTA (holding all 512 TMEM columns) runs per SM
  const size_t bytes = std::max<size_t>(QCfg<D>::kSmem, 116 * 1024);
  cudaError_t e = cudaFuncSetAttribute(bwd_dq_kernel<D, kAlibi>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e != cudaSuccess) return e;
  const unsigned grid = (unsigned)a.B * a.Hq * a.nQT;
  bwd_dq_kernel<D, kAlibi><<<grid, kThreads, bytes, st>>>(a.dq_mode == 1 ? m.qc : m.q, m.dO, m.k, m.v, m.kg, m.vg, a);
  return cudaGetLastError();
}

template <int D, bool kAlibi>
cudaError_t launch_dkv_d(const BwdArgs& a, const BwdMaps& m, cudaStream_t st) {
  const size_t bytes = std::max<size_t>(KVCfg<D>::kSmem, 116 * 1024);
  cudaError_t e = cudaFuncSetAttribute(bwd_dkv_kernel<D, kAlibi>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e != cudaSuccess) return e;
  const unsigned grid = (unsigned)a.B * a.Hkv * (a.gather ? 2 * a.nQT : a.nQT);
  bwd_dkv_kernel<D, kAlibi><<<grid, kThreads, bytes, st>>>(m.q, m.qc, m.dO, m.k, m.v, m.kg, m.vg, a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_bwd_dq(const BwdArgs& a, const BwdMaps& m, cudaStream_t st) {
  if ((int64_t)a.B * a.Hq * a.nQT == 0) return cudaSuccess;
  if (a.d == 128) return a.alibi ? launch_dq_d<128, true>(a, m, st) : launch_dq_d<128, false>(a, m, st);
  if (a.d == 64) return a.alibi ? launch_dq_d<64, true>(a, m, st) : launch_dq_d<64, false>(a, m, st);
  return cudaErrorInvalidValue;
}

cudaError_t launch_bwd_dkv(const BwdArgs& a, const BwdMaps& m, cudaStream_t st) {
  if ((int64_t)a.B * a.Hkv * a.nQT == 0) return cudaSuccess;
  if (a.d == 128) return a.alibi ? launch_dkv_d<128, true>(a, m, st) : launch_dkv_d<128, false>(a, m, st);
  if (a.d == 64) return a.alibi ? launch_dkv_d<64, true>(a, m, st) : launch_dkv_d<64, false>(a, m, st);
  return cudaErrorInvalidValue;
}

}  // namespace sattn
