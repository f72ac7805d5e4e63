// attn_tc2.cu -- K5, two query tiles per CTA: the production attention
// kernel for every case except capped separator tiles (those need a second
// query operand per tile and run on attn_tc3.cu, one query tile per CTA).
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
// Schedule:
//   - one CTA = two 128-row query tiles (Q0 rows i0..i0+127, Q1 the next 128)
//     of one (batch, head); every K/V tile either of them needs is loaded
//     once and used by both;
//   - two softmax warpgroups (one per query tile) ping-pong against the
//     tensor core; the single-thread MMA issuer interleaves
//         PV0(prev), S0(p), PV1(prev), S1(p)
//     so that while one warpgroup turns S into P the tensor core works on the
//     other tile (two independent issuers let the warpgroups fall into
//     lockstep and measured slower);
//   - P (bf16) is written back into TMEM over its own S columns and the PV
//     product reads it from there (A operand in tensor memory), so P never
//     touches shared memory;
//   - TMEM: S0 | S1 | O0 | O1 (4 x 128 fp32 columns);
//   - K ring of 2 stages, V ring of 3 stages, each fed by its own producer
//     warp;
//   - the row maximum is taken only on a row's first tile (and on the rare
//     tile whose sum shows that the running reference fell too far behind),
//     not on every tile: see kSumAccept below.
// Ordering facts used: tcgen05.commit arrives only after every earlier MMA
// of the issuing thread completed, so "S_i(p) done" implies "PV_i(prev)
// done" (O_i stable for rescaling); and one thread's MMAs execute in issue
// order, so S_i(p) cannot overwrite P_i before PV_i(prev) has read it.
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

constexpr int kThreads = 384;  // 2 softmax warpgroups + 1 warpgroup holding the producer and MMA warps
// register split (per thread): the producer/MMA warpgroup gives registers to
// the softmax warpgroups; 2*128*kRegSoftmax + 128*kRegCtrl <= 384*168
constexpr int kRegSoftmax = 208;
constexpr int kRegCtrl = 88;
static_assert(2 * 128 * kRegSoftmax + 128 * kRegCtrl <= kThreads * 168, "register split exceeds the launch budget");
constexpr int kKS = 2;         // K stages (K is consumed early: both S products of a position)
constexpr int kVS = 3;         // V stages (V is consumed one position later, by the PV products)
constexpr uint32_t kTmemCols = 512;
constexpr int kMaxSideTopk = 16;  // top-k side keys per row (the library's limit on k)
constexpr int kSinkSmem = 16;     // sink V rows staged in shared memory up to this many

// 32 consecutive 32-bit columns of this thread's lane
__device__ __forceinline__ void tmem_st32u(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
      "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]),
      "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]),
      "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}

// P = 2^(s*sl2 + neg_m) for this thread's row of a 128-key tile, packed to
// bf16 and stored to TMEM over the first 64 S columns (keys 64h..64h+63 go
// to columns 32h..32h+31); returns the fp32 sum of the row's P.
// Masked entries hold -inf and give exactly 0.
__device__ __forceinline__ float emit_p(const float (&sv)[128], float sl2, float neg_m, uint32_t taddr) {
  float ps[8];
#pragma unroll
  for (int y = 0; y < 8; ++y) ps[y] = 0.f;
#pragma unroll
  for (int hf = 0; hf < 2; ++hf) {
    uint32_t pk[32];
#pragma unroll
    for (int c = 0; c < 64; c += 2) {
      float a0, a1;
      fma2(a0, a1, sv[hf * 64 + c], sv[hf * 64 + c + 1], sl2, sl2, neg_m, neg_m);
      const float p0 = ex2_approx(a0);
      const float p1 = ex2_approx(a1);
      add2(ps[(c >> 1) & 3], ps[4 + ((c >> 1) & 3)], p0, p1);
      pk[c >> 1] = pack_bf16x2(p0, p1);
    }
    tmem_st32u(taddr + hf * 32, pk);
  }
  return ((ps[0] + ps[1]) + (ps[2] + ps[3])) + ((ps[4] + ps[5]) + (ps[6] + ps[7]));
}

// O row *= f (warp-collective: every lane takes part, f = 1 leaves a row as is)
template <int D>
__device__ __forceinline__ void scale_o(uint32_t taddr, float f) {
#pragma unroll 1
  for (int c = 0; c < D / 32; ++c) {
    float ov[32];
    tmem_ld32(taddr + c * 32, ov);
    tc_wait_ld();
#pragma unroll
    for (int y = 0; y < 32; ++y) ov[y] *= f;
    tmem_st32(taddr + c * 32, ov);
  }
}

// Union order: gathered positions [0, NG), then band tiles u in [U0, U1].
struct Union {
  int NG, U0, n;
};

__device__ __forceinline__ bool needs(const Plan& p, const Union& un, int pos) {
  if (p.rows == 0) return false;
  if (pos < un.NG) return pos < p.n_gather;
  const int u = un.U0 + (pos - un.NG);
  return u >= p.u_lo && u < p.u_lo + p.n_band;
}

template <int D, bool kAlibi>
__global__ void __launch_bounds__(kThreads, 1)
    attn_tc2_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmKg,
                    const __grid_constant__ CUtensorMap tmVg, const AttnArgs a, int nQB) {
  constexpr uint32_t kTileBytes = D * kTile * 2;
  constexpr int kChunks = D / 64;
  constexpr uint32_t kChunkBytes = kTile * 128;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = base;                                 // Q0 | Q1
  uint8_t* sK = base + 2 * kTileBytes;                // kKS stages
  uint8_t* sV = sK + kKS * kTileBytes;                // kVS stages
  uint64_t* bars = reinterpret_cast<uint64_t*>(sV + kVS * kTileBytes);
  uint64_t* q_full = bars;
  uint64_t* k_full = bars + 1;
  uint64_t* k_empty = k_full + kKS;
  uint64_t* v_full = k_empty + kKS;
  uint64_t* v_empty = v_full + kVS;
  uint64_t* s_full = v_empty + kVS;   // [2]
  uint64_t* p_full = s_full + 2;      // [2]
  uint64_t* o_done = p_full + 2;      // [2]
  uint64_t* drain = o_done + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  int* abort_i = reinterpret_cast<int*>(tmem_slot + 1);
  int* early = abort_i + 1;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int qb = blockIdx.x % nQB;          // query tiles 2 qb, 2 qb + 1 of the Q / O tensors
  const int tg0 = 2 * qb + a.q_pos0 / kTile;  // the first one's position / kTile
  const int bh = blockIdx.x / nQB;
  const int h = bh % a.Hq;
  const int b = bh / a.Hq;
  const int g = h / (a.Hq / a.Hkv);
  const Plan pl0 = make_plan(a, b, h, tg0);
  const Plan pl1 = make_plan(a, b, h, tg0 + 1);
  Union un;
  un.NG = max(pl0.n_gather, pl1.n_gather);
  {
    int u0 = 1 << 30, u1 = -1;
    if (pl0.n_band > 0) {
      u0 = min(u0, pl0.u_lo);
      u1 = max(u1, pl0.u_lo + pl0.n_band - 1);
    }
    if (pl1.n_band > 0) {
      u0 = min(u0, pl1.u_lo);
      u1 = max(u1, pl1.u_lo + pl1.n_band - 1);
    }
    un.U0 = (u1 >= 0) ? u0 : 0;
    un.n = un.NG + ((u1 >= 0) ? (u1 - u0 + 1) : 0);
  }
  const int g_plane = attn::prefix_plane(a, h, g, tg0);

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
      mbar_init(p_full + x, 128);
      mbar_init(o_done + x, 1);
    }
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
  if (warp >= 8) {
    regs_dec<kRegCtrl>();
    if (warp == 8 || warp == 10) {
    // ===================== TMA producers: warp 8 Q and K, warp 10 V =====================
    // two independent streams, so a V stage still in use never delays the next K load
    const bool kstream = (warp == 8);
    if (lane == 0 && un.n > 0) {
      if (kstream) {
        const int i0 = 2 * qb * kTile;
        mbar_expect_tx(q_full, 2 * kTileBytes);
        for (int x = 0; x < 2; ++x)
          for (int c = 0; c < kChunks; ++c)
            tma_load_4d(sQ + x * kTileBytes + c * kChunkBytes, &tmQ, q_full, c * 64, i0 + x * kTile, h, b);
      }
      const int NS = kstream ? kKS : kVS;
      uint8_t* ring = kstream ? sK : sV;
      uint64_t* full = kstream ? k_full : v_full;
      uint64_t* empty = kstream ? k_empty : v_empty;
      int issued = 0;
      bool ok = true;
      for (int p = 0; p < un.n && ok; ++p) {
        const bool gat = p < un.NG;
        const int row = gat ? p * kTile : (un.U0 + p - un.NG) * kTile;
        const int c2 = gat ? g_plane : g;
        const CUtensorMap* mp = kstream ? (gat ? &tmKg : &tmK) : (gat ? &tmVg : &tmV);
        const int st = p % NS;
        if (p >= NS) ok = mbar_wait(empty + st, ((p / NS) - 1) & 1, abort_flag, a.status, kstream ? 31 : 32);
        if (!ok) break;
        mbar_expect_tx(full + st, kTileBytes);
        for (int c = 0; c < kChunks; ++c)
          tma_load_4d(ring + st * kTileBytes + c * kChunkBytes, mp, full + st, c * 64, row, c2, b);
        ++issued;
      }
      if (!ok) {
        if (kstream) tc::wait_raw(q_full, 0);
        for (int p = max(0, issued - NS); p < issued; ++p) tc::wait_raw(full + p % NS, (p / NS) & 1);
      }
    }
    } else if (warp == 9) {
    // ===================== MMA issuer =====================
    // The whole warp runs this loop (an elected lane issues each MMA and
    // commit); both tiles' products go out in the order
    //   PV0(prev), S0(p), PV1(prev), S1(p)
    // which keeps the two softmax warpgroups half a position apart.
    if (un.n > 0) {
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
      int n_pv[2] = {0, 0};    // PV issued per tile
      int prev[2] = {-1, -1};  // union position whose PV is still pending, per tile
      int v_users[kVS];        // PVs still to come for the position held by each V stage
      for (int y = 0; y < kVS; ++y) v_users[y] = 0;
      auto issue_pv = [&](int x) -> bool {
        const int pp = prev[x];
        const int vs = pp % kVS;
        if (!wait_all(p_full + x, n_pv[x] & 1, 34 + x)) return false;
        if (!wait_all(v_full + vs, (pp / kVS) & 1, 36)) return false;
        tc_fence_after();
        const uint64_t bv = dv + (uint64_t)((vs * kTileBytes) >> 4);
#pragma unroll
        for (int kk = 0; kk < kTile / 16; ++kk)
          tc::mma_ts(tmem + 256 + x * 128, tmem + x * 128 + kk * 8, bv + (uint64_t)((kk * 16 * 128) >> 4), idesc_o,
                       (n_pv[x] > 0 || kk > 0) ? 1u : 0u);
        tc::commit(o_done + x);
        // the V stage is free once every tile that uses this position ran its PV
        if (--v_users[vs] == 0) tc::commit(v_empty + vs);
        ++n_pv[x];
        prev[x] = -1;
        return true;
      };
      for (int p = 0; p < un.n && ok; ++p) {
        const int ks = p % kKS;
        const bool need[2] = {needs(pl0, un, p), needs(pl1, un, p)};
        const int users = (need[0] ? 1 : 0) + (need[1] ? 1 : 0);
        bool k_ready = false;
        for (int x = 0; x < 2 && ok; ++x) {
          if (prev[x] >= 0) ok = issue_pv(x);
          if (!ok || !need[x]) continue;
          if (!k_ready) {
            ok = wait_all(k_full + ks, (p / kKS) & 1, 40);
            if (!ok) break;
            k_ready = true;
            v_users[p % kVS] = users;
          }
          tc_fence_after();
          const uint64_t ba = dq + (uint64_t)((x * kTileBytes) >> 4);
          const uint64_t bk = dk + (uint64_t)((ks * kTileBytes) >> 4);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint64_t off = (uint64_t)(((kk >> 2) * kChunkBytes + (kk & 3) * 32) >> 4);
            tc::mma_ss(tmem + x * 128, ba + off, bk + off, idesc_s, kk > 0 ? 1u : 0u);
          }
          tc::commit(s_full + x);
          prev[x] = p;
          if (!((x == 0) && need[1])) tc::commit(k_empty + ks);
        }
        if (ok && users == 0) {
          // no tile reads this position (cannot happen for contiguous plans); release it
          ok = wait_all(k_full + ks, (p / kKS) & 1, 40);
          if (!ok) break;
          tc::commit(k_empty + ks);
          ok = wait_all(v_full + p % kVS, (p / kVS) & 1, 36);
          if (ok) tc::commit(v_empty + p % kVS);
        }
      }
      // pending PVs of the last positions
      for (int x = 0; x < 2 && ok; ++x)
        if (prev[x] >= 0) ok = issue_pv(x);
      tc::commit(drain);
      tc::wait_raw(drain, 0);
    }
    __syncwarp();
    }
  } else {
    regs_inc<kRegSoftmax>();
    // ===================== softmax + epilogue (warpgroups 0 and 1) =====================
    const int x = warp >> 2;  // query tile of this warpgroup
    const Plan& pl = x == 0 ? pl0 : pl1;
    const int r = threadIdx.x & 127;
    const int i0 = (tg0 + x) * kTile;
    const int i = i0 + r;
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + x * 128;
    const uint32_t tO = tmem + 256 + x * 128;
    const float sl2 = a.scale_log2;
    float m_used = -CUDART_INF_F;  // running reference (log2 units) P is taken against
    float l_sum = 0.f;
    int rebase = 0;                // pending: m_used += rebase, O and l_sum *= 2^-rebase
    bool ok = true;
    int k = 0;  // tiles processed by this warpgroup
    for (int p = 0; p < un.n; ++p) {
      if (!needs(pl, un, p)) continue;
      ok = ok && mbar_wait(s_full + x, k & 1, abort_flag, a.status, 41 + x);
      tc_fence_after();
      int c_lo = 0, c_hi = kTile - 1;
      if (p < un.NG) {
        const int r0 = p * kTile;
        if (r0 + kTile > pl.g_full) {
          int lim = min(kTile, pl.g_count - r0);
          if (a.gather_mode == 1) {
            // separators kept by row i: pos < i - w; their count is a prefix count
            const int thr = i - a.window;
            const int cnt = thr > 0 ? sep_before(a.sep_words, a.T, b, thr) : 0;
            lim = max(0, min(lim, cnt - r0));
          }
          c_hi = lim - 1;
        }
      } else {
        const int j0 = (un.U0 + p - un.NG) * kTile;
        const int lo_fix = max(pl.band_lo, a.ns_band);
        const bool full = (j0 + kTile - 1 <= i0) && (j0 >= max(lo_fix, i0 + kTile - 1 - a.w_eff)) &&
                          (i0 + kTile <= a.T);
        if (!full) {
          c_lo = max(lo_fix, i - a.w_eff) - j0;
          c_hi = i - j0;
        }
      }
      const bool partial = (c_lo > 0 || c_hi < kTile - 1);
      float sv[128];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(tS + lane_off + c * 32, sv + c * 32);
      tc_wait_ld();
      if (partial) {
#pragma unroll
        for (int c = 0; c < kTile; ++c)
          if (c < c_lo || c > c_hi) sv[c] = -CUDART_INF_F;  // exp2(-inf) = 0 below
      }
      if constexpr (kAlibi) {
        // ALiBi bias in units of q.k: band keys -m (i - j) (inside the window,
        // below the cap); gathered separators lie beyond w = L: -m L
        const float sq = alibi_slope_qk(h, a.Hq, a.d);
        if (p < un.NG) {
          const float cb = sq * (float)a.alibi_cap;
#pragma unroll
          for (int c = 0; c < kTile; ++c) sv[c] -= cb;
        } else {
          const float base = -sq * (float)(i - (un.U0 + p - un.NG) * kTile);
#pragma unroll
          for (int c = 0; c < kTile; ++c) sv[c] += fmaf((float)c, sq, base);
        }
      }
      // O_x is stable from here on: S_x(p) completing implies the tile's
      // previous PV completed.  First the rebase the previous tile asked for.
      if (__any_sync(0xffffffffu, rebase != 0)) scale_o<D>(tO + lane_off, exp2_neg_int(rebase));
      if (rebase != 0) {
        m_used += (float)rebase;
        l_sum *= exp2_neg_int(rebase);
        rebase = 0;
      }
      bool exact = __any_sync(0xffffffffu, m_used == -CUDART_INF_F);
      float l_tile;
#pragma unroll 1
      for (;;) {
        if (exact) {
          // 16 independent 2-input chains of 8 steps
          float pm[16];
#pragma unroll
          for (int y = 0; y < 16; ++y) pm[y] = sv[y];
#pragma unroll
          for (int c = 16; c < kTile; ++c) pm[c & 15] = fmaxf(pm[c & 15], sv[c]);
#pragma unroll
          for (int w = 8; w > 0; w >>= 1)
#pragma unroll
            for (int y = 0; y < w; ++y) pm[y] = fmaxf(pm[y], pm[y + w]);
          const float m_new = fmaxf(m_used, pm[0] * sl2);
          float alpha = 1.f;
          bool rescale_o = false;
          if (m_new > m_used) {
            alpha = (m_used == -CUDART_INF_F) ? 0.f : ex2_approx(m_used - m_new);
            rescale_o = (k > 0) && (m_used != -CUDART_INF_F);
            l_sum *= alpha;
            m_used = m_new;
          }
          if (__any_sync(0xffffffffu, rescale_o)) scale_o<D>(tO + lane_off, rescale_o ? alpha : 1.f);
        }
        // a row with no key so far has m_used = -inf and every entry masked:
        // with a zero offset each exp2(-inf) is exactly 0
        l_tile = emit_p(sv, sl2, (m_used == -CUDART_INF_F) ? 0.f : -m_used, tS + lane_off);
        if (exact || !__any_sync(0xffffffffu, !(l_tile <= kSumAccept))) break;
        exact = true;  // some row overflowed its bound: redo against the true maxima
      }
      l_sum += l_tile;
      if (l_tile > kSumRebase) rebase = ((__float_as_int(l_tile) >> 23) & 0xff) - 126;  // 2^rebase > l_tile
      tc_wait_st();
      tc_fence_before();
      if (ok) mbar_arrive(p_full + x);
      ++k;
    }

    // ---- epilogue ----
    if (k > 0) {
      ok = ok && mbar_wait(o_done + x, (k - 1) & 1, abort_flag, a.status, 43 + x);
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
    // side keys: the starting span (sinks) and the row's top-k keys, fp32
    // top-k keys are middle keys beyond the cap: ALiBi gives them -m L (sink
    // logits carry their bias from the prep pass)
    const float tkb = kAlibi ? alibi_slope_qk(h, a.Hq, a.d) * (float)a.alibi_cap : 0.f;
    float m_fin = m_used;
    for (int j = 0; j < n_sink; ++j) m_fin = fmaxf(m_fin, sz[j] * sl2);
    float pt[kMaxSideTopk];  // top-k weights, 0 for absent keys
    int jt[kMaxSideTopk];
#pragma unroll
    for (int y = 0; y < kMaxSideTopk; ++y) {
      jt[y] = (y < a.topk) ? tki[y] : -1;
      if (jt[y] >= a.T) jt[y] = -1;
      if (jt[y] >= 0) m_fin = fmaxf(m_fin, (tkz[y] - tkb) * sl2);
    }
    const float alpha = (m_used == -CUDART_INF_F) ? 0.f : ex2_approx(m_used - m_fin);
    float l_fin = l_sum * alpha;
    for (int j = 0; j < n_sink; ++j) l_fin += ex2_approx(sz[j] * sl2 - m_fin);
#pragma unroll
    for (int y = 0; y < kMaxSideTopk; ++y) {
      pt[y] = (jt[y] >= 0) ? ex2_approx((tkz[y] - tkb) * sl2 - m_fin) : 0.f;
      l_fin += pt[y];
    }
    const float inv_l = (l_fin > 0.f) ? 1.f / l_fin : 0.f;
    const __nv_bfloat16* vbase = a.V + (size_t)b * a.v_sb + (size_t)g * a.v_sh;
    __nv_bfloat16* orow = a.O + (size_t)b * a.o_sb + (size_t)h * a.o_sh + (size_t)il * a.o_st;
    // The sinks' V rows are the same for every row of the tile: stage them in
    // this warpgroup's Q tile (free once its last MMA completed).
    const bool sinks_smem = a.n_sink > 0 && a.n_sink <= kSinkSmem;
    const __nv_bfloat16* vsink = reinterpret_cast<const __nv_bfloat16*>(sQ + x * kTileBytes);
    if (sinks_smem) {
      if (k == 0 && un.n > 0) ok = ok && mbar_wait(q_full, 0, abort_flag, a.status, 47);  // its load may be in flight
      uint4* dst = reinterpret_cast<uint4*>(sQ + x * kTileBytes);
      for (int e = r; e < a.n_sink * (D / 8); e += 128)
        dst[e] = *reinterpret_cast<const uint4*>(vbase + (size_t)(e / (D / 8)) * a.v_st + (e % (D / 8)) * 8);
      asm volatile("bar.sync %0, 128;" ::"r"(1 + x) : "memory");  // this warpgroup only
    }
#pragma unroll 1
    for (int c = 0; c < D / 32; ++c) {
      float ov[32];
      if (k > 0) {
        tmem_ld32(tO + lane_off + c * 32, ov);
        tc_wait_ld();
#pragma unroll
        for (int y = 0; y < 32; ++y) ov[y] *= alpha * o_rebase;
      } else {
#pragma unroll
        for (int y = 0; y < 32; ++y) ov[y] = 0.f;
      }
      for (int j = 0; j < n_sink; ++j) {
        const float pkv = ex2_approx(sz[j] * sl2 - m_fin);
        const __nv_bfloat16* vr = sinks_smem ? vsink + j * D + c * 32 : vbase + (size_t)j * a.v_st + c * 32;
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          const uint4 u = reinterpret_cast<const uint4*>(vr)[q4];
          const __nv_bfloat162* hv = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 vv = __bfloat1622float2(hv[e]);
            ov[q4 * 8 + 2 * e] = fmaf(pkv, vv.x, ov[q4 * 8 + 2 * e]);
            ov[q4 * 8 + 2 * e + 1] = fmaf(pkv, vv.y, ov[q4 * 8 + 2 * e + 1]);
          }
        }
      }
      // top-k rows: the 64-byte pieces of up to 4 rows are loaded before any is used
      for (int t0 = 0; t0 < a.topk; t0 += 4) {
        uint4 vv4[4][4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          int jj = -1;
#pragma unroll
          for (int y = 0; y < kMaxSideTopk; ++y)
            if (y == t0 + u) jj = jt[y];
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4)
            vv4[u][q4] = (jj >= 0) ? reinterpret_cast<const uint4*>(vbase + (size_t)jj * a.v_st + c * 32)[q4]
                                   : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          float pkv = 0.f;
#pragma unroll
          for (int y = 0; y < kMaxSideTopk; ++y)
            if (y == t0 + u) pkv = pt[y];
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            const __nv_bfloat162* hv = reinterpret_cast<const __nv_bfloat162*>(&vv4[u][q4]);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float2 vv = __bfloat1622float2(hv[e]);
              ov[q4 * 8 + 2 * e] = fmaf(pkv, vv.x, ov[q4 * 8 + 2 * e]);
              ov[q4 * 8 + 2 * e + 1] = fmaf(pkv, vv.y, ov[q4 * 8 + 2 * e + 1]);
            }
          }
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
    if (row_ok) a.lse[row_id] = (l_fin > 0.f) ? (m_fin + __log2f(l_fin)) * 0.69314718055994531f : -CUDART_INF_F;
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ALiBi is a template parameter: a run-time test inside the key loop
// measured 3-5 % slower on the kernels without it
template <int D, bool kAlibi>
cudaError_t launch_d(const AttnArgs& a, const AttnMaps& m, cudaStream_t st) {
  const size_t tile = (size_t)D * kTile * 2;
  const size_t bytes = std::max<size_t>(116 * 1024, 1024 + tile * (2 + kKS + kVS) + 256);
  cudaError_t e =
      cudaFuncSetAttribute(attn_tc2_kernel<D, kAlibi>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e != cudaSuccess) return e;
  const int nQB = (a.nQT + 1) / 2;
  const unsigned grid = (unsigned)a.B * a.Hq * nQB;
  attn_tc2_kernel<D, kAlibi><<<grid, kThreads, bytes, st>>>(m.q, m.k, m.v, m.kg, m.vg, a, nQB);
  return cudaGetLastError();
}

}  // namespace

// Two-tile kernel; the caller routes capped separator tiles (q2) and
// segment lengths that are not multiples of 256 to launch_attn_tc3.
cudaError_t launch_attn_tc2(const AttnArgs& a, const AttnMaps& m, cudaStream_t st) {
  if (a.B * a.Hq * a.nQT == 0) return cudaSuccess;
  if (a.q2) return cudaErrorInvalidValue;
  if (a.d == 128) return a.alibi ? launch_d<128, true>(a, m, st) : launch_d<128, false>(a, m, st);
  if (a.d == 64) return a.alibi ? launch_d<64, true>(a, m, st) : launch_d<64, false>(a, m, st);
  return cudaErrorInvalidValue;
}

}  // namespace sattn
