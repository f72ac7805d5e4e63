// attn_common.cuh -- pieces shared by the two forward attention kernels
// (attn_tc2.cu: two query tiles per CTA, a row per thread; attn_tc3.cu: one
// query tile per CTA, a row per lane pair): the tile plan of a query tile,
// the softmax constants and small arithmetic helpers.  The issue helpers
// (elected MMA / commit, bounded raw waits, 16x32bx2 TMEM accesses) come
// from tc_ops.cuh, the paired fp32 arithmetic from simt.cuh.
#pragma once

#include "kernels.cuh"
#include "simt.cuh"
#include "tc_ops.cuh"

namespace sattn {
namespace attn {

// A tile's P is computed against the row's running reference m (log2
// units) without first taking the tile's row maximum.  That is exact
// arithmetic for softmax as long as nothing overflows: P = 2^(s - m) is
// stored in bf16 and summed in fp32, both of which keep their relative
// precision at any magnitude.  A row whose tile sum exceeds kSumAccept
// (this includes +inf) redoes the tile against its true maximum; a row whose
// accepted sum exceeds kSumRebase moves m up by a power of two before its
// next tile, so the rescale of O and l is exact.
constexpr float kSumAccept = 0x1p32f;
constexpr float kSumRebase = 0x1p8f;

// 2^-e for an integer e in [0, 126]
__device__ __forceinline__ float exp2_neg_int(int e) { return __int_as_float((127 - e) << 23); }

// Rows of the Q / O / LSE tensors, and the prefix plane of a long head's
// query tile (tile: position / kTile).
__device__ __forceinline__ int q_rows(const AttnArgs& a) { return a.T_q > 0 ? a.T_q : a.T; }
__device__ __forceinline__ int prefix_plane(const AttnArgs& a, int h, int g, int tile) {
  return (a.gather_mode == 2 && a.long_slot[h] >= 0)
             ? a.long_slot[h] * (a.seg_N - a.seg_s0) + (tile * kTile) / a.seg_S - a.seg_s0
             : g;
}

// Key tiles one 128-row query tile visits: gathered tiles [0, n_gather),
// then band key tiles [u_lo, u_lo + n_band).  t: the tile's position / kTile.
struct Plan {
  int g_count, g_full, n_gather, band_lo, u_lo, n_band, rows;  // rows: valid rows of the tile (0 = none)
};

__device__ __forceinline__ Plan make_plan(const AttnArgs& a, int b, int h, int t) {
  Plan p;
  p.g_count = 0;
  p.g_full = 0;
  p.band_lo = 0;
  const int i0 = t * kTile;
  p.rows = (i0 < a.T) ? min(kTile, a.T - i0) : 0;
  if (p.rows == 0) {
    p.n_gather = p.n_band = p.u_lo = 0;
    return p;
  }
  if (a.gather_mode == 1) {
    p.g_full = a.ranges[(b * a.nQT + t) * 2 + 0];
    p.g_count = a.ranges[(b * a.nQT + t) * 2 + 1];
  } else if (a.gather_mode == 3) {
    // cross-attention over a compressed context: every row keeps all of it
    p.g_count = p.g_full = a.cross_len;
  } else if (a.gather_mode == 2) {
    const int s = i0 / a.seg_S;
    const int seg0 = s * a.seg_S;
    const int slot = a.long_slot[h];
    if (slot >= 0) {
      p.band_lo = seg0;
      if (s > 0) p.g_count = p.g_full = a.prefix_cnt[(b * a.n_long + slot) * (a.seg_N - a.seg_s0) + (s - a.seg_s0)];
    } else {
      p.band_lo = s > 0 ? max(0, seg0 - a.seg_M) : 0;
    }
  }
  p.n_gather = (p.g_count + kTile - 1) / kTile;
  const int i_last = i0 + p.rows - 1;
  const int j_lo = max(max(p.band_lo, 0), max(i0 - max(a.w_eff, a.w_sepband), a.ns_band));
  if (j_lo > i_last || a.gather_mode == 3) {
    p.u_lo = 0;
    p.n_band = 0;
  } else {
    p.u_lo = j_lo / kTile;
    p.n_band = i_last / kTile - p.u_lo + 1;
  }
  return p;
}

}  // namespace attn
}  // namespace sattn
