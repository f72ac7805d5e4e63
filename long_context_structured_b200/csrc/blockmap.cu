// blockmap.cu -- K2: block map and separator compaction.
//
// Structural mask of query row i ("LM-Infinite", section 方法, equation A_i;
// "SepLLM", section 五.2, mask M_ij), top-k excluded:
//   m_ij = [j <= i] * ( [j < n_start] + [i - j <= w] + [sep_j and j < i] > 0 ).
// Outputs, per sequence b:
//   sep_pos[b][r]  positions of the separators j >= n_start in ascending
//                  order, then -1
//   sep_count[b]
//   ranges[b][t]   (#sep with j < 128t - w, #sep with j < last_row(t) - w)
//   cls[b][t][u]   0 empty / 1 partial / 2 full for the 128x128 tile (t, u)
//                  over its in-range (i, j) pairs.
// The classes follow from interval arithmetic on the sink span and the band
// plus separator counts; no mask is materialised.
//
// Scratch (blockmap_scratch_bytes):
//   word prefix [B][T/32 + 1] uint2: .x = separators (j >= n_start) before
//       position 32 x, .y = bit e set iff 32 x + e is one; the count of
//       separators before any x is then one load and one popcount;
//   far class  [B][nKT rounded up to 16] u8: the class of key tile u for
//       every query tile t whose band cannot reach it (the last key of u is
//       more than w before the first query of t), which then depends on u
//       alone: 2 if every key of u is a sink or a separator, 1 if any is,
//       else 0;
//   mixed pieces [B][nQT][Kc] 16-byte: the 16-tile pieces v_lo(t) .. v_hi(t)
//       of row t, v_lo = floor(u_far(t) / 16), v_hi = floor(t / 16), where
//       u_far(t) = max(0, t - bt), bt = ceil(w / 128), is the first key tile
//       the band can reach; Kc = min(ceil(nQT / 16), floor(bt / 16) + 2)
//       bounds their number.  A piece before v_lo lies wholly in the far
//       part, a piece after v_hi wholly above the diagonal.
// Two launches:
//   sep_scan_kernel    one CTA per sequence: 32-flag words loaded 16 bytes at
//                      a time (a thread's four words are one key tile, whose
//                      far class follows from their count), block scan of
//                      the counts into the word prefix (kept in shared memory
//                      as well when it fits), then sep_pos in one coalesced
//                      pass (rank r < count selects its bit through the word
//                      prefix, the rest is -1), ranges and the mixed pieces;
//   tile_class_kernel  grid-stride over 16-byte pieces of cls, each a copy of
//                      the far row, zero, or a copy of a mixed piece: pure
//                      store bandwidth with no per-byte work.
#include <cstdint>

#include "kernels.cuh"

namespace sattn {

namespace {

constexpr int kScanThreads = 256;
constexpr int kWordsPerThread = 4;
constexpr int kRoundWords = kScanThreads * kWordsPerThread;
constexpr int kClassThreads = 256;
constexpr int kStageBytes = 96 * 1024;
static_assert(kWordsPerThread * 32 == kTile, "a scan thread's words are one key tile");

struct Layout {
  int nW, nQT, far_stride, Kc, band_tiles;
  size_t wp_off, far_off, mix_off, total;
};

__host__ __device__ inline Layout layout_of(int B, int T, int window) {
  Layout L;
  L.nW = T / 32 + 1;
  L.nQT = (T + kTile - 1) / kTile;
  L.far_stride = (L.nQT + 15) / 16 * 16;
  const long long bt = ((long long)window + kTile - 1) / kTile;
  L.band_tiles = bt > L.nQT ? L.nQT : (int)bt;
  const int pieces = (L.nQT + 15) / 16;
  L.Kc = L.band_tiles / 16 + 2 < pieces ? L.band_tiles / 16 + 2 : pieces;
  L.wp_off = 0;
  L.far_off = ((size_t)B * L.nW * 8 + 15) / 16 * 16;
  L.mix_off = L.far_off + (size_t)B * L.far_stride;
  L.total = L.mix_off + (size_t)B * L.nQT * L.Kc * 16;
  return L;
}

// separators (j >= n_start) before x, x clamped to [0, T]
__device__ __forceinline__ int pre_at(const uint2* wp, int T, int x) {
  x = max(0, min(T, x));
  const uint2 e = wp[x >> 5];
  return (int)e.x + __popc(e.y & ((1u << (x & 31)) - 1u));
}

// bit k of the result = byte k of v is non-zero.  After the compare each byte
// is 0 or 1; the multiply adds byte k shifted by 8k + 7m for m = 0..3, so
// byte k lands on bit 21 + k exactly once and no two terms share a bit.
__device__ __forceinline__ uint32_t nonzero_nibble(uint32_t v) {
  const uint32_t x = __vcmpne4(v, 0u) & 0x01010101u;
  return ((x * 0x00204081u) >> 21) & 0xFu;
}

__device__ __forceinline__ uint32_t nonzero_bits16(uint4 v) {
  return nonzero_nibble(v.x) | nonzero_nibble(v.y) << 4 | nonzero_nibble(v.z) << 8 | nonzero_nibble(v.w) << 12;
}

// class of key tile u for query tile t (u <= t), from the word prefix
__device__ __forceinline__ uint8_t tile_class(const uint2* wp, int T, int ns, int w, int t, int u) {
  const int i0 = t * kTile;
  const int i1 = min(T - 1, i0 + kTile - 1);
  const int j0 = u * kTile;
  const int j1 = min(T - 1, j0 + kTile - 1);
  if (j0 > i1) return 0;
  // full: causal for every row, and every key either a sink, inside the band
  // of the last row, or a separator (j < i holds since j <= i0 <= i and j = i
  // lies in the band)
  if (j1 <= i0) {
    const int lo = max(j0, ns);
    const int hi = (int)min((long long)j1, (long long)i1 - w - 1);  // keys that need the separator rule
    if (lo > hi) return 2;
    if (pre_at(wp, T, hi + 1) - pre_at(wp, T, lo) == hi - lo + 1) return 2;
  }
  if (j0 < ns || (long long)j1 >= (long long)max(i0, j0) - w) return 1;
  const int lo = max(j0, ns);
  const int hi = min(j1, i1 - 1);
  return (lo <= hi && pre_at(wp, T, hi + 1) - pre_at(wp, T, lo) > 0) ? 1 : 0;
}

// position of the k-th (0-based) set bit of y, k < popc(y): halve the window
// five times, stepping into the upper half when the lower one holds <= k
__device__ __forceinline__ int nth_set_bit(uint32_t y, int k) {
  int p = 0;
#pragma unroll
  for (int sh = 16; sh > 0; sh >>= 1) {
    const int c = __popc(y & ((1u << sh) - 1u));
    if (k >= c) {
      k -= c;
      y >>= sh;
      p += sh;
    }
  }
  return p;
}

// Position of the r-th separator (0-based, r < count), from the word prefix:
// the last word whose count before it is <= r holds it (words after it start
// above r), at the (r - before)-th set bit.  `w` is a starting guess at or
// before the answer; the result's word is left in it.
__device__ __forceinline__ int select_sep(const uint2* wp, int nW, int r, int& w) {
  uint2 e = wp[w];
  while (w + 1 < nW && (int)wp[w + 1].x <= r) e = wp[++w];
  return w * 32 + nth_set_bit(e.y, r - (int)e.x);
}

// first word whose count-before exceeds r, minus one (binary search)
__device__ __forceinline__ int word_of_rank(const uint2* wp, int nW, int r) {
  int lo = 0, hi = nW - 1;  // wp[0].x = 0 <= r
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if ((int)wp[mid].x <= r) lo = mid;
    else hi = mid - 1;
  }
  return lo;
}

// the far row follows the word-prefix row in shared memory, 16-byte aligned
__host__ __device__ inline size_t stage_far_offset(int nW) { return ((size_t)nW * 8 + 15) / 16 * 16; }

// Dynamic shared memory: the word-prefix row then the far row when they fit
// in kStageBytes (staged = 1), else both are read from global memory.
__global__ void __launch_bounds__(kScanThreads) sep_scan_kernel(BlockmapArgs a, int staged) {
  extern __shared__ __align__(16) uint8_t stage[];
  __shared__ int warp_tot[kScanThreads / 32];
  __shared__ int carry_sh;
  const int b = blockIdx.x;
  const int T = a.T, ns = a.n_start;
  const Layout L = layout_of(a.B, T, a.window);
  uint8_t* scratch = static_cast<uint8_t*>(a.scratch);
  uint2* wp_g = reinterpret_cast<uint2*>(scratch + L.wp_off) + (size_t)b * L.nW;
  uint8_t* far_g = scratch + L.far_off + (size_t)b * L.far_stride;
  uint2* wp = staged ? reinterpret_cast<uint2*>(stage) : wp_g;
  uint8_t* far = staged ? stage + stage_far_offset(L.nW) : far_g;
  const uint8_t* f = a.is_sep ? a.is_sep + (size_t)b * T : nullptr;
  const bool vec = f && (reinterpret_cast<uintptr_t>(f) & 15) == 0;
  int32_t* pos = a.sep_pos + (size_t)b * T;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int n_flag_words = (T + 31) / 32;  // nW - 1 when T % 32 == 0: the sentinel follows the loop
  if (threadIdx.x == 0) carry_sh = 0;
  for (int base = 0; base < n_flag_words; base += kRoundWords) {
    // this thread's words: the 128 keys of key tile u
    const int w0 = base + threadIdx.x * kWordsPerThread;
    const int u = w0 / kWordsPerThread;
    uint32_t m[kWordsPerThread];
#pragma unroll
    for (int q = 0; q < kWordsPerThread; ++q) {
      const int j0 = (w0 + q) * 32;
      uint32_t mq = 0;
      if (f && j0 < T) {
        if (vec && j0 + 32 <= T) {
          const uint4 lo = __ldg(reinterpret_cast<const uint4*>(f + j0));
          const uint4 hi = __ldg(reinterpret_cast<const uint4*>(f + j0 + 16));
          mq = nonzero_bits16(lo) | nonzero_bits16(hi) << 16;
        } else {
          const int n = min(32, T - j0);
          for (int e = 0; e < n; ++e) mq |= (f[j0 + e] != 0 ? 1u : 0u) << e;
        }
        if (j0 < ns) mq = (ns - j0 >= 32) ? 0u : (mq & ~((1u << (ns - j0)) - 1u));
      }
      m[q] = mq;
    }
    int cnt = 0;
#pragma unroll
    for (int q = 0; q < kWordsPerThread; ++q) cnt += __popc(m[q]);
    // far class of key tile u: every key a sink or a separator -> 2, any -> 1
    if (a.cls && u < L.nQT) {
      const int j0 = u * kTile, j1 = min(T - 1, j0 + kTile - 1);
      const int lo = max(j0, ns);
      const uint8_t c = (lo > j1 || cnt == j1 - lo + 1) ? 2 : ((j0 < ns || cnt > 0) ? 1 : 0);
      far[u] = c;
      if (staged) far_g[u] = c;
    }
    int incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    if (warp == 0) {
      const int v = lane < kScanThreads / 32 ? warp_tot[lane] : 0;
      int sc = v;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, sc, o);
        if (lane >= o) sc += y;
      }
      if (lane < kScanThreads / 32) warp_tot[lane] = sc - v;  // exclusive prefix of warp totals
    }
    __syncthreads();
    int run = carry_sh + warp_tot[warp] + incl - cnt;
#pragma unroll
    for (int q = 0; q < kWordsPerThread; ++q) {
      const int wq = w0 + q;
      if (wq < n_flag_words) {
        const uint2 e = make_uint2((uint32_t)run, m[q]);
        wp[wq] = e;
        if (staged) wp_g[wq] = e;
      }
      run += __popc(m[q]);
    }
    __syncthreads();  // carry_sh and warp_tot are consumed
    if (threadIdx.x == kScanThreads - 1) carry_sh = run;
    __syncthreads();
  }
  const int total = carry_sh;
  if (threadIdx.x == 0) {
    a.sep_count[b] = total;
    if (n_flag_words < L.nW) {
      const uint2 e = make_uint2((uint32_t)total, 0u);
      wp[n_flag_words] = e;
      if (staged) wp_g[n_flag_words] = e;
    }
  }
  __syncthreads();  // the word prefix and the far row are complete
  // sep_pos in one coalesced pass: rank x < total -> its position, else -1;
  // four consecutive ranks per thread, 16-byte stores where aligned
  if ((reinterpret_cast<uintptr_t>(pos) & 15) == 0) {
    const int n4 = T >> 2;
    for (int x4 = threadIdx.x; x4 < n4; x4 += kScanThreads) {
      const int r0 = 4 * x4;
      int4 o = make_int4(-1, -1, -1, -1);
      if (r0 < total) {
        int w = word_of_rank(wp, L.nW, r0);
        o.x = select_sep(wp, L.nW, r0, w);
        if (r0 + 1 < total) o.y = select_sep(wp, L.nW, r0 + 1, w);
        if (r0 + 2 < total) o.z = select_sep(wp, L.nW, r0 + 2, w);
        if (r0 + 3 < total) o.w = select_sep(wp, L.nW, r0 + 3, w);
      }
      reinterpret_cast<int4*>(pos)[x4] = o;
    }
    for (int x = 4 * n4 + threadIdx.x; x < T; x += kScanThreads) {
      int w = x < total ? word_of_rank(wp, L.nW, x) : 0;
      pos[x] = x < total ? select_sep(wp, L.nW, x, w) : -1;
    }
  } else {
    for (int x = threadIdx.x; x < T; x += kScanThreads) {
      int w = x < total ? word_of_rank(wp, L.nW, x) : 0;
      pos[x] = x < total ? select_sep(wp, L.nW, x, w) : -1;
    }
  }
  const int w = a.window;
  for (int t = threadIdx.x; t < L.nQT; t += kScanThreads) {
    const int i0 = t * kTile;
    const int i1 = min(T - 1, i0 + kTile - 1);
    a.ranges[((size_t)b * L.nQT + t) * 2 + 0] = pre_at(wp, T, i0 - w);
    a.ranges[((size_t)b * L.nQT + t) * 2 + 1] = pre_at(wp, T, i1 - w);
  }
  if (!a.cls) return;
  // mixed pieces: the far bytes (u < u_far) as one 16-byte load masked to
  // their count, then tile_class over this lane's near tiles only (u_far..t
  // within the piece), so lanes do not run it for each other's bytes
  uint4* mix = reinterpret_cast<uint4*>(scratch + L.mix_off) + (size_t)b * L.nQT * L.Kc;
  const int n_mix = L.nQT * L.Kc;
  for (int e = threadIdx.x; e < n_mix; e += kScanThreads) {
    const int t = e / L.Kc, k = e - t * L.Kc;
    const int u_far = max(0, t - L.band_tiles);
    const int v = u_far / 16 + k;
    if (v > t / 16) continue;  // never read
    const int keep = min(16, max(0, u_far - 16 * v));  // far bytes in this piece
    unsigned long long lo = 0, hi = 0;
    if (keep > 0) {
      const uint4 fv = *reinterpret_cast<const uint4*>(far + 16 * v);
      lo = (unsigned long long)fv.y << 32 | fv.x;
      hi = (unsigned long long)fv.w << 32 | fv.z;
      lo &= keep >= 8 ? ~0ull : (1ull << (8 * keep)) - 1ull;
      hi &= keep >= 16 ? ~0ull : (keep <= 8 ? 0ull : (1ull << (8 * (keep - 8))) - 1ull);
    }
    const int n1 = min(16 * v + 15, t);
    for (int uu = max(16 * v, u_far); uu <= n1; ++uu) {
      const unsigned long long c = tile_class(wp, T, ns, w, t, uu);
      const int kb = uu - 16 * v;
      if (kb < 8) lo |= c << (8 * kb);
      else hi |= c << (8 * (kb - 8));
    }
    mix[e] = make_uint4((uint32_t)lo, (uint32_t)(lo >> 32), (uint32_t)hi, (uint32_t)(hi >> 32));
  }
}

// index math in I: 32 bits whenever the piece count fits
template <typename I>
__global__ void __launch_bounds__(kClassThreads) tile_class_kernel(BlockmapArgs a, int vec) {
  const Layout L = layout_of(a.B, a.T, a.window);
  const uint8_t* scratch = static_cast<const uint8_t*>(a.scratch);
  const uint8_t* far = scratch + L.far_off;
  const uint8_t* mix = scratch + L.mix_off;
  const I nQT = (I)L.nQT, Kc = (I)L.Kc;
  const I stride = (I)gridDim.x * blockDim.x;
  const I tid = (I)blockIdx.x * blockDim.x + threadIdx.x;
  if (vec) {
    const I per_row = nQT / 16;
    const I n = (I)a.B * nQT * per_row;
    for (I e = tid; e < n; e += stride) {
      const I row = e / per_row;
      const I v = e - row * per_row;
      const I b = row / nQT, t = row - b * nQT;
      const I v_lo = (t > (I)L.band_tiles ? t - (I)L.band_tiles : 0) / 16, v_hi = t / 16;
      uint4 out = make_uint4(0u, 0u, 0u, 0u);
      if (v < v_lo) out = __ldg(reinterpret_cast<const uint4*>(far + (size_t)b * L.far_stride + 16 * v));
      else if (v <= v_hi) out = __ldg(reinterpret_cast<const uint4*>(mix + ((size_t)row * Kc + (v - v_lo)) * 16));
      *reinterpret_cast<uint4*>(a.cls + (size_t)e * 16) = out;
    }
  } else {
    const I n = (I)a.B * nQT * nQT;
    for (I e = tid; e < n; e += stride) {
      const I row = e / nQT;
      const I u = e - row * nQT;
      const I b = row / nQT, t = row - b * nQT;
      const I v_lo = (t > (I)L.band_tiles ? t - (I)L.band_tiles : 0) / 16, v = u / 16;
      uint8_t c = 0;
      if (v < v_lo) c = far[(size_t)b * L.far_stride + u];
      else if (v <= t / 16) c = mix[((size_t)row * Kc + (v - v_lo)) * 16 + (u - 16 * v)];
      a.cls[e] = c;
    }
  }
}

}  // namespace

int sm_count() {
  static int cached[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (!cached[dev]) {
    int n = 0;
    cached[dev] = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && n > 0 ? n : 148;
  }
  return cached[dev];
}

size_t blockmap_scratch_bytes(int B, int T, int window) {
  if (B < 1 || T < 1 || window < 0) return 0;
  return layout_of(B, T, window).total;
}

cudaError_t launch_blockmap(const BlockmapArgs& a, cudaStream_t st) {
  if (a.B == 0 || a.T == 0) return cudaSuccess;
  const Layout L = layout_of(a.B, a.T, a.window);
  const size_t stage = stage_far_offset(L.nW) + L.far_stride;
  const int staged = stage <= (size_t)kStageBytes ? 1 : 0;
  const size_t smem = staged ? stage : 0;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(sep_scan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kStageBytes);
    if (e != cudaSuccess) return e;
  }
  sep_scan_kernel<<<a.B, kScanThreads, smem, st>>>(a, staged);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess || !a.cls) return e;
  const int vec = (L.nQT % 16 == 0 && (reinterpret_cast<uintptr_t>(a.cls) & 15) == 0) ? 1 : 0;
  const long long items = (long long)a.B * L.nQT * L.nQT / (vec ? 16 : 1);
  const long long want = (items + kClassThreads - 1) / kClassThreads;
  const long long cap = (long long)sm_count() * (2048 / kClassThreads);
  const unsigned grid = (unsigned)(want < cap ? want : cap);
  // 32-bit indices while e + stride cannot wrap
  if (items + (long long)grid * kClassThreads < (1ll << 32))
    tile_class_kernel<uint32_t><<<grid, kClassThreads, 0, st>>>(a, vec);
  else
    tile_class_kernel<unsigned long long><<<grid, kClassThreads, 0, st>>>(a, vec);
  return cudaGetLastError();
}

}  // namespace sattn
