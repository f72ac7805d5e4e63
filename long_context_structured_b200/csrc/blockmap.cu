// blockmap.cu -- K2: block map and separator compaction.
//
// Structural mask of query row i ("LM-Infinite", section 方法, equation A_i;
// "SepLLM", section 五.2, mask M_ij), top-k excluded:
//   m_ij = [j <= i] * ( [j < n_start] + [i - j <= w] + [sep_j and j < i] > 0 ).
// Outputs, per sequence b:
//   prefix[b][x]   number of separators j >= n_start with j < x, x in [0, T]
//   sep_pos[b][r]  their positions in ascending order, then -1
//   sep_count[b]
//   ranges[b][t]   (#sep with j < 128t - w, #sep with j < last_row(t) - w)
//   cls[b][t][u]   0 empty / 1 partial / 2 full for the 128x128 tile (t, u)
//                  over its in-range (i, j) pairs.
// The classes follow from interval arithmetic on the sink span and the band
// plus separator counts from `prefix`; no mask is materialised.
#include "kernels.cuh"

namespace sattn {

namespace {

constexpr int kScanThreads = 1024;

__global__ void __launch_bounds__(kScanThreads) sep_scan_kernel(BlockmapArgs a) {
  __shared__ int warp_tot[32];
  __shared__ int total_sh;
  const int b = blockIdx.x;
  const int T = a.T;
  const int chunk = (T + kScanThreads - 1) / kScanThreads;
  const int j0 = threadIdx.x * chunk;
  const int j1 = min(T, j0 + chunk);
  const uint8_t* f = a.is_sep ? a.is_sep + (size_t)b * T : nullptr;
  int cnt = 0;
  if (f)
    for (int j = max(j0, a.n_start); j < j1; ++j) cnt += f[j] != 0;
  // block exclusive scan of cnt
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = cnt;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int v = warp_tot[lane];
    int s = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int u = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += u;
    }
    warp_tot[lane] = s - v;  // exclusive prefix of warp totals
    if (lane == 31) total_sh = s;
  }
  __syncthreads();
  int run = warp_tot[warp] + incl - cnt;
  int32_t* pre = a.prefix + (size_t)b * (T + 1);
  int32_t* pos = a.sep_pos + (size_t)b * T;
  for (int j = j0; j < j1; ++j) {
    pre[j] = run;
    if (f && j >= a.n_start && f[j]) pos[run++] = j;
  }
  const int total = total_sh;
  if (threadIdx.x == 0) {
    pre[T] = total;
    a.sep_count[b] = total;
  }
  for (int x = total + threadIdx.x; x < T; x += kScanThreads) pos[x] = -1;
}

__device__ __forceinline__ int pre_at(const int32_t* pre, int T, int x) {
  x = max(0, min(T, x));
  return pre[x];
}

// one CTA per (b, t); threads over key tiles u
__global__ void tile_class_kernel(BlockmapArgs a, int nQT, int nKT) {
  const int t = blockIdx.x;
  const int b = blockIdx.y;
  const int T = a.T, ns = a.n_start, w = a.window;
  const int32_t* pre = a.prefix + (size_t)b * (T + 1);
  const int i0 = t * kTile;
  const int i1 = min(T - 1, i0 + kTile - 1);
  if (threadIdx.x == 0) {
    a.ranges[((size_t)b * nQT + t) * 2 + 0] = pre_at(pre, T, i0 - w);
    a.ranges[((size_t)b * nQT + t) * 2 + 1] = pre_at(pre, T, i1 - w);
  }
  if (!a.cls) return;
  for (int u = threadIdx.x; u < nKT; u += blockDim.x) {
    const int j0 = u * kTile;
    const int j1 = min(T - 1, j0 + kTile - 1);
    uint8_t c;
    if (j0 > i1) {
      c = 0;
    } else {
      // full: causal for every row, and every key either a sink, inside the
      // band of the last row, or a separator (j < i holds since j <= i0 <= i
      // and j = i lies in the band)
      bool full = false;
      if (j1 <= i0) {
        const int lo = max(j0, ns);
        const int hi = min(j1, i1 - w - 1);  // keys that need the separator rule
        if (lo > hi) {
          full = true;
        } else {
          const int seps = pre_at(pre, T, hi + 1) - pre_at(pre, T, lo);
          full = (seps == hi - lo + 1);
        }
      }
      if (full) {
        c = 2;
      } else {
        bool any = (j0 < ns) || (j1 >= max(i0, j0) - w);
        if (!any) {
          const int lo = max(j0, ns);
          const int hi = min(j1, i1 - 1);
          if (lo <= hi) any = (pre_at(pre, T, hi + 1) - pre_at(pre, T, lo)) > 0;
        }
        c = any ? 1 : 0;
      }
    }
    a.cls[((size_t)b * nQT + t) * nKT + u] = c;
  }
}

}  // namespace

cudaError_t launch_blockmap(const BlockmapArgs& a, cudaStream_t st) {
  if (a.B == 0 || a.T == 0) return cudaSuccess;
  sep_scan_kernel<<<a.B, kScanThreads, 0, st>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int nQT = (a.T + kTile - 1) / kTile;
  const int nKT = nQT;
  dim3 grid(nQT, a.B);
  tile_class_kernel<<<grid, 128, 0, st>>>(a, nQT, nKT);
  return cudaGetLastError();
}

}  // namespace sattn
